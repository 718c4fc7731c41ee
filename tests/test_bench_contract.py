"""bench.py's host logic on a machine without a GPU: the algorithmic work and roofline
arithmetic behind the reported `roofline` object, the GEMM variant rule (against the
kernel's own constants), the traffic lookup's key, and the reference arm's JSON line (the
oracle timed on the host cores)."""
import json
import os
import re
import subprocess
import sys

import pytest

import workloads as WL

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PEAKS = dict(hbm_gbs=6000.0, bf16_tflops=1500.0, bf16_tflops_sustained=1200.0, source="test")


def test_algorithmic_work_of_a_step():
    cfg = WL.CONFIGS["cfg1"]                        # V 126464, d 4096, B 1, L 4096, k 32
    a = bench.algorithmic(cfg, 1024)
    assert a["flops"] == 2 * 1024 * 126464 * 4096
    # W once, the masked rows once, the mask, tok/conf/lse per row, idx/tok_sel/n_sel
    assert a["bytes"] == (2 * 126464 * 4096 + 2 * 1024 * 4096 + 4096 + 12 * 1024
                          + 4 * (2 * 32 + 1))


def test_gemm_roofline_peak_follows_the_region_length():
    """Burst peak for a short timed region, sustained peak from LONG_REGION_S on, fixed by
    the region's length (not by a throttle flag); both fractions always reported."""
    cfg = WL.CONFIGS["cfg1"]
    M = 1024
    t = 2.0 * M * cfg.V * cfg.d / 1000e12            # a launch running at 1000 TFLOP/s
    r = bench.gemm_roofline(cfg, M, PEAKS, t, True, "lmhead_auto_kernel<0>", region_s=0.014)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(1000.0)
    assert r["peak"] == 1500.0 and r["frac"] == pytest.approx(1000 / 1500)
    long_ = bench.gemm_roofline(cfg, M, PEAKS, t, True, "lmhead_auto_kernel<0>",
                                region_s=bench.LONG_REGION_S, sm_mhz=1250.0)
    assert long_["peak"] == 1200.0 and long_["frac"] == pytest.approx(1000 / 1200)
    assert long_["frac_of_burst"] == pytest.approx(1000 / 1500)
    assert long_["frac_of_sustained"] == pytest.approx(1000 / 1200)
    assert long_["tflops_per_ghz"] == pytest.approx(800.0)
    assert long_["gemm_mcycles"] == pytest.approx(t * 1250.0)


def test_clock_summary():
    s = bench.summarize_clock_samples([(1965.0, 1965.0, 400.0, set()),
                                       (1400.0, 1965.0, 990.0, {"sw_power_cap"}),
                                       (1300.0, 1965.0, 1000.0, {"sw_power_cap"})])
    assert s["samples"] == 3 and s["sm_mhz"] == 1400.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["power_w"] == 990.0
    assert bench.summarize_clock_samples([])["samples"] == 0


def test_default_workload_is_the_largest_single_gpu_config():
    cfg = WL.CONFIGS[bench.DEFAULT_CONFIG]
    assert (cfg.B, cfg.L, cfg.d, cfg.V, cfg.r) == (1, 131072, 4096, 126464, 0.9)
    assert max(c.B * c.L * c.r if c.mask == "bernoulli" else 0 for c in WL.CONFIGS.values()) \
        == cfg.B * cfg.L * cfg.r
    assert 50 <= bench.default_steps(cfg) <= 200                 # ~10 s of ~0.1 s steps
    assert bench.default_steps(WL.CONFIGS["cfg1"]) == 1000
    assert bench.default_steps(WL.CONFIGS["cfg0"]) == 1000


def test_gemm_roofline_hbm_bound():
    cfg = WL.CONFIGS["cfg1_m64"]
    M = 64
    nbytes = 2.0 * cfg.V * cfg.d + 2.0 * M * cfg.d
    r = bench.gemm_roofline(cfg, M, PEAKS, nbytes / 5000e9, False, "lmhead_auto_kernel<0>")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(5000.0) and r["frac"] == pytest.approx(5000 / 6000)
    assert r["algorithmic_bytes"] == nbytes


def test_bound_switches_at_the_ridge_point():
    """Flops 2MVd at P against bytes 2d(V + M) at BW: the tensor pipe bounds the GEMM from
    M* = V / (V BW / P - 1) rows up (about 250.5 rows for V = 126464 at these peaks)."""
    cfg = WL.CONFIGS["cfg1"]
    ratio = PEAKS["hbm_gbs"] * 1e9 / (PEAKS["bf16_tflops"] * 1e12)
    m_star = cfg.V / (cfg.V * ratio - 1.0)
    assert 250 < m_star < 251
    bound = lambda m: bench.gemm_roofline(cfg, m, PEAKS, 1e-3, True, "k")["bound"]
    assert bound(250) == "hbm" and bound(251) == "tensor"


def test_gemm_variant_rule_matches_the_kernel():
    text = open(os.path.join(ROOT, "mask_only_logits_b200", "csrc", "lmhead.cuh")).read()
    single = int(re.search(r"kSingleMaxRows\s*=\s*(\d+)", text).group(1))
    assert re.search(r"auto_variant\(int count\) \{ return count > kSingleMaxRows \? 2 : 1; \}", text)
    for c in (1, single, single + 1, 1024, 16384, 16385, 117961):
        assert bench.gemm_paired(0, c) == (c > single), c
    assert not bench.gemm_paired(1, 1024) and bench.gemm_paired(2, 10)


def test_traffic_is_reported_only_for_the_captured_code(tmp_path, monkeypatch):
    rec = dict(captures=[dict(workload="cfg1", kernel="lmhead_auto_kernel<0>",
                              source_sha256=bench.gemm_source_hash(),
                              dram_read_bytes=1000, dram_write_bytes=24)])
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.measured_traffic("cfg1", "lmhead_auto_kernel<0>") == 1024
    assert bench.measured_traffic("cfg2", "lmhead_auto_kernel<0>") is None
    assert bench.measured_traffic("cfg1", "lmhead_auto_kernel<1>") is None
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "another version")
    assert bench.measured_traffic("cfg1", "lmhead_auto_kernel<0>") is None


def test_source_hash_ignores_comments_only():
    h = bench.gemm_source_hash()
    assert re.fullmatch(r"[0-9a-f]{64}", h) and h == bench.gemm_source_hash()


def _run_bench(args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_json_line():
    res = _run_bench(["--impl", "reference", "--config", "cfg0", "--steps", "3", "--warmup", "3",
                      "--ref-seconds", "3"])
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["steps"] == 3 and d["warmup"] == 3 and d["higher_is_better"]
    assert d["vs_baseline"] is None and d["data"] == "synthetic" and d["dtype"] == "f64"
    assert d["config"]["workload"].startswith("cfg0")
    # the config names the workload only, exactly as the library's arm reports it
    assert d["config"] == bench.workload_config(WL.CONFIGS["cfg0"], d["config"]["masked_rows"])
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["host_cpus"] >= 1 and cb["blas"] and cb["sample"]
    assert d["e2e"] == dict(value=d["value"], unit=d["unit"], h2d_bytes_per_step=0,
                            d2h_bytes_per_step=0)


def test_reference_arm_other_ranks_do_nothing():
    res = _run_bench(["--impl", "reference", "--config", "cfg0", "--steps", "3", "--warmup", "3"],
                     dict(RANK="1", WORLD_SIZE="2"))
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == ""


def test_library_arm_refuses_to_run_without_a_gpu():
    """The library's arm has no CPU fallback: on a machine without CUDA it exits non-zero
    at once, naming the reason, and prints no result line."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    res = _run_bench(["--config", "cfg0", "--steps", "3", "--warmup", "3"])
    assert res.returncode != 0
    assert "needs a CUDA device" in res.stderr
    assert res.stdout.strip() == ""
