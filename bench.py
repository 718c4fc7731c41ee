"""Benchmark of the diffusion-LLM decode step: mask-only logits + confidence unmasking.

One step = the whole hot path on one batch: mask compaction, masked-row gather, the
tensor-core LM head with the fused softmax-statistics epilogue, lse_merge and the
per-sequence top-k unmask selection (``dllm_decode_step``).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config cfg3_r0.9] [--impl ours|reference]

The default workload is the largest one that fits one GPU: B1 L131072 d4096 V126464 with
90% of the positions masked (the 128k-context, high-mask-ratio case of the Mosaic page,
Fig. 3, where the logits are the memory peak).  Prints ONE JSON line (rank 0).  ``value``
= masked rows per second over the whole job (device time, inputs resident in HBM);
``e2e`` = the same through ``DecodeStep.run_host_pipeline`` with each step's mask and
masked rows of H read from pinned host memory and the selection copied back, every step.
``config`` names the workload only (identical in both arms); how the steps were launched
is under ``run``.  Under torchrun each rank runs its own replica of the workload (weak scaling,
no data-path collective): the decode steps of independent batches share nothing.
``--impl reference`` times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as WL  # noqa: E402

METRIC = "masked rows/sec & TFLOP/s (frac of roofline) for mask-only logits+unmask"
UNIT = "masked_rows/s"


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


GEMM_SOURCES = ["mask_only_logits_b200/csrc/lmhead.cuh", "mask_only_logits_b200/csrc/ptx.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "lmhead_traffic.json")


def gemm_source_hash() -> str:
    """SHA-256 of the GEMM's code: its sources with comments and whitespace removed, so that
    an edited comment does not void a capture while any change to the code does."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        text = open(os.path.join(ROOT, rel)).read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)        # block comments
        text = re.sub(r"//[^\n]*", " ", text)                      # line comments
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()


def measured_traffic(workload: str, kernel: str):
    """DRAM bytes (read + write) per GEMM launch from the committed ncu capture, if it was
    taken on this workload and kernel and the GEMM's sources have not changed since."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    rec = json.load(open(TRAFFIC_FILE))
    for c in rec.get("captures", []):
        if (c["workload"] == workload and c["kernel"] == kernel
                and c["source_sha256"] == gemm_source_hash()):
            return c["dram_read_bytes"] + c["dram_write_bytes"]
    return None


def algorithmic(cfg, M: int) -> dict:
    """Work of one step: flops of the dense contraction and bytes that must move once."""
    flops = 2.0 * M * cfg.V * cfg.d
    bytes_ = (2.0 * cfg.V * cfg.d          # W once
              + 2.0 * M * cfg.d            # masked rows of H once
              + cfg.B * cfg.L              # mask
              + 12.0 * M                   # tok, conf, lse
              + 4.0 * cfg.B * (2 * cfg.k + 1))   # idx, tok_sel, n_sel
    return dict(flops=flops, bytes=bytes_)


def roofline_s(cfg, M: int, peaks: dict) -> float:
    a = algorithmic(cfg, M)
    return max(a["flops"] / (peaks["bf16_tflops"] * 1e12), a["bytes"] / (peaks["hbm_gbs"] * 1e9))


def gemm_paired(variant: int, count: int) -> bool:
    """Whether the GEMM runs on CTA pairs: forced (1, 2), or the library's choice from the
    masked count (pairs above 128 rows)."""
    return variant == 2 or (variant == 0 and count > 128)


# A timed region at least this long runs in the regime of the measured sustained bf16 rate
# (a seconds-long GEMM loop under the 1 kW power cap); shorter ones in the burst regime.
LONG_REGION_S = 1.0


def gemm_roofline(cfg, count: int, peaks: dict, gemm_s: float, paired: bool, kernel: str,
                  region_s: float = 0.0, sm_mhz: float | None = None) -> dict:
    """Roofline of the dominant kernel (the masked LM-head GEMM with its fused epilogue):
    the tensor pipe when its flops take longer than its bytes at the measured peaks, else
    HBM.  Algorithmic work per launch: 2 * count * V * d flops; bytes = W once (2 V d) plus
    the gathered masked rows once (2 count d).

    The tensor peak follows the length of the timed region the GEMM ran in, fixed in
    advance: the measured burst bf16 rate for a short region (the kernel in the burst
    regime, before the power cap takes hold), the measured sustained rate when the region
    lasts LONG_REGION_S or more (steps of a long loop, as that figure was measured).  Both
    fractions are always reported.  With the median SM clock of the region, the GEMM's
    duration in clock cycles and its rate per GHz are reported too, so that runs at
    different capped clocks can be compared."""
    flops = 2.0 * count * cfg.V * cfg.d
    gemm_bytes = 2.0 * cfg.V * cfg.d + 2.0 * count * cfg.d
    tensor_bound = flops / (peaks["bf16_tflops"] * 1e12) >= gemm_bytes / (peaks["hbm_gbs"] * 1e9)
    out = dict(bound="tensor" if tensor_bound else "hbm",
               kernel=("masked_lmhead, " + ("paired-SM" if paired else "single-SM") +
                       f" tcgen05 ({kernel})" if kernel.startswith("lmhead_kernel") else
                       "masked_lmhead, " + kernel))
    tflops = flops / gemm_s / 1e12
    gbs = gemm_bytes / gemm_s / 1e9
    if tensor_bound:
        sustained = peaks.get("bf16_tflops_sustained")
        use_sustained = region_s >= LONG_REGION_S and sustained is not None
        peak = sustained if use_sustained else peaks["bf16_tflops"]
        out.update(achieved=tflops, peak=peak, unit="TFLOP/s", frac=tflops / peak,
                   frac_of_burst=tflops / peaks["bf16_tflops"],
                   frac_of_sustained=tflops / sustained if sustained else None,
                   peak_source=peaks["source"] + (
                       f" sustained bf16 GEMM (timed region of {region_s:.1f} s >= "
                       f"{LONG_REGION_S:g} s)" if use_sustained else
                       f" burst bf16 GEMM (timed region of {region_s:.3f} s)"),
                   achieved_gbs=gbs)
    else:
        out.update(achieved=gbs, peak=peaks["hbm_gbs"], unit="GB/s", frac=gbs / peaks["hbm_gbs"],
                   peak_source=peaks["source"] + " (HBM copy)", achieved_tflops=tflops)
    out.update(gemm_ms_avg=gemm_s * 1e3, algorithmic_bytes=gemm_bytes, algorithmic_flops=flops,
               traffic=measured_traffic(cfg.name, kernel))
    if sm_mhz:
        out.update(sm_mhz_median=sm_mhz, gemm_mcycles=gemm_s * sm_mhz,
                   tflops_per_ghz=tflops / (sm_mhz / 1e3))
    return out


# ------------------------------------------------------------------------------ clocks
_REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def _nvml_reason_bits(nv) -> dict:
    """NVML's clock-event reason bits for the four reasons the record reports."""
    g = lambda new, old: getattr(nv, new, getattr(nv, old, 0))
    return {"hw_slowdown": g("nvmlClocksEventReasonHwSlowdown", "nvmlClocksThrottleReasonHwSlowdown"),
            "hw_thermal_slowdown": g("nvmlClocksEventReasonHwThermalSlowdown",
                                     "nvmlClocksThrottleReasonHwThermalSlowdown"),
            "sw_thermal_slowdown": g("nvmlClocksEventReasonSwThermalSlowdown",
                                     "nvmlClocksThrottleReasonSwThermalSlowdown"),
            "sw_power_cap": g("nvmlClocksEventReasonSwPowerCap", "nvmlClocksThrottleReasonSwPowerCap")}


def summarize_clock_samples(samples: list) -> dict:
    """Median SM clock, the highest max clock, median power and every reason seen, over
    samples of (sm_mhz, max_mhz, power_w, set of active reason names)."""
    if not samples:
        return dict(sm_mhz=None, sm_max_mhz=None, reasons=[], samples=0)
    sm = [x[0] for x in samples]
    pw = [x[2] for x in samples if x[2] is not None]
    reasons = sorted(set().union(*[x[3] for x in samples]))
    return dict(sm_mhz=statistics.median(sm), sm_max_mhz=max(x[1] for x in samples),
                reasons=reasons, samples=len(samples),
                power_w=statistics.median(pw) if pw else None)


class ClockSampler:
    """SM clock, power and throttle reasons of the GPU the bench runs on, sampled while the
    timed region runs: read-only NVML queries from a thread every `period_ms`, plus one
    sample as the region starts and one as it ends, so that even a region of a few
    milliseconds carries its own record.  Falls back to an `nvidia-smi --query-gpu` loop
    when NVML cannot be loaded."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device, period_ms: int = 20):
        self.device = device
        self.period = period_ms
        self.samples: list = []
        self.source = None
        self._nv = self._handle = None
        self._stop = threading.Event()
        self._t = None
        self.proc = None

    # ---- NVML
    def _open_nvml(self) -> bool:
        try:
            import pynvml as nv
            nv.nvmlInit()
            props = torch.cuda.get_device_properties(self.device)
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            self._handle = nv.nvmlDeviceGetHandleByPciBusId(bus)
            self._nv = nv
            self._bits = _nvml_reason_bits(nv)
            self._max = nv.nvmlDeviceGetMaxClockInfo(self._handle, nv.NVML_CLOCK_SM)
            self._sample()
            return True
        except Exception:  # noqa: BLE001 - no NVML: fall back to nvidia-smi
            self._nv = None
            return False

    def _sample(self):
        nv, h = self._nv, self._handle
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        try:
            pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        except Exception:  # noqa: BLE001
            pw = None
        get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        bits = get(h)
        active = {name for name, b in self._bits.items() if b and bits & b}
        self.samples.append((float(sm), float(self._max), pw, active))

    def _loop(self):
        while not self._stop.wait(self.period / 1000.0):
            try:
                self._sample()
            except Exception:  # noqa: BLE001
                return

    # ---- nvidia-smi fallback
    def _open_smi(self):
        idx = torch.device(self.device).index or 0
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={idx}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", f"-lms={self.period}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read_smi, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx, pw = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            active = {n for n, f in zip(_REASON_NAMES, parts[5:9]) if f.lower() == "active"}
            self.samples.append((sm, mx, pw, active))

    def __enter__(self):
        if self._open_nvml():
            self.source = "nvml"
            self._t = threading.Thread(target=self._loop, daemon=True)
            self._t.start()
        else:
            self.source = "nvidia-smi"
            self._open_smi()
        return self

    def __exit__(self, *exc):
        if self._nv is not None:
            self._stop.set()
            if self._t is not None:
                self._t.join(timeout=5)
            try:
                self._sample()
                self._nv.nvmlShutdown()
            except Exception:  # noqa: BLE001
                pass
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self._t is not None:
                self._t.join(timeout=5)

    def summary(self) -> dict:
        out = summarize_clock_samples(self.samples)
        out["source"] = self.source
        return out


# ---------------------------------------------------------------------------- oracle leg
class OracleRunner:
    """The fp64 CPU oracle on one workload, for timing: the inputs' bf16 bits, the mask's
    compaction and W in fp64 are prepared once (W is the resident model weight, converted
    once as the GPU path uploads it once); ``time_rows`` then times the oracle's logits
    statistics for a set of compacted rows plus the unmask selection over them."""

    def __init__(self, inp: dict):
        import oracle.oracle as O
        self.O = O
        self.k = inp["k"]
        self.Hb, self.Wb = WL.bf16_bits(inp["H"]), WL.bf16_bits(inp["W"])
        M = inp["M"].numpy()
        if inp["cfg"].block_only:
            M = O.window_mask(M, inp["win_lo"], inp["win_hi"])
        self.L = M.shape[1]
        self.row_idx, self.seq_off, self.count = O.mask_compact(M)
        self.W64 = O.bf16_bits_to_f64(self.Wb)

    def time_rows(self, rows: np.ndarray) -> tuple[float, float]:
        """(seconds, rows) for the oracle on these compacted rows."""
        O = self.O
        t0 = time.perf_counter()
        ref = O.rows_stats_chunked(self.Hb[self.row_idx[rows]], self.Wb, W64=self.W64)
        O.select_unmask(ref[3], self.row_idx[rows], np.array([0, rows.size]), self.L, self.k)
        return time.perf_counter() - t0, float(rows.size)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"), default=1)
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def blas_backend() -> str:
    """The BLAS library NumPy's matmul runs on, with its version (e.g. "openblas 0.3.29")."""
    try:
        from threadpoolctl import threadpool_info
        libs = [f"{i.get('internal_api')} {i.get('version')}" for i in threadpool_info()
                if i.get("user_api") == "blas"]
        return ", ".join(libs) or "unknown"
    except Exception:  # noqa: BLE001
        return "unknown"


def cpu_baseline(inp: dict, budget_s: float = 10.0) -> dict:
    """The oracle on a bounded sample of the workload's masked rows: the sample doubles until
    one run takes about budget_s; when every masked row fits in less, whole passes over the
    workload repeat until budget_s is spent.  Rows per second over the reported runs."""
    cfg = inp["cfg"]
    run = OracleRunner(inp)
    count = run.count
    rng = np.random.default_rng(0)
    n_rows = min(count, 32)
    while True:
        rows = np.sort(rng.choice(count, size=n_rows, replace=False))
        t, n = run.time_rows(rows)
        if t >= budget_s or n_rows == count:
            break
        n_rows = min(count, max(2 * n_rows, int(n_rows * budget_s / max(t, 1e-3))))
    passes = 1
    while t < budget_s and n_rows == count:           # the whole workload, again
        t1, n1 = run.time_rows(rows)
        t, n, passes = t + t1, n + n1, passes + 1
    what = (f"{n_rows} of {count} masked rows" if passes == 1 else
            f"all {count} masked rows, {passes} passes")
    return dict(value=n / t, unit=UNIT, cores=blas_threads(), kind="oracle",
                host_cpus=os.cpu_count(), blas=blas_backend(),
                sample=f"{what} of {cfg.name} (fp64 NumPy logits over all V={cfg.V} with W "
                       f"converted once, statistics, top-k over the sample), {t:.1f} s")


def run_reference(args, cfg) -> None:
    """The oracle as the reference arm: rank 0 only, on the host cores.  Each step times the
    oracle on a random sample of the workload's masked rows, sized from a measured per-row
    cost so that warm-up and timed steps together take about --ref-seconds (two minutes)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = WL.make_inputs(cfg, seed=0)
    run = OracleRunner(inp)
    count = run.count
    rng = np.random.default_rng(0)
    pick = lambda n: np.sort(rng.choice(count, size=min(count, n), replace=False))
    t8, n8 = run.time_rows(pick(8))
    t32, n32 = run.time_rows(pick(32))
    per_row = max((t32 - t8) / max(n32 - n8, 1.0), t32 / max(n32, 1.0) * 0.5, 1e-6)
    fixed = max(t8 - n8 * per_row, 0.0)
    per_step = args.ref_seconds / max(1, args.steps + args.warmup)
    rows_per_step = int(max(1, min(count, (per_step - fixed) / per_row)))
    for _ in range(args.warmup):
        run.time_rows(pick(rows_per_step))
    tot_t, tot_n = 0.0, 0.0
    for _ in range(args.steps):
        t, n = run.time_rows(pick(rows_per_step))
        tot_t += t
        tot_n += n
    value = tot_n / tot_t
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=1e3 * tot_t / args.steps, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                config=workload_config(cfg, count),
                cpu_baseline=dict(value=value, unit=UNIT, cores=blas_threads(), kind="oracle",
                                  host_cpus=os.cpu_count(), blas=blas_backend(),
                                  sample=f"{rows_per_step} random masked rows per step of "
                                         f"{cfg.name} (W converted to fp64 once)"),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


DEFAULT_CONFIG = "cfg3_r0.9"


def default_steps(cfg) -> int:
    """Timed steps when none are given: about 10 s of steps at 70% of the step's roofline
    (the expected masked count), at least 20 and at most 1000."""
    peaks = load_peaks()
    if cfg.mask == "bernoulli":
        M = cfg.B * cfg.L * cfg.r
    elif cfg.mask == "suffix":
        M = cfg.B * cfg.n_suffix
    else:
        M = cfg.B * (cfg.block if cfg.block_only else cfg.L // 2)
    est = roofline_s(cfg, int(M), peaks) / 0.7 + 20e-6
    return int(min(1000, max(20, round(10.0 / est))))


def rows_of_step(inp: dict) -> int:
    """Masked rows whose logits one step computes: all masked positions, or with
    current-block-only logits those inside each sequence's window."""
    M = inp["M"].numpy() != 0
    if not inp["cfg"].block_only:
        return int(M.sum())
    pos = np.arange(M.shape[1])[None, :]
    inside = (pos >= inp["win_lo"][:, None]) & (pos < inp["win_hi"][:, None])
    return int((M & inside).sum())


def workload_config(cfg, count: int) -> dict:
    return dict(workload=f"{cfg.name}: {cfg.description}", B=cfg.B, L=cfg.L, d=cfg.d, V=cfg.V,
                k=cfg.k, masked_rows=count,
                l2="inputs larger than L2: W (%.2f GB) is streamed every step" % (2 * cfg.V * cfg.d / 1e9)
                if 2 * cfg.V * cfg.d > 126e6 else "L2-resident inputs (no flush)",
                parallelism="one independent replica per GPU")


# ------------------------------------------------------------------------------ our arm
def run_vocab_sharded(args, cfg) -> None:
    """One decode step with the vocabulary projection split by rows over the ranks
    (``sharded.VocabShardedStep``): every rank holds the same H and mask and its shard of W;
    the step's only exchange is an all-gather of the per-row partials.  Strong scaling: the
    job processes one step's masked rows per step whatever the number of ranks."""
    from mask_only_logits_b200 import dist as D
    info = D.rank_info()
    world, rank, local = info.world, info.rank, info.local_rank
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = D.init_process_group("nccl", timeout_s=120, device=dev) if world > 1 else None
    inp = WL.make_inputs(cfg, seed=0)                 # the same problem on every rank
    count = rows_of_step(inp)
    cpu = cpu_baseline(inp) if rank == 0 and world == 1 and not args.no_cpu_baseline else None
    import mask_only_logits_b200 as dl
    from mask_only_logits_b200.sharded import VocabShardedStep
    dl.debug_set_gemm_variant(args.gemm_variant)
    step = VocabShardedStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k, rank=rank, world=world, device=dev)
    H, M = inp["H"].to(dev), inp["M"].to(dev)
    W_shard = inp["W"][step.v0:step.v1].contiguous().to(dev)
    win_lo = None if inp["win_lo"] is None else torch.from_numpy(inp["win_lo"]).to(dev)
    win_hi = None if inp["win_hi"] is None else torch.from_numpy(inp["win_hi"]).to(dev)
    stream = torch.cuda.current_stream(dev)
    blk = cfg.block_only

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step.run(H, M, W_shard, win_lo, win_hi, stream, blk)
    torch.cuda.synchronize(dev)
    if dl.get_status(stream) != 0 or int(step.count[0]) != count:
        raise RuntimeError("warm-up failed")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step.run(H, M, W_shard, win_lo, win_hi, stream, blk)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    t_ms = ev0.elapsed_time(ev1)
    barrier()
    dl.prof_begin()
    for _ in range(args.steps):
        step.run(H, M, W_shard, win_lo, win_hi, stream, blk)
    torch.cuda.synchronize(dev)
    gemm_ms, gemm_launches, launches = dl.prof_end()
    if dl.get_status(stream) != 0:
        raise RuntimeError("device status after the timed region")
    t_ms, gemm_ms = D.max_over_ranks([t_ms, gemm_ms], dev)
    # end to end: H and the mask read from pinned host memory by the library's compaction
    # and gather kernels (only the mask and the masked rows cross the bus), the selection
    # copied back, every step
    e2e_steps = args.e2e_steps or args.steps
    H_host, M_host = inp["H"].pin_memory(), inp["M"].pin_memory()
    idx_host = torch.empty(cfg.B, cfg.k, dtype=torch.int32).pin_memory()
    step.run(H_host, M_host, W_shard, win_lo, win_hi, stream, blk)
    barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        step.run(H_host, M_host, W_shard, win_lo, win_hi, stream, blk)
        idx_host.copy_(step.idx, non_blocking=True)
    torch.cuda.synchronize(dev)
    e2e_ms = D.max_over_ranks([(time.perf_counter() - t0) * 1e3], dev)[0]
    barrier()
    if rank == 0:
        peaks = load_peaks()
        shard_cfg = WL.get_config(cfg.name, V=step.v1 - step.v0)
        ms_step = t_ms / args.steps
        clk_summary = clk.summary()
        roof = gemm_roofline(shard_cfg, count, peaks, gemm_ms / max(1, gemm_launches) / 1e3,
                             gemm_paired(args.gemm_variant, count), "vocabulary shard",
                             region_s=t_ms / 1e3, sm_mhz=clk_summary["sm_mhz"])
        roof["traffic"] = None
        roof["shard"] = f"rows [{step.v0}, {step.v1}) of W on rank 0"
        line = dict(
            metric=METRIC, value=count * args.steps / (t_ms / 1e3), unit=UNIT, n_gpus=world,
            steps=args.steps, warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True,
            scaling="strong", vs_baseline=None, dtype="bf16", data="synthetic",
            config=workload_config(cfg, count),
            run=dict(parallelism=f"vocabulary-parallel over {world} GPU(s)"),
            roofline=roof, gpu_launches=launches,
            e2e=dict(value=count * e2e_steps / (e2e_ms / 1e3), unit=UNIT,
                     h2d_bytes_per_step=cfg.B * cfg.L + 2 * cfg.d * count,
                     d2h_bytes_per_step=cfg.B * cfg.k * 4, ms_per_step=e2e_ms / e2e_steps,
                     note="every rank's kernels read the mask and the masked rows of H from "
                          "pinned host memory and the selection is copied back each step (no "
                          "overlap between steps); wall clock, max over ranks"),
            clocks=clk_summary)
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about 10 s of steps, 20 to 1000)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=DEFAULT_CONFIG,
                    help="workload (default: the largest single-GPU one, cfg3 at r_m = 0.9)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="--impl reference: oracle seconds that warm-up and timed steps take together")
    ap.add_argument("--no-full-baseline", action="store_true",
                    help="skip timing the full-logits torch path the method replaces")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--graph", action="store_true",
                    help="time replays of the step captured in a CUDA graph (one launch per step)")
    ap.add_argument("--serial", action="store_true",
                    help="run each step's staging (compaction, gather) on the compute stream "
                         "instead of overlapping it with the previous step's GEMM")
    ap.add_argument("--shard", default="replica", choices=["replica", "vocab"],
                    help="replica: one independent step per rank (weak scaling); vocab: one "
                         "step with W split by rows over the ranks (strong scaling)")
    ap.add_argument("--policy", default="confidence", choices=["confidence", "entropy", "margin"],
                    help="score the positions to unmask are ranked by (entropy / margin run the "
                         "GEMM's extended epilogue)")
    ap.add_argument("--threshold", type=float, default=None,
                    help="threshold-based parallel unmasking on the policy's score (default: top-k)")
    ap.add_argument("--gemm-variant", type=int, default=0, choices=[0, 1, 2],
                    help="0 = library default, 1 = single-SM GEMM, 2 = paired-SM GEMM")
    ap.add_argument("--arena", action="store_true",
                    help="the step's workspace in a virtual-memory arena mapped for the step's "
                         "own masked count (steps run one at a time); reports the mapped bytes "
                         "against the count's need and the fixed worst-case workspace")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    cfg = WL.CONFIGS[args.config]
    if args.steps is None:
        args.steps = default_steps(cfg)

    if args.impl == "reference":
        run_reference(args, cfg)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: the library's arm needs a CUDA device (there is no CPU "
                         "fallback); --impl reference times the oracle on the host")
    if args.shard == "vocab":
        run_vocab_sharded(args, cfg)
        return
    from mask_only_logits_b200 import dist as D
    info = D.rank_info()
    world, rank, local = info.world, info.rank, info.local_rank
    dist = None
    if world > 1:
        torch.cuda.set_device(local)
        dist = D.init_process_group("nccl", timeout_s=120, device=torch.device("cuda", local))

    # inputs (each rank its own seeded batch), and the oracle baseline before any GPU work
    inp = WL.make_inputs(cfg, seed=D.replica_seed(0, rank))
    count = rows_of_step(inp)
    blk = cfg.block_only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp)

    import mask_only_logits_b200 as dl
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    H = inp["H"].to(dev)
    M = inp["M"].to(dev)
    W = inp["W"].to(dev)
    win_lo = None if inp["win_lo"] is None else torch.from_numpy(inp["win_lo"]).to(dev)
    win_hi = None if inp["win_hi"] is None else torch.from_numpy(inp["win_hi"]).to(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    base_mem = torch.cuda.memory_allocated(dev)
    dl.debug_set_gemm_variant(args.gemm_variant)
    step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k, device=dev, policy=args.policy,
                         threshold=args.threshold, arena=args.arena)
    stream = torch.cuda.current_stream(dev)
    arena_rec = None
    if args.arena:
        # the host knows the step's masked count (it built the mask): map just that much
        torch.cuda.synchronize(dev)
        free0, _ = torch.cuda.mem_get_info(dev)
        need = step.size_for_rows(count)
        torch.cuda.synchronize(dev)
        free1, _ = torch.cuda.mem_get_info(dev)
        arena_rec = dict(workspace_need_bytes=int(need), mapped_bytes=step.arena.mapped,
                         device_bytes_taken=int(free0 - free1),
                         reserved_va_bytes=step.arena.reserved, chunk_bytes=step.arena.chunk,
                         fixed_workspace_bytes=dl.workspace_bytes(cfg.B, cfg.L, cfg.d, cfg.V),
                         note="workspace in a dllm_arena mapped for this step's masked count "
                              "(dllm_workspace_bytes_rows) against the fixed workspace sized "
                              "for every position masked; device_bytes_taken = drop of "
                              "cudaMemGetInfo's free bytes when the arena was mapped")

    def run_step(H_, M_):
        if args.arena:
            return step.run(H_, M_, W, win_lo, win_hi, stream, blk, max_rows=count)
        return step.run(H_, M_, W, win_lo, win_hi, stream, blk)

    for _ in range(args.warmup):
        run_step(H, M)
    torch.cuda.synchronize(dev)
    status = dl.get_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    if int(step.count[0]) != count:
        raise RuntimeError(f"the step computed {int(step.count[0])} rows, expected {count}")
    step_peak = torch.cuda.max_memory_allocated(dev) - base_mem

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # ---- device-resident timed region: the steps alone ----
    if args.graph:
        step.capture(H, M, W, win_lo, win_hi, blk)
        for _ in range(3):
            step.replay(stream)
        torch.cuda.synchronize(dev)

    overlap = not (args.graph or args.serial or args.arena)
    if overlap:
        # the staging of step i+1 (compaction of the mask, gather of the masked rows) runs
        # on a second stream while step i's GEMM and selection run on this one
        prep_stream = torch.cuda.Stream(dev)
        step.run_overlapped([(H, M)] * 3, W, win_lo, win_hi, stream, prep_stream, blk)
        torch.cuda.synchronize(dev)
        step_peak = torch.cuda.max_memory_allocated(dev) - base_mem   # with the 2nd workspace

    def one_step():
        if args.graph:
            step.replay(stream)
        else:
            run_step(H, M)

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        barrier()
        ev0.record(stream)
        if overlap:
            step.run_overlapped([(H, M)] * args.steps, W, win_lo, win_hi, stream, prep_stream,
                                blk)
        else:
            for _ in range(args.steps):
                one_step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    t_ms = ev0.elapsed_time(ev1)
    # ---- the same steps again with the library's CUDA events around every GEMM launch
    # (the dominant kernel's live duration) and its count of kernel launches; kept out of
    # the region above because an event between two kernels stops them from overlapping
    barrier()
    with ClockSampler(dev) as clk_gemm:
        dl.prof_begin()
        for _ in range(args.steps):
            run_step(H, M)
        torch.cuda.synchronize(dev)
        gemm_ms, gemm_launches, launches = dl.prof_end()
    status = dl.get_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    t_ms, gemm_ms = D.max_over_ranks([t_ms, gemm_ms], dev)
    # rows processed by the whole job per step: every rank's own batch (seeded per rank, so
    # Bernoulli masks give each rank its own count)
    job_rows = int(round(D.sum_over_ranks([count], dev)[0]))
    full_base = (full_logits_baseline(H, M, W, cfg.k, win_lo, win_hi, blk, dev)
                 if world == 1 and not args.no_full_baseline else None)
    torch.cuda.empty_cache()            # hand the baseline's logits back to the device

    # ---- end to end from pinned host memory ----
    # as many steps as the device-resident region, so that both settle into the same
    # power-capped clock (a short region partly runs before the cap takes hold)
    e2e_steps = args.e2e_steps or args.steps
    H_host = inp["H"].pin_memory()
    M_host = inp["M"].pin_memory()
    for _ in range(3):
        step.run_host(H_host, M_host, W, win_lo, win_hi, stream, blk)
    barrier()

    def host_steps(n):
        # the decode loop a serving process runs: each step's inputs copied in from pinned
        # host memory (overlapping the previous step) and its selection copied back; in
        # arena mode one step at a time (the mapping follows each step's mask)
        if args.arena:
            for _ in range(n):
                yield step.run_host(H_host, M_host, W, win_lo, win_hi, stream, blk)
        else:
            yield from step.run_host_pipeline([(H_host, M_host)] * n, W, win_lo, win_hi, stream,
                                              block_only=blk)

    for _ in host_steps(3):
        pass
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clk_e2e:
        barrier()
        t0 = time.perf_counter()
        n_out = 0
        for _ in host_steps(e2e_steps):
            n_out += 1
        torch.cuda.synchronize(dev)
        e2e_s = time.perf_counter() - t0
    e2e_ms = D.max_over_ranks([e2e_s * 1e3], dev)[0]
    assert n_out == e2e_steps
    barrier()

    if rank == 0:
        peaks = load_peaks()
        clk_summary = clk.summary()
        clk_gemm_summary = clk_gemm.summary()
        a = algorithmic(cfg, count)
        ms_step = t_ms / args.steps
        rows_s = job_rows * args.steps / (t_ms / 1e3)
        gemm_avg_s = gemm_ms / max(1, gemm_launches) / 1e3
        roof = roofline_s(cfg, count, peaks)
        step_tflops = a["flops"] / (ms_step / 1e3) / 1e12
        step_gbs = a["bytes"] / (ms_step / 1e3) / 1e9
        full_logits = cfg.B * cfg.L * cfg.V * 4
        paired = gemm_paired(args.gemm_variant, count)
        mode = 1 if step.stats else 0
        gemm_kernel_name = (f"lmhead_auto_kernel<{mode}>" if args.gemm_variant == 0 else
                            f"lmhead_kernel<{args.gemm_variant}, {mode}>")
        line = dict(
            metric=METRIC, value=rows_s, unit=UNIT, n_gpus=world, steps=args.steps,
            warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True, scaling="weak",
            vs_baseline=None, dtype="bf16", data="synthetic",
            config=workload_config(cfg, count),
            run=dict(masked_rows_all_ranks=job_rows, policy=args.policy,
                     threshold=args.threshold,
                     launch=("CUDA graph replay" if args.graph else
                             "one stream, steps in sequence, workspace in an arena" if args.arena
                             else "one stream, steps in sequence" if args.serial else
                             "two streams: staging of step i+1 overlaps step i")),
            tflops=step_tflops, gbs=step_gbs,
            roofline_frac_step=roof / (ms_step / 1e3),
            roofline_ms=roof * 1e3,
            roofline=gemm_roofline(cfg, count, peaks, gemm_avg_s, paired, gemm_kernel_name,
                                   region_s=t_ms / 1e3, sm_mhz=clk_gemm_summary["sm_mhz"]),
            gpu_launches=launches,
            memory=dict(peak_step_bytes=int(step_peak) if not args.arena else None,
                        full_logits_fp32_bytes=int(full_logits),
                        workspaces=1 if not overlap else 2,
                        note="peak = torch allocations of the step (outputs + workspace; two "
                             "workspaces when staging overlaps the previous step) over the "
                             "resident inputs; full_logits_fp32_bytes = B*L*V fp32 logits"),
            e2e=dict(value=job_rows * e2e_steps / (e2e_ms / 1e3), unit=UNIT,
                     h2d_bytes_per_step=(step.h2d_bytes() if args.arena else
                                         step.h2d_bytes_zero_copy(count)),
                     d2h_bytes_per_step=step.d2h_bytes(),
                     ms_per_step=e2e_ms / e2e_steps, steps=e2e_steps,
                     clocks=clk_e2e.summary(),
                     note="DecodeStep.run_host_pipeline: per step, the mask and the masked rows "
                          "of H are read from pinned host memory by the library's compaction "
                          "and gather kernels (only those bytes cross the bus) on a staging "
                          "stream, overlapping the previous step's GEMM; the selection is "
                          "copied back to pinned memory; wall clock, device synchronised at "
                          "both ends"),
            clocks=clk_summary,
            clocks_gemm_pass=clk_gemm_summary,
        )
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if full_base is not None:
            line["full_logits_baseline"] = full_base
        if arena_rec is not None:
            line["memory"]["arena"] = arena_rec
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def full_logits_baseline(H, M, W, k, win_lo, win_hi, block_only, dev, iters=10):
    """The path mask-only logits replaces, in plain torch on the same GPU: logits for every
    position (one cuBLAS bf16 GEMM, [B*L, V]), then the masked rows gathered, their fp32
    softmax statistics and the per-sequence top-k of the confidence.  Returns its time per
    step and the device bytes it allocates (None when the logits alone would exceed 48 GB)."""
    B, L = M.shape
    V = W.shape[0]
    if B * L * V * 2 > 48e9:
        return None
    lo = None if win_lo is None else win_lo.tolist()
    hi = None if win_hi is None else win_hi.tolist()

    def step():
        logits = H @ W.t()                                         # [B*L, V] bf16
        mask = M.reshape(-1) != 0
        if block_only:
            pos = torch.arange(L, device=dev).repeat(B)
            seq = torch.arange(B, device=dev).repeat_interleave(L)
            mask = mask & (pos >= win_lo[seq]) & (pos < win_hi[seq])
        rows = mask.nonzero().squeeze(1)
        z = logits.index_select(0, rows).float()
        mx, tok = z.max(dim=1)
        conf = torch.exp(mx - torch.logsumexp(z, dim=1))
        seq_of = rows // L
        sel = []
        for b in range(B):
            keep = seq_of == b
            if lo is not None:
                p = rows - b * L
                keep = keep & (p >= lo[b]) & (p < hi[b])
            c = conf[keep]
            sel.append(torch.topk(c, min(k, c.numel())).indices if c.numel() else c)
        return tok, sel

    torch.cuda.synchronize(dev)
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    for _ in range(3):
        step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        step()
    e1.record()
    torch.cuda.synchronize(dev)
    peak = torch.cuda.max_memory_allocated(dev) - base
    return dict(ms_per_step=e0.elapsed_time(e1) / iters, peak_bytes=int(peak),
                logits_bytes=int(B * L * V * 2),
                note="plain torch on the same GPU: cuBLAS bf16 logits for all B*L positions, "
                     "gather of the masked rows, fp32 max / logsumexp, per-sequence topk")


if __name__ == "__main__":
    main()
