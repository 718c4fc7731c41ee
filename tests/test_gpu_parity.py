"""End-to-end parity of the decode step (dllm_decode_step through the C ABI) against the
fp64 CPU oracle, on every workload at full size.

Bar: compaction and the unmask selection bit-exact (the selection on the GPU's own fp32
confidences; against the oracle's fp64 confidences, ties within the tolerance excepted);
lse and conf within 2e-3 relative; argmax exact except rows whose top-2 logit gap is below
1e-3.  cfg0 and cfg1 are checked on every masked row, the others on a seeded sample of
512 masked rows plus every selected row (and, for cfg4, every row of the unmask windows).
"""
import numpy as np
import pytest
import torch

import gpu_util as GU
import oracle.oracle as O
import workloads as WL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import mask_only_logits_b200 as dl
    return dl


def run_gpu(dl, inp):
    cfg = inp["cfg"]
    dev = GU.to_device(inp)
    step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, inp["k"])
    out = step.run(dev["H"], dev["M"], dev["W"], dev["win_lo"], dev["win_hi"],
                   block_only=cfg.block_only)
    assert dl.get_status() == 0
    c = int(out["count"][0])
    res = {key: out[key].cpu().numpy() for key in ("tok", "conf", "lse", "row_idx", "seq_off",
                                                   "idx", "n_sel", "tok_sel", "conf_sel")}
    res["count"] = c
    for key in ("tok", "conf", "lse", "row_idx"):
        res[key] = res[key][:c]
    del step, dev
    torch.cuda.empty_cache()
    return res


def check_step(dl, inp, all_rows: bool, window_rows: bool = False):
    cfg = inp["cfg"]
    Hb, Wb, M = GU.inputs_bits(inp)
    if cfg.block_only:             # current-block-only logits: the rows inside the windows
        M = O.window_mask(M, inp["win_lo"], inp["win_hi"])
    g = run_gpu(dl, inp)
    # compaction: bit-exact
    row_idx, seq_off, count = O.mask_compact(M)
    assert g["count"] == count
    np.testing.assert_array_equal(g["row_idx"], row_idx)
    np.testing.assert_array_equal(g["seq_off"], seq_off)
    # selection: bit-exact against the oracle's top-k of the GPU's own confidences
    GU.check_selection_exact(g["idx"], g["n_sel"], g["conf"], row_idx, seq_off, cfg.L, inp["k"],
                             inp["win_lo"], inp["win_hi"], O)
    # per-row statistics on the rows under test
    sel_rows = []
    for b in range(cfg.B):
        for p in g["idx"][b, :g["n_sel"][b]]:
            sel_rows.append(np.searchsorted(row_idx, b * cfg.L + p))
    if all_rows:
        rows = np.arange(count)
    else:
        rows = WL.sample_rows(count, 512, seed=0)
        extra = [np.asarray(sel_rows, dtype=np.int64)]
        if window_rows:
            for b in range(cfg.B):
                lo = np.searchsorted(row_idx, b * cfg.L + inp["win_lo"][b])
                hi = np.searchsorted(row_idx, b * cfg.L + inp["win_hi"][b])
                extra.append(np.arange(lo, hi))
        rows = np.unique(np.concatenate([rows] + extra)).astype(np.int64)
    ref = O.oracle_rows(Hb, Wb, M, rows)
    stats = GU.check_rows(g["tok"], g["conf"], g["lse"], ref, rows, cfg.name)
    # tok_sel / conf_sel are the tok / conf of the selected rows
    for b in range(cfg.B):
        n = g["n_sel"][b]
        r = [np.searchsorted(row_idx, b * cfg.L + p) for p in g["idx"][b, :n]]
        np.testing.assert_array_equal(g["tok_sel"][b, :n], g["tok"][r])
        np.testing.assert_array_equal(g["conf_sel"][b, :n], g["conf"][r])
    # selection against the oracle's own fp64 confidences where it knows every candidate
    if all_rows or window_rows:
        conf_by_row = dict(zip(rows.tolist(), ref["conf"].tolist()))
        ref_idx, ref_n = O.select_unmask(
            np.array([conf_by_row.get(i, -1.0) for i in range(count)]), row_idx, seq_off,
            cfg.L, inp["k"], inp["win_lo"], inp["win_hi"])

        def conf_of_pos(b, p):
            return conf_by_row[int(np.searchsorted(row_idx, b * cfg.L + p))]
        stats["selection_ties_excused"] = GU.check_selection_tolerant(
            g["idx"], g["n_sel"], ref_idx, ref_n, conf_of_pos)
    print(cfg.name, stats)
    return g, stats


def test_cfg0_every_row_and_full_logits_invariant(dl):
    inp = WL.make_inputs(WL.CONFIGS["cfg0"], seed=0)
    g, _ = check_step(dl, inp, all_rows=True)
    # the oracle's literal full-then-gather definition gives the same statistics
    Hb, Wb, M = GU.inputs_bits(inp)
    full = O.full_then_gather(Hb, Wb, M)
    GU.check_rows(g["tok"], g["conf"], g["lse"],
                  dict(tok=full["tok"], conf=full["conf"], lse=full["lse"],
                       gap=O.top2_gap(full["Z_full"][full["row_idx"]])),
                  np.arange(full["count"]), "cfg0-full")


@pytest.mark.parametrize("seed", [1, 2])
def test_cfg0_other_seeds(dl, seed):
    check_step(dl, WL.make_inputs(WL.CONFIGS["cfg0"], seed=seed), all_rows=True)


def test_cfg1_every_row(dl):
    check_step(dl, WL.make_inputs(WL.CONFIGS["cfg1"], seed=0), all_rows=True)


def test_cfg1_m64_every_row(dl):
    check_step(dl, WL.make_inputs(WL.CONFIGS["cfg1_m64"], seed=0), all_rows=True)


def test_cfg2_sampled(dl):
    check_step(dl, WL.make_inputs(WL.CONFIGS["cfg2"], seed=0), all_rows=False)


def test_cfg3_sweep_sampled(dl):
    names = ["cfg3_r0.1", "cfg3_r0.5", "cfg3_r0.9"]
    sweep = WL.make_sweep_inputs(names, seed=0)
    for n in names:
        check_step(dl, sweep[n], all_rows=False)


def test_cfg4_sampled_and_windows(dl):
    check_step(dl, WL.make_inputs(WL.CONFIGS["cfg4"], seed=0), all_rows=False, window_rows=True)


def test_cfg4_block_every_row(dl):
    """Current-block-only logits (dllm_decode_block_step) on cfg4: every in-window row
    against the oracle, and the same selection as the oracle's full windowed step."""
    inp = WL.make_inputs(WL.CONFIGS["cfg4_block"], seed=0)
    g, _ = check_step(dl, inp, all_rows=True)
    assert g["count"] == 8 * 32


@pytest.mark.parametrize("B,L,d,V,k,r", [(3, 1000, 128, 777, 5, 0.7), (5, 64, 64, 300, 40, 1.0),
                                         (2, 20000, 256, 4096, 16, 0.5)])
def test_block_only_random_windows(dl, B, L, d, V, k, r):
    """Block-only steps with windows of random placement and width (empty, inverted and
    out-of-range ones included) over Bernoulli masks."""
    inp = WL.make_inputs(WL.custom_config(B, L, d, V, k, r=r, block_only=True), seed=7)
    rng = np.random.default_rng(B + L)
    lo = rng.integers(-4, L, size=B)
    hi = lo + rng.integers(-2, max(3, L // 2), size=B)
    hi[0] = lo[0]                                           # one empty window
    inp["win_lo"], inp["win_hi"] = lo.astype(np.int32), hi.astype(np.int32)
    check_step(dl, inp, all_rows=True)


@pytest.mark.parametrize("B,L,d,V,k,mask,r", [
    (2, 300, 64, 257, 5, "bernoulli", 0.5),      # d = 64 (one K block), V tail of 1
    (3, 777, 192, 1000, 16, "bernoulli", 0.9),   # ragged everything
    (1, 64, 128, 255, 70, "bernoulli", 1.0),     # k larger than the masked count
    (2, 100, 64, 1, 3, "bernoulli", 0.5),        # V = 1: conf = 1, lse = the logit
    (4, 50, 64, 300, 4, "bernoulli", 0.0),       # nothing masked
    (1, 40000, 256, 4096, 1024, "bernoulli", 0.7),   # many m-tiles, largest k
    (1, 2048, 128, 5000, 16, "bernoulli", 1.0),      # 8 m-tiles of 256 rows
    (1, 1000, 64, 37800, 32, "bernoulli", 1.0),      # remainder holders (both variants)
    (1, 12000, 64, 3000, 8, "bernoulli", 0.08),      # sparse mask, few m-tiles of a long L
    (1, 3840, 64, 20000, 8, "bernoulli", 1.0),       # 30 m-tiles: tail split 18 + 12
    (1, 13300, 64, 5000, 8, "bernoulli", 1.0),       # 104 m-tiles: 2 full groups + 18 + 12
])
def test_edge_shapes(dl, B, L, d, V, k, mask, r):
    cfg = WL.custom_config(B, L, d, V, k, mask=mask, r=r)
    inp = WL.make_inputs(cfg, seed=5)
    check_step(dl, inp, all_rows=True)


def test_run_host_matches_device(dl):
    inp = WL.make_inputs(WL.CONFIGS["cfg0"], seed=0)
    cfg = inp["cfg"]
    dev = GU.to_device(inp)
    step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
    d_out = step.run(dev["H"], dev["M"], dev["W"])
    idx_dev = d_out["idx"].cpu().clone()
    h_out = step.run_host(inp["H"].pin_memory(), inp["M"].pin_memory(), dev["W"])
    assert torch.equal(h_out["idx"], idx_dev)
    assert step.h2d_bytes() == cfg.B * cfg.L * (cfg.d * 2 + 1)


@pytest.mark.parametrize("name", ["cfg0", "cfg1"])
def test_single_sm_variant(dl, name):
    """The single-SM (cta_group::1) GEMM variant meets the same bar."""
    dl.debug_set_gemm_variant(1)
    try:
        check_step(dl, WL.make_inputs(WL.CONFIGS[name], seed=0), all_rows=True)
        cfg = WL.custom_config(3, 777, 192, 1000, 16, r=0.9)
        check_step(dl, WL.make_inputs(cfg, seed=5), all_rows=True)
    finally:
        dl.debug_set_gemm_variant(0)


def test_pair_variant_large(dl):
    """The paired-SM (cta_group::2) GEMM on a large workload (default there: single SMs)."""
    dl.debug_set_gemm_variant(2)
    try:
        check_step(dl, WL.make_inputs(WL.CONFIGS["cfg4"], seed=0), all_rows=False, window_rows=True)
    finally:
        dl.debug_set_gemm_variant(0)


def test_run_host_pipeline_matches_device_steps(dl):
    """Overlapped staging must not mix batches: each yielded selection equals that batch's
    device-resident step."""
    cfg = WL.CONFIGS["cfg0"]
    inps = [WL.make_inputs(cfg, seed=s) for s in (0, 1, 2, 3, 4)]
    W = inps[0]["W"].cuda()                      # one resident W for every batch
    step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
    expected = []
    for inp in inps:
        out = step.run(inp["H"].cuda(), inp["M"].cuda(), W)
        expected.append((out["idx"].cpu().clone(), out["n_sel"].cpu().clone(),
                         out["tok_sel"].cpu().clone()))
    batches = [(inp["H"].pin_memory(), inp["M"].pin_memory()) for inp in inps]
    got = [(o["idx"].clone(), o["n_sel"].clone(), o["tok_sel"].clone())
           for o in step.run_host_pipeline(batches, W)]
    assert len(got) == len(expected)
    for (gi, gn, gt), (ei, en, et) in zip(got, expected):
        assert torch.equal(gi, ei) and torch.equal(gn, en) and torch.equal(gt, et)
    assert not all(torch.equal(got[0][0], g[0]) for g in got[1:])   # batches really differ


def test_pinned_host_inputs_match_device(dl):
    """H and the mask in page-locked host memory (read over the bus by the compaction and
    gather kernels) give bit-identical results to the same inputs in device memory."""
    for name, variant in (("cfg0", 0), ("cfg4", 0), ("cfg1_m64", 1)):
        inp = WL.make_inputs(WL.CONFIGS[name], seed=1)
        cfg = inp["cfg"]
        dev = GU.to_device(inp)
        dl.debug_set_gemm_variant(variant)
        try:
            step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
            a = {k: v.clone() for k, v in step.run(dev["H"], dev["M"], dev["W"], dev["win_lo"],
                                                   dev["win_hi"]).items()}
            b = step.run(inp["H"].pin_memory(), inp["M"].pin_memory(), dev["W"], dev["win_lo"],
                         dev["win_hi"])
            torch.cuda.synchronize()
            assert dl.get_status() == 0
            c = int(a["count"][0])
            assert int(b["count"][0]) == c
            for key in ("tok", "conf", "lse", "row_idx"):
                assert torch.equal(a[key][:c], b[key][:c]), (name, key)
            for key in ("idx", "n_sel", "tok_sel", "conf_sel", "seq_off"):
                assert torch.equal(a[key], b[key]), (name, key)
        finally:
            dl.debug_set_gemm_variant(0)


def test_pageable_host_input_rejected(dl):
    """Pageable host memory cannot be read by the kernels: rejected before any launch."""
    import ctypes
    inp = WL.make_inputs(WL.CONFIGS["cfg0"], seed=0)
    cfg = inp["cfg"]
    H_pageable = np.ascontiguousarray(WL.bf16_bits(inp["H"]))        # plain host memory
    n = cfg.B * cfg.L
    i32 = dict(dtype=torch.int32, device="cuda")
    outs = [torch.empty(n, **i32), torch.empty(n, device="cuda"), torch.empty(n, device="cuda"),
            torch.empty(n, **i32), torch.empty(cfg.B + 1, **i32), torch.empty(4, **i32)]
    ws = torch.empty(dl.workspace_bytes(cfg.B, cfg.L, cfg.d, cfg.V), dtype=torch.uint8, device="cuda")
    M, W = inp["M"].cuda(), inp["W"].cuda()
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = dl.lib().dllm_masked_logits(ctypes.c_void_p(H_pageable.ctypes.data), P(M), P(W), cfg.B,
                                     cfg.L, cfg.d, cfg.V, *[P(t) for t in outs], P(ws), ws.numel(),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == -10                                                   # DLLM_ERR_MEMORY
    assert dl.get_status() == 0


def test_host_pipeline_block_only_and_windows(dl):
    """The two-stream pipeline with current-block-only steps and with selection windows."""
    cfg = WL.custom_config(4, 1024, 128, 3000, 4, mask="semi_ar", block=32)
    inps = [WL.make_inputs(cfg, seed=s) for s in (3, 4, 5)]
    W = inps[0]["W"].cuda()
    lo, hi = WL.make_windows(cfg)
    lo_d, hi_d = torch.from_numpy(lo).cuda(), torch.from_numpy(hi).cuda()
    for block_only in (False, True):
        step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
        expected = []
        for inp in inps:
            out = step.run(inp["H"].cuda(), inp["M"].cuda(), W, lo_d, hi_d, block_only=block_only)
            expected.append((out["idx"].cpu().clone(), out["n_sel"].cpu().clone()))
        batches = [(inp["H"].pin_memory(), inp["M"].pin_memory()) for inp in inps]
        got = [(o["idx"].clone(), o["n_sel"].clone())
               for o in step.run_host_pipeline(batches, W, lo_d, hi_d, block_only=block_only)]
        assert len(got) == len(expected)
        for (gi, gn), (ei, en) in zip(got, expected):
            assert torch.equal(gi, ei) and torch.equal(gn, en)
        assert dl.get_status() == 0


@pytest.mark.parametrize("name,block_only", [("cfg0", False), ("cfg4_block", True), ("cfg1", False)])
def test_cuda_graph_replay_matches_eager(dl, name, block_only):
    """A captured step replayed on new contents of its input buffers gives the eager step's
    results bit for bit (same kernels, same launch shapes)."""
    cfg = WL.CONFIGS[name]
    inps = [WL.make_inputs(cfg, seed=s) for s in (0, 1)]
    W = inps[0]["W"].cuda()
    H = inps[0]["H"].cuda()
    M = inps[0]["M"].cuda()
    lo = None if inps[0]["win_lo"] is None else torch.from_numpy(inps[0]["win_lo"]).cuda()
    hi = None if inps[0]["win_hi"] is None else torch.from_numpy(inps[0]["win_hi"]).cuda()
    eager = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
    graphed = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
    graphed.capture(H, M, W, lo, hi, block_only=block_only)
    for inp in inps:
        H.copy_(inp["H"])
        M.copy_(inp["M"])
        e = {k: v.clone() for k, v in eager.run(H, M, W, lo, hi, block_only=block_only).items()}
        g = graphed.replay()
        torch.cuda.synchronize()
        assert dl.get_status() == 0
        c = int(e["count"][0])
        assert int(g["count"][0]) == c
        for key in ("tok", "conf", "lse", "row_idx"):
            assert torch.equal(e[key][:c], g[key][:c]), key
        for key in ("idx", "n_sel", "tok_sel", "conf_sel"):
            assert torch.equal(e[key], g[key]), key


def test_step_memory_is_far_below_full_logits(dl):
    """The step allocates no [B*L, V] buffer and the library allocates no device memory:
    after warm-up, running steps changes neither torch's allocations nor the device's free
    memory, and everything the step owns (outputs + workspace) is a small fraction of the
    bf16 full-logits tensor it avoids."""
    for name in ("cfg1", "cfg4"):
        inp = WL.make_inputs(WL.CONFIGS[name], seed=0)
        cfg = inp["cfg"]
        dev = GU.to_device(inp)
        step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
        for _ in range(2):
            step.run(dev["H"], dev["M"], dev["W"], dev["win_lo"], dev["win_hi"])
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()
        before_alloc = torch.cuda.memory_allocated()
        free_before, _ = torch.cuda.mem_get_info()
        for _ in range(3):
            step.run(dev["H"], dev["M"], dev["W"], dev["win_lo"], dev["win_hi"])
        torch.cuda.synchronize()
        free_after, _ = torch.cuda.mem_get_info()
        assert dl.get_status() == 0
        assert torch.cuda.max_memory_allocated() == before_alloc, name   # nothing allocated
        assert free_after >= free_before, name                          # not even by the library
        owned = step.ws.numel() + sum(t.numel() * t.element_size() for t in
                                      (step.tok, step.conf, step.lse, step.row_idx, step.seq_off,
                                       step.count, step.sel_buf))
        full_logits_bf16 = cfg.B * cfg.L * cfg.V * 2
        assert owned < full_logits_bf16 / 10, (name, owned, full_logits_bf16)
        del step, dev
        torch.cuda.empty_cache()


def test_overlapped_steps_match_single_steps(dl):
    """Steps overlapped on two streams (staging of step i+1 during step i) select exactly
    what single steps select, batch by batch, and leave the last step's outputs."""
    for name in ("cfg0", "cfg1", "cfg4"):            # cfg1: the launch mode bench.py times
        cfg = WL.CONFIGS[name]
        inp0 = WL.make_inputs(cfg, seed=21)
        host = [(inp0["H"], inp0["M"])]
        for sd in (22, 23, 24, 25):              # more batches: new H and mask, same W
            g = torch.Generator().manual_seed(sd)
            H = (torch.randn(cfg.B * cfg.L, cfg.d, generator=g) * cfg.h_std).to(torch.bfloat16)
            host.append((H, WL.make_mask(cfg, g)))
        W = inp0["W"].cuda()
        lo = None if inp0["win_lo"] is None else torch.from_numpy(inp0["win_lo"]).cuda()
        hi = None if inp0["win_hi"] is None else torch.from_numpy(inp0["win_hi"]).cuda()
        step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
        dev = [(H.cuda(), M.cuda()) for H, M in host]
        expected = []
        for H, M in dev:
            step.run(H, M, W, lo, hi)
            expected.append(step.sel_buf.clone())
        sel_out = [torch.empty_like(step.sel_buf) for _ in dev]
        out = step.run_overlapped(dev, W, lo, hi, sel_out=sel_out)
        torch.cuda.synchronize()
        assert dl.get_status() == 0
        for got, exp in zip(sel_out, expected):
            assert torch.equal(got, exp), name
        assert torch.equal(step.sel_buf, expected[-1])
        c = int(out["count"][0])
        ref_rows, _, ref_c = O.mask_compact(host[-1][1].numpy())
        assert c == ref_c and np.array_equal(out["row_idx"][:c].cpu().numpy(), ref_rows)


def test_overlapped_steps_from_a_generator(dl):
    """Batches yielded by a generator that writes each one (on the current stream) just
    before yielding it: the staging of every step waits for that write, so the selections
    equal single steps on the same inputs.  Run with a producer stream as the current
    stream, and with the compute stream itself as the current stream."""
    cfg = WL.CONFIGS["cfg1"]
    inp0 = WL.make_inputs(cfg, seed=31)
    host = []
    for sd in (32, 33, 34, 35):
        g = torch.Generator().manual_seed(sd)
        H = (torch.randn(cfg.B * cfg.L, cfg.d, generator=g) * cfg.h_std).to(torch.bfloat16)
        M = WL.make_mask(cfg, g) if sd % 2 else torch.roll(WL.make_mask(cfg, g), 7 * sd, 1)
        host.append((H.pin_memory(), M.pin_memory()))
    W = inp0["W"].cuda()
    step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k)
    expected = []
    for H, M in host:
        step.run(H.cuda(), M.cuda(), W)
        expected.append(step.sel_buf.clone())
    torch.cuda.synchronize()
    compute = torch.cuda.Stream()
    for producer in (torch.cuda.Stream(), compute):
        # two pairs of buffers, each overwritten every other batch: a staging that read too
        # early would see an older batch (or a half-written one)
        bufs = [(torch.zeros(cfg.B * cfg.L, cfg.d, dtype=torch.bfloat16, device="cuda"),
                 torch.zeros(cfg.B, cfg.L, dtype=torch.uint8, device="cuda")) for _ in range(2)]
        used = [None, None]

        def batches():
            for i, (H, M) in enumerate(host):
                Hd, Md = bufs[i & 1]
                if used[i & 1] is not None:
                    torch.cuda.current_stream().wait_event(used[i & 1])
                Hd.copy_(H, non_blocking=True)
                Md.copy_(M, non_blocking=True)
                ev = torch.cuda.Event()
                used[i & 1] = ev
                yield Hd, Md
                ev.record(compute)               # the step reading this pair is enqueued

        sel_out = [torch.empty_like(step.sel_buf) for _ in host]
        with torch.cuda.stream(producer):
            step.run_overlapped(batches(), W, stream=compute, sel_out=sel_out)
        torch.cuda.synchronize()
        assert dl.get_status() == 0
        for got, exp in zip(sel_out, expected):
            assert torch.equal(got, exp)
