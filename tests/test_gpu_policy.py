"""Unmask-policy variants on the GPU against the oracle: softmax entropy and top-2
probability margin per masked row (dllm_masked_logits_ex), and threshold-based parallel
unmasking (dllm_select_unmask_ex), descending and ascending.

Tolerances (fp32 accumulation of bf16 products, like lse and conf): entropy within 2e-3
relative plus 2e-5 absolute; margin within 2e-3 relative plus 1e-4 x conf absolute (the
margin is (1 - exp(m2 - m)) / s, so an error d in the top-2 logit gap moves it by about
d x conf).  Selections are bit-exact against the oracle run on the GPU's own scores.
"""
import numpy as np
import pytest
import torch

import oracle.oracle as O
import workloads as WL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import mask_only_logits_b200 as dl
    return dl


@pytest.fixture(params=[0, 1, 2], ids=["default", "single", "pair"])
def variant(request, dl):
    dl.debug_set_gemm_variant(request.param)
    yield request.param
    dl.debug_set_gemm_variant(0)


def _run_ex(dl, inp, stats, win=None):
    cfg = inp["cfg"]
    n = cfg.B * cfg.L
    dev = dict(H=inp["H"].cuda(), M=inp["M"].cuda(), W=inp["W"].cuda())
    f32 = dict(dtype=torch.float32, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    tok, conf, lse = torch.empty(n, **i32), torch.empty(n, **f32), torch.empty(n, **f32)
    ent = torch.empty(n, **f32) if stats & dl.STAT_ENTROPY else None
    mar = torch.empty(n, **f32) if stats & dl.STAT_MARGIN else None
    row_idx, seq_off, count = torch.empty(n, **i32), torch.empty(cfg.B + 1, **i32), torch.empty(4, **i32)
    ws = torch.empty(dl.workspace_bytes(cfg.B, cfg.L, cfg.d, cfg.V), dtype=torch.uint8, device="cuda")
    lo = hi = None
    if win is not None:
        lo = torch.from_numpy(np.asarray(win[0], dtype=np.int32)).cuda()
        hi = torch.from_numpy(np.asarray(win[1], dtype=np.int32)).cuda()
    dl.masked_logits_ex(dev["H"], dev["M"], dev["W"], stats, tok, conf, lse, ent, mar, row_idx,
                        seq_off, count, ws, win_lo=lo, win_hi=hi)
    assert dl.get_status() == 0
    c = int(count[0])
    out = dict(count=c, tok=tok[:c].cpu().numpy(), conf=conf[:c].cpu().numpy(),
               lse=lse[:c].cpu().numpy(), row_idx=row_idx[:c].cpu().numpy(),
               seq_off=seq_off.cpu().numpy())
    if ent is not None:
        out["entropy"] = ent[:c].cpu().numpy()
    if mar is not None:
        out["margin"] = mar[:c].cpu().numpy()
    return out


def _check_policy(g, ref, rows):
    e_g = g["entropy"][rows].astype(np.float64)
    m_g = g["margin"][rows].astype(np.float64)
    assert np.all(np.isfinite(e_g)) and np.all(np.isfinite(m_g))
    assert np.all(np.abs(e_g - ref["entropy"]) <= 2e-3 * np.abs(ref["entropy"]) + 2e-5), \
        float(np.max(np.abs(e_g - ref["entropy"])))
    assert np.all(np.abs(m_g - ref["margin"]) <= 2e-3 * np.abs(ref["margin"]) + 1e-4 * ref["conf"]), \
        float(np.max(np.abs(m_g - ref["margin"]) / ref["conf"]))
    # the plain statistics are unchanged by the extended epilogue
    np.testing.assert_allclose(g["lse"][rows], ref["lse"], rtol=2e-3)
    np.testing.assert_allclose(g["conf"][rows], ref["conf"], rtol=2e-3)


@pytest.mark.parametrize("B,L,d,V,r", [(1, 256, 256, 4096, 0.5),      # cfg0 shapes
                                       (2, 300, 64, 1000, 0.8),       # V tail, ragged rows
                                       (1, 6000, 128, 700, 0.9),      # several groups: merged
                                       (1, 1000, 64, 37800, 1.0),     # remainder holders
                                       (1, 50, 64, 1, 1.0)])          # V = 1: entropy 0
def test_entropy_margin(dl, variant, B, L, d, V, r):
    inp = WL.make_inputs(WL.custom_config(B, L, d, V, 4, r=r), seed=3)
    g = _run_ex(dl, inp, dl.STAT_ENTROPY | dl.STAT_MARGIN)
    Hb, Wb, M = WL.bf16_bits(inp["H"]), WL.bf16_bits(inp["W"]), inp["M"].numpy()
    rows = np.arange(g["count"])
    ref = O.oracle_rows(Hb, Wb, M, rows)
    _check_policy(g, ref, rows)
    ok_tok = (g["tok"] == ref["tok"]) | (ref["gap"] < 1e-3)
    assert ok_tok.all()


def test_entropy_margin_cfg1_every_row(dl):
    inp = WL.make_inputs(WL.CONFIGS["cfg1"], seed=0)
    g = _run_ex(dl, inp, dl.STAT_ENTROPY | dl.STAT_MARGIN)
    Hb, Wb, M = WL.bf16_bits(inp["H"]), WL.bf16_bits(inp["W"]), inp["M"].numpy()
    rows = np.arange(g["count"])
    _check_policy(g, O.oracle_rows(Hb, Wb, M, rows), rows)


def test_entropy_margin_current_block_only(dl, variant):
    """dllm_masked_logits_window: statistics for the masked rows inside the windows only."""
    inp = WL.make_inputs(WL.custom_config(4, 3000, 128, 5000, 4, r=0.8), seed=6)
    lo = np.array([0, 100, 2990, 1500])
    hi = np.array([32, 164, 3100, 1200])                       # the last window is empty
    g = _run_ex(dl, inp, dl.STAT_ENTROPY | dl.STAT_MARGIN, (lo, hi))
    Mw = O.window_mask(inp["M"].numpy(), lo, hi)
    ref = O.oracle_rows(WL.bf16_bits(inp["H"]), WL.bf16_bits(inp["W"]), Mw)
    assert g["count"] == ref["count"]
    np.testing.assert_array_equal(g["row_idx"], ref["row_idx"])
    np.testing.assert_array_equal(g["seq_off"], ref["seq_off"])
    _check_policy(g, ref, np.arange(g["count"]))


def test_margin_exact_ties_and_single_flags(dl):
    # duplicated vocabulary rows -> the top logit is attained twice: margin exactly 0
    rng = np.random.default_rng(4)
    W = torch.from_numpy((rng.standard_normal((300, 64)) * 0.3).astype(np.float32)).to(torch.bfloat16)
    W[200] = W[7]
    inp = WL.make_inputs(WL.custom_config(1, 128, 64, 300, 4, r=1.0), seed=1)
    inp["W"] = W
    g = _run_ex(dl, inp, dl.STAT_MARGIN)
    ref = O.oracle_rows(WL.bf16_bits(inp["H"]), WL.bf16_bits(W), inp["M"].numpy())
    tie_rows = np.flatnonzero(ref["margin"] == 0.0)
    assert np.all(g["margin"][tie_rows] == 0.0)
    assert "entropy" not in g
    g2 = _run_ex(dl, inp, dl.STAT_ENTROPY)
    assert "margin" not in g2 and np.all(np.isfinite(g2["entropy"]))


def _select_ex(dl, score_np, M_np, k, tau, min_sel, ascending, win=None):
    B, L = M_np.shape
    row_idx, seq_off, count = O.mask_compact(M_np)
    score = torch.from_numpy(score_np.astype(np.float32)).cuda()
    idx = torch.full((B, k), -9, dtype=torch.int32, device="cuda")
    n_sel = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    sc_sel = torch.empty((B, k), dtype=torch.float32, device="cuda")
    lo = hi = None
    if win is not None:
        lo = torch.from_numpy(win[0].astype(np.int32)).cuda()
        hi = torch.from_numpy(win[1].astype(np.int32)).cuda()
    dl.select_unmask_ex(score, torch.from_numpy(row_idx).cuda(), torch.from_numpy(seq_off).cuda(),
                        B, L, k, tau, min_sel, idx, n_sel, ascending, lo, hi, score_sel=sc_sel)
    s32 = score_np.astype(np.float32).astype(np.float64)
    # ascending order == descending order of the negated scores (negation is exact)
    ref_idx, ref_n = O.select_unmask_threshold(-s32 if ascending else s32, row_idx, seq_off, L,
                                               k, -tau if ascending else tau, min_sel,
                                               None if win is None else win[0],
                                               None if win is None else win[1])
    np.testing.assert_array_equal(n_sel.cpu().numpy(), ref_n)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    return idx.cpu().numpy(), n_sel.cpu().numpy()


@pytest.mark.parametrize("ascending", [False, True])
@pytest.mark.parametrize("tau,min_sel,k", [(0.5, 1, 64), (0.9, 1, 16), (0.99, 0, 16),
                                           (0.99, 3, 16), (-1.0, 1, 32), (0.25, 1, 1024)])
def test_threshold_select_bit_exact(dl, ascending, tau, min_sel, k):
    rng = np.random.default_rng(abs(int(tau * 100)) + k)
    B, L = 3, 5000
    M = (rng.random((B, L)) < 0.6).astype(np.uint8)
    n = int(M.sum())
    score = (rng.integers(0, 64, size=n) / 64.0).astype(np.float32)     # many exact ties
    if ascending:
        score = -score + 0.5                                               # negative values too
    _select_ex(dl, score, M, k, tau, min_sel, ascending)


def test_threshold_select_plain_topk_and_windows(dl):
    rng = np.random.default_rng(9)
    M = WL.make_mask(WL.CONFIGS["cfg4"]).numpy()
    n = int(M.sum())
    score = rng.standard_normal(n).astype(np.float32)
    lo, hi = WL.make_windows(WL.CONFIGS["cfg4"])
    idx, n_sel = _select_ex(dl, score, M, 4, float("-inf"), 1, False, (lo, hi))
    row_idx, seq_off, _ = O.mask_compact(M)
    t_idx, t_n = O.select_unmask(score, row_idx, seq_off, M.shape[1], 4, lo, hi)
    assert np.array_equal(idx, t_idx) and np.array_equal(n_sel, t_n)
    _select_ex(dl, score, M, 8, 0.0, 2, False, (lo, hi))
    _select_ex(dl, score, M, 8, 0.0, 2, True, (lo, hi))
    _select_ex(dl, score, M, 32, float("inf"), 1, True)


def test_entropy_driven_step(dl):
    """Entropy-driven unmasking end to end: entropies from the GEMM epilogue, then the k
    lowest-entropy positions (ascending) with a threshold, against the oracle's selection
    on the same (GPU) entropies."""
    inp = WL.make_inputs(WL.CONFIGS["cfg0"], seed=2)
    g = _run_ex(dl, inp, dl.STAT_ENTROPY)
    M = inp["M"].numpy()
    ent = g["entropy"]
    tau = float(np.quantile(ent, 0.1))
    ent_dev = torch.from_numpy(ent).cuda()
    B, L = M.shape
    idx = torch.empty((B, 8), dtype=torch.int32, device="cuda")
    n_sel = torch.empty((B,), dtype=torch.int32, device="cuda")
    dl.select_unmask_ex(ent_dev, torch.from_numpy(g["row_idx"]).cuda(),
                        torch.from_numpy(g["seq_off"]).cuda(), B, L, 8, tau, 1, idx, n_sel,
                        ascending=True)
    e64 = ent.astype(np.float64)
    ref_idx, ref_n = O.select_unmask_threshold(-e64, g["row_idx"], g["seq_off"], L, 8, -tau, 1)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(n_sel.cpu().numpy(), ref_n)


# thresholds exactly representable in float32, so that the fp32 comparison on the GPU and
# the fp64 one of the oracle agree for every score
@pytest.mark.parametrize("policy,threshold,min_sel", [("entropy", None, 1), ("margin", None, 1),
                                                     ("confidence", 0.015625, 2),
                                                     ("entropy", 9.0, 0), ("margin", 2.0 ** -10, 1)])
def test_decode_step_policies(dl, policy, threshold, min_sel):
    """DecodeStep with an unmasking policy: the selection equals the oracle's threshold
    selection on the step's own GPU scores (bit-exact), and the per-row scores match the
    oracle's within the policy tolerances."""
    inp = WL.make_inputs(WL.CONFIGS["cfg4"] if policy == "margin" else WL.CONFIGS["cfg0"], seed=7)
    cfg = inp["cfg"]
    step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k, policy=policy, threshold=threshold,
                         min_sel=min_sel)
    lo = None if inp["win_lo"] is None else torch.from_numpy(inp["win_lo"]).cuda()
    hi = None if inp["win_hi"] is None else torch.from_numpy(inp["win_hi"]).cuda()
    out = step.run(inp["H"].cuda(), inp["M"].cuda(), inp["W"].cuda(), lo, hi)
    assert dl.get_status() == 0
    c = int(out["count"][0])
    score = out["conf"] if policy == "confidence" else out[policy]
    s32 = score[:c].cpu().numpy().astype(np.float64)
    row_idx, seq_off = out["row_idx"][:c].cpu().numpy(), out["seq_off"].cpu().numpy()
    asc = policy == "entropy"
    tau = threshold if threshold is not None else (np.inf if asc else -np.inf)
    ref_idx, ref_n = O.select_unmask_threshold(-s32 if asc else s32, row_idx, seq_off, cfg.L, cfg.k,
                                               -tau if asc else tau, min_sel, inp["win_lo"],
                                               inp["win_hi"])
    np.testing.assert_array_equal(out["n_sel"].cpu().numpy(), ref_n)
    np.testing.assert_array_equal(out["idx"].cpu().numpy(), ref_idx)
    # the selected scores are those of the selected rows
    for b in range(cfg.B):
        n = int(ref_n[b])
        r = [np.searchsorted(row_idx, b * cfg.L + p) for p in ref_idx[b, :n]]
        np.testing.assert_array_equal(out["conf_sel"][b, :n].cpu().numpy(), s32[r].astype(np.float32))
    # scores against the oracle on a sample of rows
    rows = np.arange(c) if c <= 600 else WL.sample_rows(c, 300, seed=1)
    ref = O.oracle_rows(WL.bf16_bits(inp["H"]), WL.bf16_bits(inp["W"]), inp["M"].numpy(), rows)
    if policy == "entropy":
        e = s32[rows]
        assert np.all(np.abs(e - ref["entropy"]) <= 2e-3 * np.abs(ref["entropy"]) + 2e-5)
    elif policy == "margin":
        m = s32[rows]
        assert np.all(np.abs(m - ref["margin"]) <= 2e-3 * np.abs(ref["margin"]) + 1e-4 * ref["conf"])


def test_policy_pipeline_matches_device_steps(dl):
    """The host pipeline with an entropy policy selects what device-resident steps select."""
    cfg = WL.CONFIGS["cfg0"]
    inps = [WL.make_inputs(cfg, seed=s) for s in (11, 12, 13)]
    W = inps[0]["W"].cuda()
    step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k, policy="entropy", threshold=7.0)
    expected = []
    for inp in inps:
        out = step.run(inp["H"].cuda(), inp["M"].cuda(), W)
        expected.append((out["idx"].cpu().clone(), out["n_sel"].cpu().clone()))
    batches = [(inp["H"].pin_memory(), inp["M"].pin_memory()) for inp in inps]
    got = [(o["idx"].clone(), o["n_sel"].clone()) for o in step.run_host_pipeline(batches, W)]
    for (gi, gn), (ei, en) in zip(got, expected):
        assert torch.equal(gi, ei) and torch.equal(gn, en)


@pytest.mark.parametrize("policy,threshold", [("entropy", 7.0), ("margin", None),
                                              ("confidence", 0.015625)])
def test_policy_overlapped_steps_block_only(dl, policy, threshold):
    """Overlapped steps (staging on a second stream) with a policy and current-block-only
    logits select what single device-resident steps select, batch by batch."""
    cfg = WL.CONFIGS["cfg4_block"]
    inps = [WL.make_inputs(cfg, seed=s) for s in (31, 32, 33)]
    W = inps[0]["W"].cuda()
    lo = torch.from_numpy(inps[0]["win_lo"]).cuda()
    hi = torch.from_numpy(inps[0]["win_hi"]).cuda()
    step = dl.DecodeStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k, policy=policy, threshold=threshold)
    dev = [(inp["H"].cuda(), inp["M"].cuda()) for inp in inps]
    expected = []
    for H, M in dev:
        step.run(H, M, W, lo, hi, block_only=True)
        expected.append(step.sel_buf.clone())
    sel_out = [torch.empty_like(step.sel_buf) for _ in dev]
    step.run_overlapped(dev, W, lo, hi, block_only=True, sel_out=sel_out)
    torch.cuda.synchronize()
    assert dl.get_status() == 0
    for got, exp in zip(sel_out, expected):
        assert torch.equal(got, exp)
    # the block-only row set of the last batch: the masked positions inside the windows
    c = int(step.count[0])
    Mw = O.window_mask(inps[-1]["M"].numpy(), inps[0]["win_lo"], inps[0]["win_hi"])
    assert c == int(Mw.sum())
    assert np.array_equal(step.row_idx[:c].cpu().numpy(), np.flatnonzero(Mw.reshape(-1)))


@pytest.mark.parametrize("ascending", [False, True])
def test_threshold_select_rank_path_boundary(dl, ascending):
    """Threshold selection on 255 / 256 / 257 candidates (the rank placement and the radix
    select meet at 256), exact ties, min_sel floors above and below the passing count."""
    rng = np.random.default_rng(5)
    B, L = 3, 300
    M = np.zeros((B, L), np.uint8)
    for b, n_b in enumerate((255, 256, 257)):
        M[b, rng.choice(L, n_b, replace=False)] = 1
    n = int(M.sum())
    score = (rng.integers(0, 32, size=n) / 32.0).astype(np.float32)
    if ascending:
        score = -score + 0.25
    for tau, min_sel, k in ((0.5, 1, 256), (0.97, 20, 64), (0.0, 0, 300), (2.0, 5, 8)):
        _select_ex(dl, score, M, k, tau, min_sel, ascending)
