"""Kernel-level parity on the GPU, through the C ABI: compaction (bit-exact), the
tensor-core GEMM's raw logits, lse_merge, and select_unmask (bit-exact)."""
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


# ------------------------------------------------------------------------------- compaction
def _compact_case(dl, M_np):
    B, L = M_np.shape
    M = torch.from_numpy(M_np).cuda()
    n = B * L
    row_idx = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    seq_off = torch.full((B + 1,), -7, dtype=torch.int32, device="cuda")
    count = torch.full((4,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(dl.workspace_bytes(B, L, 64, 1), dtype=torch.uint8, device="cuda")
    dl.mask_compact(M, row_idx, seq_off, count, ws)
    assert dl.get_status() == 0
    r_ref, s_ref, c_ref = O.mask_compact(M_np)
    c = int(count[0])
    assert c == c_ref
    np.testing.assert_array_equal(row_idx[:c].cpu().numpy(), r_ref)
    np.testing.assert_array_equal(seq_off.cpu().numpy(), s_ref)
    # entries past count are untouched
    assert bool((row_idx[c:] == -7).all())


@pytest.mark.parametrize("B,L,p", [(1, 256, 0.5), (1, 4096, 0.25), (1, 131072, 0.9), (1, 131072, 0.1),
                                   (8, 8192, 0.5), (3, 1000, 0.5), (5, 1, 0.5), (7, 3, 0.6),
                                   (2, 8191, 0.3), (1, 8193, 0.99), (4, 17, 0.0), (4, 17, 1.0),
                                   (1, 16, 1.0), (1, 15, 1.0), (37, 1111, 0.5),
                                   # 16 tiles (one launch) / 17 and 19 tiles (count + scatter)
                                   (16, 8192, 0.5), (1, 131073, 0.5), (3, 50000, 0.4),
                                   # 64 tiles (offsets summed per CTA) / 65, 129 and 184 tiles
                                   # (offsets from the scan launch)
                                   (64, 8192, 0.5), (65, 8192, 0.5), (1, 1048577, 0.5),
                                   (3, 500000, 0.6)])
def test_compact_bit_exact(dl, B, L, p):
    rng = np.random.default_rng(B * 1000 + L)
    M = (rng.random((B, L)) < p).astype(np.uint8)
    _compact_case(dl, M)


def test_compact_nonbinary_and_workload_masks(dl):
    rng = np.random.default_rng(1)
    M = rng.integers(0, 4, size=(2, 999)).astype(np.uint8) * 85    # 0, 85, 170, 255
    _compact_case(dl, M)
    for name in ("cfg0", "cfg1", "cfg4"):
        cfg = WL.CONFIGS[name]
        g = torch.Generator().manual_seed(0)
        _compact_case(dl, WL.make_mask(cfg, g).numpy())


def _compact_window_case(dl, M_np, lo, hi):
    B, L = M_np.shape
    n = B * L
    row_idx = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    seq_off = torch.full((B + 1,), -7, dtype=torch.int32, device="cuda")
    count = torch.full((4,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(dl.workspace_bytes(B, L, 64, 1), dtype=torch.uint8, device="cuda")
    dl.mask_compact(torch.from_numpy(M_np).cuda(), row_idx, seq_off, count, ws,
                    win_lo=torch.from_numpy(lo.astype(np.int32)).cuda(),
                    win_hi=torch.from_numpy(hi.astype(np.int32)).cuda())
    assert dl.get_status() == 0
    r_ref, s_ref, c_ref = O.mask_compact(O.window_mask(M_np, lo, hi))
    c = int(count[0])
    assert c == c_ref
    np.testing.assert_array_equal(row_idx[:c].cpu().numpy(), r_ref)
    np.testing.assert_array_equal(seq_off.cpu().numpy(), s_ref)
    assert bool((row_idx[c:] == -7).all())


@pytest.mark.parametrize("B,L,p", [(1, 256, 0.5), (8, 8192, 1.0), (3, 1000, 0.5), (7, 3, 0.6),
                                   (5, 1, 1.0), (2, 8191, 0.3), (37, 1111, 0.5), (1, 131072, 0.9),
                                   (64, 17, 0.8), (16, 8192, 0.7), (20, 8192, 0.7), (1, 131073, 0.5),
                                   (80, 8192, 0.7), (2, 300001, 0.5)])
def test_compact_windows_bit_exact(dl, B, L, p):
    """Current-block-only compaction: windows of random placement and width, including
    empty, inverted, negative and past-the-end ones, and sequences shorter than a vector."""
    rng = np.random.default_rng(B * 31 + L)
    M = (rng.random((B, L)) < p).astype(np.uint8)
    lo = rng.integers(-5, L + 3, size=B)
    hi = lo + rng.integers(-3, max(2, L // 3), size=B)
    _compact_window_case(dl, M, lo, hi)
    # every window the whole sequence / no window at all / one position
    _compact_window_case(dl, M, np.zeros(B, np.int64), np.full(B, L))
    _compact_window_case(dl, M, np.full(B, L), np.full(B, L + 5))
    _compact_window_case(dl, M, np.full(B, L - 1), np.full(B, L))


def test_compact_windows_semi_ar(dl):
    cfg = WL.CONFIGS["cfg4"]
    M = WL.make_mask(cfg).numpy()
    lo, hi = WL.make_windows(cfg)
    _compact_window_case(dl, M, lo, hi)


# ------------------------------------------------------------------- tensor-core GEMM logits
def _rand_bf16(rng, shape, std):
    return torch.from_numpy((rng.standard_normal(shape) * std).astype(np.float32)).to(torch.bfloat16)


@pytest.fixture(params=[2, 1], ids=["pair", "single"])
def variant(request, dl):
    """Run a test with the paired-SM GEMM (default) and with the single-SM GEMM."""
    dl.debug_set_gemm_variant(request.param)
    yield request.param
    dl.debug_set_gemm_variant(0)


@pytest.mark.parametrize("B,L,d,V,p", [(1, 256, 256, 4096, 0.5),      # cfg0 shapes
                                       (2, 200, 128, 1000, 0.7),       # ragged rows, V tail
                                       (1, 300, 64, 300, 1.0),         # one K block, V tail
                                       (1, 1024, 1024, 2048, 0.6),     # many K blocks
                                       (3, 97, 192, 777, 0.9),         # odd everything
                                       (1, 5, 64, 1, 1.0),             # V = 1
                                       (1, 6000, 128, 700, 0.9),       # several m-tile groups
                                       (1, 2048, 64, 3000, 1.0),       # 8 m-tiles of 256
                                       (1, 2300, 64, 2000, 1.0),       # 9 of 256 / 18 of 128: streams
                                       (1, 1000, 64, 20000, 1.0),      # 8 m-tiles of 128
                                       (1, 1000, 64, 37800, 1.0),      # remainder holders
                                       # one m-tile whose vocabulary tiles do not divide
                                       # evenly among the 74 pairs / 148 CTAs
                                       (1, 100, 128, 40000, 1.0),      # 157 tiles, 2 K blocks
                                       (1, 128, 192, 75000, 0.9),      # 3 K blocks, V tail
                                       (2, 128, 1024, 40000, 1.0),     # 16 K blocks, 256 rows
                                       (1, 256, 128, 19044, 0.95)])    # 75 tiles over 74 pairs
def test_lmhead_raw_logits(dl, variant, B, L, d, V, p):
    rng = np.random.default_rng(d + V)
    H = _rand_bf16(rng, (B * L, d), 1.0)
    W = _rand_bf16(rng, (V, d), 0.02)
    M = (rng.random((B, L)) < p).astype(np.uint8)
    n = B * L
    out = torch.full((n, V), float("nan"), dtype=torch.float32, device="cuda")
    row_idx = torch.empty(n, dtype=torch.int32, device="cuda")
    seq_off = torch.empty(B + 1, dtype=torch.int32, device="cuda")
    count = torch.empty(4, dtype=torch.int32, device="cuda")
    ws = torch.empty(dl.workspace_bytes(B, L, d, V), dtype=torch.uint8, device="cuda")
    dl.debug_lmhead_logits(H.cuda(), torch.from_numpy(M).cuda(), W.cuda(), out, row_idx, seq_off,
                           count, ws)
    assert dl.get_status() == 0
    c = int(count[0])
    r_ref, _, c_ref = O.mask_compact(M)
    assert c == c_ref
    H64 = O.bf16_bits_to_f64(WL.bf16_bits(H))[r_ref]
    W64 = O.bf16_bits_to_f64(WL.bf16_bits(W))
    Z = O.logits_rows(H64, W64)
    scale = np.abs(H64) @ np.abs(W64).T               # sum |h||w|: fp32 accumulation bound
    got = out[:c].cpu().numpy().astype(np.float64)
    err = np.abs(got - Z)
    assert np.all(np.isfinite(got))
    assert np.all(err <= 1e-5 * scale + 1e-7), float((err / (scale + 1e-30)).max())


# ----------------------------------------------------------------------------- lse_merge
@pytest.mark.parametrize("n_rows,n_split", [(1, 1), (300, 7), (1000, 64), (4097, 3)])
def test_lse_merge_hook(dl, n_rows, n_split):
    rng = np.random.default_rng(n_rows)
    V = 40 * n_split
    Z = rng.standard_normal((n_rows, V)) * 4
    Z[0, 5] = Z[0, V - 3] = Z[0].max() + 2.0          # a tie across splits: lowest wins
    bounds = np.linspace(0, V, n_split + 1).astype(int)
    parts = [O.partial_stats(Z, a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    pm = torch.tensor(np.stack([p[0] for p in parts]), dtype=torch.float32, device="cuda")
    ps = torch.tensor(np.stack([p[1] for p in parts]), dtype=torch.float32, device="cuda")
    pa = torch.tensor(np.stack([p[2] for p in parts]), dtype=torch.int32, device="cuda")
    tok = torch.empty(n_rows, dtype=torch.int32, device="cuda")
    conf = torch.empty(n_rows, dtype=torch.float32, device="cuda")
    lse = torch.empty(n_rows, dtype=torch.float32, device="cuda")
    dl.debug_lse_merge(pm.contiguous(), ps.contiguous(), pa.contiguous(), tok, conf, lse)
    # reference: the oracle's merge of the same fp32-rounded partials
    p32 = [(m.astype(np.float32).astype(np.float64), s.astype(np.float32).astype(np.float64), a)
           for m, s, a in parts]
    t_ref, m_ref, lse_ref, conf_ref = O.lse_merge(p32)
    assert tok.cpu().numpy().tolist() == t_ref.tolist()
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(conf.cpu().numpy(), conf_ref, rtol=1e-5)
    assert tok[0].item() == 5


# ------------------------------------------------------------------------- select_unmask
def _select_case(dl, conf_np, M_np, k, win=None, tok_np=None):
    B, L = M_np.shape
    row_idx, seq_off, count = O.mask_compact(M_np)
    assert conf_np.size == count
    conf = torch.from_numpy(conf_np.astype(np.float32)).cuda()
    ri = torch.from_numpy(row_idx).cuda()
    so = torch.from_numpy(seq_off).cuda()
    idx = torch.full((B, k), -9, dtype=torch.int32, device="cuda")
    n_sel = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    tok = torch.from_numpy(tok_np).cuda() if tok_np is not None else None
    tok_sel = torch.empty((B, k), dtype=torch.int32, device="cuda") if tok is not None else None
    conf_sel = torch.empty((B, k), dtype=torch.float32, device="cuda")
    lo = hi = None
    if win is not None:
        lo = torch.from_numpy(win[0].astype(np.int32)).cuda()
        hi = torch.from_numpy(win[1].astype(np.int32)).cuda()
    if conf.numel() == 0:        # keep a valid, aligned pointer for empty inputs
        conf = torch.empty(4, dtype=torch.float32, device="cuda")
        ri = torch.empty(4, dtype=torch.int32, device="cuda")
    dl.select_unmask(conf, ri, so, B, L, k, idx, n_sel, lo, hi, tok, tok_sel, conf_sel)
    ref_idx, ref_n = O.select_unmask(conf_np.astype(np.float32), row_idx, seq_off, L, k,
                                     None if win is None else win[0],
                                     None if win is None else win[1])
    np.testing.assert_array_equal(n_sel.cpu().numpy(), ref_n)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    # tok_sel / conf_sel follow the selection
    cs = conf_sel.cpu().numpy()
    for b in range(B):
        for j in range(k):
            p = ref_idx[b, j]
            if p < 0:
                assert cs[b, j] == 0.0
                continue
            r = np.searchsorted(row_idx, b * L + p)
            assert cs[b, j] == np.float32(conf_np[r])
            if tok is not None:
                assert int(tok_sel[b, j]) == int(tok_np[r])


@pytest.mark.parametrize("B,L,k,p,ties", [(1, 256, 8, 0.5, False), (1, 4096, 32, 0.25, True),
                                          (1, 131072, 128, 0.9, False), (1, 131072, 128, 0.9, True),
                                          (8, 8192, 4, 0.5, True), (3, 100, 200, 0.5, False),
                                          (2, 64, 1, 1.0, True), (4, 3000, 1024, 0.7, False),
                                          (4, 3000, 1000, 0.7, True)])
def test_select_bit_exact(dl, B, L, k, p, ties):
    rng = np.random.default_rng(L + k)
    M = (rng.random((B, L)) < p).astype(np.uint8)
    n = int(M.astype(bool).sum())
    if ties:   # few distinct values: many exact ties, decided by position
        conf = (rng.integers(1, 9, size=n) / 8.0).astype(np.float32)
    else:
        conf = rng.random(n).astype(np.float32) * 0.999 + 0.001
    tok = rng.integers(0, 1000, size=n).astype(np.int32)
    _select_case(dl, conf, M, k, tok_np=tok)


def test_select_windows_and_empty(dl):
    rng = np.random.default_rng(3)
    B, L = 8, 8192
    M = WL.make_mask(WL.CONFIGS["cfg4"]).numpy()
    n = int(M.sum())
    conf = (rng.integers(1, 5, size=n) / 4.0).astype(np.float32)
    lo, hi = WL.make_windows(WL.CONFIGS["cfg4"])
    _select_case(dl, conf, M, 4, (lo, hi))
    _select_case(dl, conf, M, 40, (lo, hi))                       # k > window size
    _select_case(dl, conf, M, 4, (lo - 4000, lo - 3000))          # windows outside the mask
    # empty sequences and an all-unmasked batch
    M2 = np.zeros((3, 50), np.uint8)
    M2[1, 10:20] = 1
    _select_case(dl, rng.random(10).astype(np.float32), M2, 5)
    _select_case(dl, np.zeros(0, np.float32), np.zeros((2, 40), np.uint8), 3)


@pytest.mark.parametrize("k", [1, 4, 64, 300])
def test_select_rank_path_boundary(dl, k):
    """Sequences with 255, 256 (placed by rank) and 257 (radix select) candidates, one per
    sequence in one launch, with exact ties: every path gives the oracle's selection."""
    rng = np.random.default_rng(k)
    B, L = 3, 400
    M = np.zeros((B, L), np.uint8)
    for b, n_b in enumerate((255, 256, 257)):
        M[b, rng.choice(L, n_b, replace=False)] = 1
    n = int(M.sum())
    conf = (rng.integers(1, 17, size=n) / 16.0).astype(np.float32)
    tok = rng.integers(0, 1000, size=n).astype(np.int32)
    _select_case(dl, conf, M, k, tok_np=tok)
    # a window that leaves 256 candidates in one sequence and 257 in another
    lo = np.array([0, 0, 0], np.int32)
    hi = np.array([L, L, L], np.int32)
    _select_case(dl, conf, M, k, (lo, hi))
