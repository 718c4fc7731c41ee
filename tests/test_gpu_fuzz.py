"""Seeded random shapes through the whole step on the GPU, against the oracle: batch size,
sequence length, d, V, k, mask ratio, windows (selection-only or current-block-only),
extended statistics and the GEMM variant are all drawn per case.  Bars as in
test_gpu_parity.py / test_gpu_policy.py (tok exact except near-ties, lse / conf within
2e-3, selection bit-exact on the GPU's own scores)."""
import os

import numpy as np
import pytest
import torch

import gpu_util as GU
import oracle.oracle as O
import workloads as WL

pytestmark = pytest.mark.gpu

N_CASES = int(os.environ.get("DLLM_FUZZ_CASES", "100"))


@pytest.fixture(scope="module")
def dl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import mask_only_logits_b200 as dl
    return dl


def _draw(seed):
    rng = np.random.default_rng(1000 + seed)
    B = int(rng.integers(1, 5))
    L = int(rng.choice([1, 7, 64, 255, 256, 1000, 3000, 5000]))
    d = int(rng.choice([64, 128, 192, 256, 512]))
    V = int(rng.choice([1, 3, 255, 256, 257, 4096, 7777, 20000]))
    k = int(rng.choice([1, 2, 8, 33, 128]))
    r = float(rng.choice([0.0, 0.05, 0.5, 0.9, 1.0]))
    windows = int(rng.integers(0, 3))          # 0 none, 1 selection windows, 2 block-only
    variant = int(rng.integers(0, 3))
    stats = int(rng.integers(0, 4))
    return rng, B, L, d, V, k, r, windows, variant, stats


@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_step(dl, seed):
    rng, B, L, d, V, k, r, windows, variant, stats = _draw(seed)
    inp = WL.make_inputs(WL.custom_config(B, L, d, V, k, r=r, block_only=windows == 2), seed=seed)
    lo = hi = None
    if windows:
        lo = rng.integers(-2, L + 1, size=B).astype(np.int32)
        hi = (lo + rng.integers(0, max(2, L // 2), size=B)).astype(np.int32)
    M = inp["M"].numpy()
    Mrows = O.window_mask(M, lo, hi) if windows == 2 else M
    row_idx, seq_off, count = O.mask_compact(Mrows)
    n = B * L
    dev = GU.to_device(inp)
    i32 = dict(dtype=torch.int32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    tok, conf, lse = torch.empty(n, **i32), torch.empty(n, **f32), torch.empty(n, **f32)
    ent = torch.empty(n, **f32) if stats & 1 else None
    mar = torch.empty(n, **f32) if stats & 2 else None
    ri, so, cnt = torch.empty(n, **i32), torch.empty(B + 1, **i32), torch.empty(4, **i32)
    ws = torch.empty(dl.workspace_bytes(B, L, d, V), dtype=torch.uint8, device="cuda")
    lo_d = None if lo is None else torch.from_numpy(lo).cuda()
    hi_d = None if hi is None else torch.from_numpy(hi).cuda()
    dl.debug_set_gemm_variant(variant)
    try:
        dl.masked_logits_ex(dev["H"], dev["M"], dev["W"], stats, tok, conf, lse, ent, mar, ri, so,
                            cnt, ws, win_lo=lo_d if windows == 2 else None,
                            win_hi=hi_d if windows == 2 else None)
        idx = torch.empty(B, k, **i32)
        n_sel = torch.empty(B, **i32)
        dl.select_unmask(conf, ri, so, B, L, k, idx, n_sel, lo_d if windows else None,
                         hi_d if windows else None)
        assert dl.get_status() == 0
    finally:
        dl.debug_set_gemm_variant(0)
    c = int(cnt[0])
    case = dict(B=B, L=L, d=d, V=V, k=k, r=r, windows=windows, variant=variant, stats=stats)
    assert c == count, case
    np.testing.assert_array_equal(ri[:c].cpu().numpy(), row_idx)
    np.testing.assert_array_equal(so.cpu().numpy(), seq_off)
    conf_g = conf[:c].cpu().numpy()
    GU.check_selection_exact(idx.cpu().numpy(), n_sel.cpu().numpy(), conf_g, row_idx, seq_off, L,
                             k, lo if windows else None, hi if windows else None, O)
    if c == 0:
        return
    rows = np.arange(c) if c <= 1500 else WL.sample_rows(c, 600, seed=seed)
    ref = O.oracle_rows(WL.bf16_bits(inp["H"]), WL.bf16_bits(inp["W"]), Mrows, rows)
    GU.check_rows(tok[:c].cpu().numpy(), conf_g, lse[:c].cpu().numpy(), ref, rows, str(case))
    if ent is not None:
        e = ent[:c].cpu().numpy().astype(np.float64)[rows]
        assert np.all(np.abs(e - ref["entropy"]) <= 2e-3 * np.abs(ref["entropy"]) + 2e-5), case
    if mar is not None:
        m = mar[:c].cpu().numpy().astype(np.float64)[rows]
        assert np.all(np.abs(m - ref["margin"]) <= 2e-3 * np.abs(ref["margin"]) + 1e-4 * ref["conf"]), case
