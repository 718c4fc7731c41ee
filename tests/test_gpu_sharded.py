"""The vocabulary-parallel path on one GPU: the vocabulary is split into S contiguous
shards, ``masked_partials`` runs on each shard in turn and writes its partials straight into
that shard's slot of the gathered layout (what the all-gather would deliver), then
``lse_merge`` and the selection run as on every rank.  Only the collective is left out
(checked on CPU with gloo ranks in ``test_dist_gloo.py``); every kernel of the path runs.

Bar: as the single-GPU step (tok exact except near-ties, lse / conf within 2e-3 relative,
entropy / margin as in ``test_gpu_policy.py``), against the fp64 oracle over the whole
vocabulary; the selection bit-exact against the oracle's top-k of the merged confidences.
"""
import numpy as np
import pytest
import torch

import gpu_util as GU
import oracle.oracle as O
import workloads as WL
from mask_only_logits_b200 import dist as D

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import mask_only_logits_b200 as dl
    return dl


def _emulated_shards(dl, inp, S, stats=0):
    """All S shards of one step on this GPU; returns merged per-row results and the count."""
    from mask_only_logits_b200.sharded import PartialLayout
    cfg = inp["cfg"]
    dev = GU.to_device(inp)
    n = cfg.B * cfg.L
    lay = PartialLayout(n, extended=stats != 0)
    gathered = lay.empty(S, "cuda")
    gathered.fill_(float("nan"))                      # nothing stale can pass for a result
    i32 = dict(dtype=torch.int32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    row_idx, seq_off, count = torch.empty(n, **i32), torch.empty(cfg.B + 1, **i32), torch.empty(4, **i32)
    for j in range(S):
        v0, v1 = D.shard_range(cfg.V, j, S)
        ws = torch.empty(dl.workspace_bytes(cfg.B, cfg.L, cfg.d, v1 - v0), dtype=torch.uint8, device="cuda")
        f = lay.fields_of(gathered[j])
        dl.masked_partials(dev["H"], dev["M"], dev["W"][v0:v1].contiguous(), v0, stats, f["m"],
                           f["s"], f["a"], f.get("t"), f.get("m2"), row_idx, seq_off, count, ws)
    gf = lay.fields_of(gathered)
    tok, conf, lse = torch.empty(n, **i32), torch.empty(n, **f32), torch.empty(n, **f32)
    ent = torch.empty(n, **f32) if stats & dl.STAT_ENTROPY else None
    mar = torch.empty(n, **f32) if stats & dl.STAT_MARGIN else None
    dl.lse_merge(gf["m"], gf["s"], gf["a"], gf.get("t"), gf.get("m2"), lay.split_stride, S, count,
                 n, stats, tok, conf, lse, ent, mar)
    assert dl.get_status() == 0
    c = int(count[0])
    out = dict(count=c, tok=tok[:c].cpu().numpy(), conf=conf[:c].cpu().numpy(),
               lse=lse[:c].cpu().numpy(), row_idx=row_idx[:c].cpu().numpy(),
               seq_off=seq_off.cpu().numpy(), conf_dev=conf, row_idx_dev=row_idx,
               seq_off_dev=seq_off, tok_dev=tok)
    if ent is not None:
        out["entropy"] = ent[:c].cpu().numpy()
    if mar is not None:
        out["margin"] = mar[:c].cpu().numpy()
    return out


@pytest.mark.parametrize("name,S", [("cfg0", 2), ("cfg0", 3), ("cfg1", 2), ("cfg1", 4),
                                    ("cfg1", 8), ("cfg1_m64", 8), ("cfg4", 2)])
def test_sharded_matches_oracle(dl, name, S):
    inp = WL.make_inputs(WL.CONFIGS[name], seed=0)
    cfg = inp["cfg"]
    g = _emulated_shards(dl, inp, S)
    Hb, Wb, M = GU.inputs_bits(inp)
    row_idx, seq_off, count = O.mask_compact(M)
    assert g["count"] == count
    np.testing.assert_array_equal(g["row_idx"], row_idx)
    rows = np.arange(count) if count <= 2048 else WL.sample_rows(count, 512, seed=0)
    ref = O.oracle_rows(Hb, Wb, M, rows)
    GU.check_rows(g["tok"], g["conf"], g["lse"], ref, rows, f"{name}/S={S}")
    # the selection on the merged confidences, bit-exact
    idx = torch.empty(cfg.B, cfg.k, dtype=torch.int32, device="cuda")
    n_sel = torch.empty(cfg.B, dtype=torch.int32, device="cuda")
    lo = None if inp["win_lo"] is None else torch.from_numpy(inp["win_lo"]).cuda()
    hi = None if inp["win_hi"] is None else torch.from_numpy(inp["win_hi"]).cuda()
    dl.select_unmask(g["conf_dev"], g["row_idx_dev"], g["seq_off_dev"], cfg.B, cfg.L, cfg.k, idx,
                     n_sel, lo, hi)
    GU.check_selection_exact(idx.cpu().numpy(), n_sel.cpu().numpy(), g["conf"], row_idx, seq_off,
                             cfg.L, cfg.k, inp["win_lo"], inp["win_hi"], O)


@pytest.mark.parametrize("B,L,d,V,S", [(2, 300, 64, 1000, 3), (1, 700, 128, 4097, 5),
                                       (1, 200, 64, 7, 7), (3, 97, 192, 777, 2)])
def test_sharded_ragged_shards(dl, B, L, d, V, S):
    """Shards of odd sizes, including one-row shards (V = S = 7)."""
    inp = WL.make_inputs(WL.custom_config(B, L, d, V, 4, r=0.8), seed=11)
    g = _emulated_shards(dl, inp, S)
    Hb, Wb, M = GU.inputs_bits(inp)
    ref = O.oracle_rows(Hb, Wb, M)
    GU.check_rows(g["tok"], g["conf"], g["lse"], ref, np.arange(g["count"]), f"ragged S={S}")


def test_sharded_entropy_margin(dl):
    inp = WL.make_inputs(WL.custom_config(1, 1500, 128, 9000, 8, r=0.7), seed=4)
    g = _emulated_shards(dl, inp, 3, stats=dl.STAT_ENTROPY | dl.STAT_MARGIN)
    Hb, Wb, M = GU.inputs_bits(inp)
    ref = O.oracle_rows(Hb, Wb, M)
    e, m = g["entropy"].astype(np.float64), g["margin"].astype(np.float64)
    assert np.all(np.abs(e - ref["entropy"]) <= 2e-3 * np.abs(ref["entropy"]) + 2e-5)
    assert np.all(np.abs(m - ref["margin"]) <= 2e-3 * np.abs(ref["margin"]) + 1e-4 * ref["conf"])


def test_shard_tie_keeps_lowest_token(dl):
    """A maximum attained in two shards: the merged token is the one of the lower shard."""
    rng = np.random.default_rng(8)
    V, d = 600, 64
    # every other vocabulary row tiny: tokens 120 and 450 (equal rows) hold the maximum of
    # every row whose hidden state points along them (about half of the rows)
    W = torch.from_numpy((rng.standard_normal((V, d)) * 0.001).astype(np.float32)).to(torch.bfloat16)
    W[120] = torch.from_numpy((rng.standard_normal(d) * 0.3).astype(np.float32)).to(torch.bfloat16)
    W[450] = W[120]                           # shard 0 owns 120, shard 1 owns 450 (S = 2)
    inp = WL.make_inputs(WL.custom_config(1, 128, d, V, 4, r=1.0), seed=2)
    inp["W"] = W
    g = _emulated_shards(dl, inp, 2)
    ref = O.oracle_rows(GU.inputs_bits(inp)[0], WL.bf16_bits(W), inp["M"].numpy())
    at_tie = ref["tok"] == 120
    assert at_tie.sum() > 10
    assert np.all(g["tok"][at_tie] == 120)


def test_vocab_sharded_step_single_rank(dl):
    """VocabShardedStep with one rank (no collective): the full step through partials."""
    from mask_only_logits_b200.sharded import VocabShardedStep
    inp = WL.make_inputs(WL.CONFIGS["cfg0"], seed=3)
    cfg = inp["cfg"]
    dev = GU.to_device(inp)
    st = VocabShardedStep(cfg.B, cfg.L, cfg.d, cfg.V, cfg.k, rank=0, world=1)
    out = st.run(dev["H"], dev["M"], dev["W"])
    assert dl.get_status() == 0
    c = int(out["count"][0])
    Hb, Wb, M = GU.inputs_bits(inp)
    ref = O.oracle_rows(Hb, Wb, M)
    GU.check_rows(out["tok"][:c].cpu().numpy(), out["conf"][:c].cpu().numpy(),
                  out["lse"][:c].cpu().numpy(), ref, np.arange(c), "sharded-step")
    row_idx, seq_off, _ = O.mask_compact(M)
    GU.check_selection_exact(out["idx"].cpu().numpy(), out["n_sel"].cpu().numpy(),
                             out["conf"][:c].cpu().numpy(), row_idx, seq_off, cfg.L, cfg.k,
                             None, None, O)


def test_sharded_block_only_windows(dl):
    """Vocabulary shards with current-block-only rows (windows applied at compaction)."""
    cfg = WL.custom_config(4, 1024, 128, 3001, 4, mask="semi_ar", block=32)
    inp = WL.make_inputs(cfg, seed=6)
    lo, hi = WL.make_windows(cfg)
    dev = GU.to_device(inp)
    lo_d, hi_d = torch.from_numpy(lo).cuda(), torch.from_numpy(hi).cuda()
    from mask_only_logits_b200.sharded import PartialLayout
    S, n = 3, cfg.B * cfg.L
    lay = PartialLayout(n, extended=False)
    gathered = lay.empty(S, "cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    row_idx, seq_off, count = torch.empty(n, **i32), torch.empty(cfg.B + 1, **i32), torch.empty(4, **i32)
    for j in range(S):
        v0, v1 = D.shard_range(cfg.V, j, S)
        ws = torch.empty(dl.workspace_bytes(cfg.B, cfg.L, cfg.d, v1 - v0), dtype=torch.uint8, device="cuda")
        f = lay.fields_of(gathered[j])
        dl.masked_partials(dev["H"], dev["M"], dev["W"][v0:v1].contiguous(), v0, 0, f["m"], f["s"],
                           f["a"], None, None, row_idx, seq_off, count, ws, win_lo=lo_d, win_hi=hi_d)
    gf = lay.fields_of(gathered)
    tok, conf, lse = torch.empty(n, **i32), torch.empty(n, device="cuda"), torch.empty(n, device="cuda")
    dl.lse_merge(gf["m"], gf["s"], gf["a"], None, None, lay.split_stride, S, count, n, 0, tok, conf, lse)
    assert dl.get_status() == 0
    c = int(count[0])
    Mw = O.window_mask(inp["M"].numpy(), lo, hi)
    ref = O.oracle_rows(WL.bf16_bits(inp["H"]), WL.bf16_bits(inp["W"]), Mw)
    assert c == ref["count"] == cfg.B * 32
    np.testing.assert_array_equal(row_idx[:c].cpu().numpy(), ref["row_idx"])
    GU.check_rows(tok[:c].cpu().numpy(), conf[:c].cpu().numpy(), lse[:c].cpu().numpy(), ref,
                  np.arange(c), "sharded-block")
