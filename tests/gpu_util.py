"""Helpers shared by the GPU parity tests (marshalling and comparison rules only)."""
from __future__ import annotations

import numpy as np
import torch

import workloads as WL

# Tolerances of the parity bar: lse and conf relative error, and the top-2 logit gap below
# which the argmax may legitimately differ between fp32 accumulation and the fp64 oracle.
RTOL_LSE = 2e-3
RTOL_CONF = 2e-3
ARGMAX_GAP = 1e-3


def to_device(inp: dict) -> dict:
    out = dict(H=inp["H"].cuda(), W=inp["W"].cuda(), M=inp["M"].cuda())
    out["win_lo"] = None if inp["win_lo"] is None else torch.from_numpy(inp["win_lo"]).cuda()
    out["win_hi"] = None if inp["win_hi"] is None else torch.from_numpy(inp["win_hi"]).cuda()
    return out


def check_rows(gpu_tok, gpu_conf, gpu_lse, ref: dict, rows: np.ndarray, label: str) -> dict:
    """Compare GPU per-row results (compacted order) at `rows` with oracle arrays aligned
    with `rows`.  Returns error statistics; raises AssertionError on a violation."""
    g_tok = np.asarray(gpu_tok)[rows]
    g_conf = np.asarray(gpu_conf, dtype=np.float64)[rows]
    g_lse = np.asarray(gpu_lse, dtype=np.float64)[rows]
    # relative error of lse; below |lse| = 1 (only reachable with a tiny vocabulary, e.g.
    # V = 1 where lse is the single logit) the error is taken as absolute
    e_lse = np.abs(g_lse - ref["lse"]) / np.maximum(np.abs(ref["lse"]), 1.0)
    e_conf = np.abs(g_conf - ref["conf"]) / ref["conf"]
    tok_bad = (g_tok != ref["tok"]) & (ref["gap"] >= ARGMAX_GAP)
    stats = dict(rows=int(rows.size), max_rel_lse=float(e_lse.max(initial=0)),
                 max_rel_conf=float(e_conf.max(initial=0)),
                 tok_mismatch_excused=int(((g_tok != ref["tok"]) & ~tok_bad).sum()),
                 tok_mismatch=int(tok_bad.sum()))
    assert np.all(np.isfinite(g_lse)) and np.all(np.isfinite(g_conf)), label
    assert stats["max_rel_lse"] <= RTOL_LSE, (label, stats)
    assert stats["max_rel_conf"] <= RTOL_CONF, (label, stats)
    assert stats["tok_mismatch"] == 0, (label, stats, np.flatnonzero(tok_bad)[:10])
    return stats


def check_selection_exact(idx, n_sel, conf_gpu, row_idx, seq_off, L, k, win_lo, win_hi, O):
    """The GPU's selection equals the oracle's top-k on the GPU's own fp32 confidences."""
    ref_idx, ref_n = O.select_unmask(np.asarray(conf_gpu, dtype=np.float32), row_idx, seq_off,
                                     L, k, win_lo, win_hi)
    np.testing.assert_array_equal(np.asarray(n_sel), ref_n)
    np.testing.assert_array_equal(np.asarray(idx), ref_idx)


def check_selection_tolerant(idx, n_sel, ref_idx, ref_n, conf_of_pos, rtol=RTOL_CONF):
    """GPU selection vs the oracle's (fp64 conf) selection, as sets per sequence.  A
    difference is excused when the differing element's oracle confidence is within rtol of
    the oracle's k-th (smallest selected) confidence: a tie within the tolerance."""
    idx, ref_idx = np.asarray(idx), np.asarray(ref_idx)
    np.testing.assert_array_equal(np.asarray(n_sel), ref_n)
    excused = 0
    for b in range(idx.shape[0]):
        n = int(ref_n[b])
        g, r = set(idx[b, :n].tolist()), set(ref_idx[b, :n].tolist())
        if g == r:
            continue
        kth = min(conf_of_pos(b, p) for p in r)
        for p in g ^ r:
            c = conf_of_pos(b, p)
            assert abs(c - kth) <= rtol * kth, (b, p, c, kth)
            excused += 1
    return excused


def inputs_bits(inp: dict):
    return WL.bf16_bits(inp["H"]), WL.bf16_bits(inp["W"]), inp["M"].numpy()
