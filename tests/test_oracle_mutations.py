"""Plant plausible mistakes in a private copy of the oracle and check that the pins catch
each one: a dropped term, a wrong sign, a wrong index, a transposed operand, a reversed
tie-break.  The mistakes live only in the copy, on the CPU."""
import importlib.util
import os

import numpy as np
import pytest

import oracle_pins as P

ORACLE_FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "oracle", "oracle.py")


def _fresh_copy():
    spec = importlib.util.spec_from_file_location("oracle_mutant", ORACLE_FILE)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _row_stats_argmin(Z):
    m = Z.max(axis=1)
    tok = Z.argmin(axis=1).astype(np.int32)
    s = np.exp(Z - m[:, None]).sum(axis=1)
    return tok, m, m + np.log(s), np.exp(m - (m + np.log(s)))


def _row_stats_drop_m(Z):
    m = Z.max(axis=1)
    s = np.exp(Z - m[:, None]).sum(axis=1)
    lse = np.log(s)                                   # dropped "+ m"
    return Z.argmax(axis=1).astype(np.int32), m, lse, np.exp(m - (m + np.log(s)))


def _row_stats_sign(Z):
    m = Z.max(axis=1)
    s = np.exp(Z - m[:, None]).sum(axis=1)
    lse = m + np.log(s)
    return Z.argmax(axis=1).astype(np.int32), m, lse, np.exp(lse - m)   # wrong sign


def _row_stats_no_shift(Z):
    m = Z.max(axis=1)
    s = np.exp(Z).sum(axis=1)                          # forgot to subtract the max
    lse = m + np.log(s)
    return Z.argmax(axis=1).astype(np.int32), m, lse, np.exp(m - lse)


def _row_stats_last_argmax(Z):
    m = Z.max(axis=1)
    rev = Z[:, ::-1]
    tok = (Z.shape[1] - 1 - rev.argmax(axis=1)).astype(np.int32)   # highest index on ties
    s = np.exp(Z - m[:, None]).sum(axis=1)
    lse = m + np.log(s)
    return tok, m, lse, np.exp(m - lse)


def _logits_transposed(H64, W64):
    return (W64 @ H64.T)                               # transposed result


def _bf16_shift15(bits):
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(15)).view(np.float32).astype(np.float64)


def _lse_merge_no_rescale(parts):
    ms = np.stack([p[0] for p in parts])
    ss = np.stack([p[1] for p in parts])
    aa = np.stack([p[2] for p in parts])
    m = ms.max(axis=0)
    s = ss.sum(axis=0)                                 # dropped exp(m_j - m*)
    first = (ms == m[None, :]).argmax(axis=0)
    tok = aa[first, np.arange(aa.shape[1])].astype(np.int32)
    lse = m + np.log(s)
    return tok, m, lse, np.exp(m - lse)


def _mask_compact_bad_offsets(M):
    M = np.asarray(M)
    flat = M.reshape(-1) != 0
    row_idx = np.flatnonzero(flat).astype(np.int32)
    per_seq = (M.reshape(M.shape[0], -1) != 0).sum(axis=1)
    seq_off = np.concatenate([np.cumsum(per_seq), [row_idx.size]]).astype(np.int32)  # shifted
    return row_idx, seq_off, int(row_idx.size)


def _make_select(variant):
    def select_unmask(conf, row_idx, seq_off, L, k, win_lo=None, win_hi=None):
        conf = np.asarray(conf)
        row_idx = np.asarray(row_idx, dtype=np.int64)
        seq_off = np.asarray(seq_off, dtype=np.int64)
        B = seq_off.size - 1
        idx = np.full((B, k), -1, dtype=np.int32)
        n_sel = np.zeros(B, dtype=np.int32)
        for b in range(B):
            r0, r1 = seq_off[b], seq_off[b + 1]
            pos = row_idx[r0:r1] - (0 if variant == "no_seq_base" else b * L)
            c = conf[r0:r1]
            if win_lo is not None:
                keep = (pos >= win_lo[b]) & (pos <= win_hi[b]) if variant == "closed_window" \
                    else (pos >= win_lo[b]) & (pos < win_hi[b])
                pos, c = pos[keep], c[keep]
            if variant == "tie_desc":
                order = np.lexsort((-pos, -c))
            elif variant == "ascending":
                order = np.lexsort((pos, c))
            else:
                order = np.lexsort((pos, -c))
            take = order[:k]
            n_sel[b] = take.size
            idx[b, :take.size] = pos[take]
        return idx, n_sel
    return select_unmask


def _policy_entropy_log2(Z):
    Z = np.asarray(Z, dtype=np.float64)
    m = Z.max(axis=1, keepdims=True)
    p = np.exp(Z - m)
    p = p / p.sum(axis=1, keepdims=True)
    ent = -(p * np.log2(np.where(p > 0, p, 1.0))).sum(axis=1)      # wrong log base
    s = np.sort(p, axis=1)
    return ent, s[:, -1] - (s[:, -2] if p.shape[1] > 1 else 0)


def _policy_margin_of_logits(Z):
    Z = np.asarray(Z, dtype=np.float64)
    m = Z.max(axis=1, keepdims=True)
    p = np.exp(Z - m)
    p = p / p.sum(axis=1, keepdims=True)
    ent = -(p * np.log(np.where(p > 0, p, 1.0))).sum(axis=1)
    s = np.sort(Z, axis=1)                                           # logits, not probabilities
    return ent, s[:, -1] - (s[:, -2] if Z.shape[1] > 1 else 0)


def _threshold_strict(score, row_idx, seq_off, L, k, threshold, min_sel=1, win_lo=None, win_hi=None):
    score = np.asarray(score)
    row_idx = np.asarray(row_idx, dtype=np.int64)
    seq_off = np.asarray(seq_off, dtype=np.int64)
    B = seq_off.size - 1
    idx = np.full((B, k), -1, dtype=np.int32)
    n_sel = np.zeros(B, dtype=np.int32)
    for b in range(B):
        pos = row_idx[seq_off[b]:seq_off[b + 1]] - b * L
        c = score[seq_off[b]:seq_off[b + 1]]
        if win_lo is not None:
            keep = (pos >= win_lo[b]) & (pos < win_hi[b])
            pos, c = pos[keep], c[keep]
        n_q = int((c > threshold).sum())                              # strict: drops equality
        n_take = min(k, max(min(min_sel, c.size), n_q))
        order = np.lexsort((pos, -c))[:n_take]
        n_sel[b] = n_take
        idx[b, :n_take] = pos[order]
    return idx, n_sel


def _window_mask_closed(M, win_lo, win_hi):
    M = np.asarray(M)
    l = np.arange(M.shape[1])[None, :]
    inside = (l >= np.asarray(win_lo)[:, None]) & (l <= np.asarray(win_hi)[:, None])   # closed
    return ((M != 0) & inside).astype(np.uint8)


def _window_mask_ignores_seq(M, win_lo, win_hi):
    M = np.asarray(M)
    l = np.arange(M.shape[1])[None, :]
    inside = (l >= int(np.asarray(win_lo)[0])) & (l < int(np.asarray(win_hi)[0]))  # seq 0's window
    return ((M != 0) & inside).astype(np.uint8)


def _policy_entropy_no_mean(Z):
    Z = np.asarray(Z, dtype=np.float64)
    m = Z.max(axis=1, keepdims=True)
    e = np.exp(Z - m)
    tot = e.sum(axis=1)
    ent = np.log(tot)                                  # dropped "- sum p (z - m)"
    p = e / tot[:, None]
    s = np.sort(p, axis=1)
    return ent, s[:, -1] - (s[:, -2] if p.shape[1] > 1 else 0)


def _threshold_no_floor(score, row_idx, seq_off, L, k, threshold, min_sel=1, win_lo=None,
                        win_hi=None):
    score = np.asarray(score)
    row_idx = np.asarray(row_idx, dtype=np.int64)
    seq_off = np.asarray(seq_off, dtype=np.int64)
    B = seq_off.size - 1
    idx = np.full((B, k), -1, dtype=np.int32)
    n_sel = np.zeros(B, dtype=np.int32)
    for b in range(B):
        pos = row_idx[seq_off[b]:seq_off[b + 1]] - b * L
        c = score[seq_off[b]:seq_off[b + 1]]
        if win_lo is not None:
            keep = (pos >= win_lo[b]) & (pos < win_hi[b])
            pos, c = pos[keep], c[keep]
        n_take = min(k, int((c >= threshold).sum()))             # min_sel floor ignored
        order = np.lexsort((pos, -c))[:n_take]
        n_sel[b] = n_take
        idx[b, :n_take] = pos[order]
    return idx, n_sel


def _partial_local_argmax(Z, v0, v1):
    Zs = Z[:, v0:v1]
    m = Zs.max(axis=1)
    return m, np.exp(Zs - m[:, None]).sum(axis=1), Zs.argmax(axis=1).astype(np.int32)  # no + v0


def _mask_compact_not_flattened(M):
    M = np.asarray(M)
    B = M.shape[0]
    bs, ls = np.nonzero(M != 0)
    row_idx = ls.astype(np.int32)                                 # l instead of b * L + l
    per_seq = (M != 0).sum(axis=1)
    return row_idx, np.concatenate([[0], np.cumsum(per_seq)]).astype(np.int32), int(row_idx.size)


def _top2_gap_zero(Z):
    return np.zeros(Z.shape[0])                                    # every near-tie excused


def _make_chunked_drops_last_column(mod):
    def rows_stats_chunked(H_rows_bits, W_bits, chunk=mod.V_CHUNK, with_policy=False, W64=None):
        H64 = mod.bf16_bits_to_f64(H_rows_bits)
        V = W_bits.shape[0]
        Z = np.zeros((H64.shape[0], V), dtype=np.float64)
        for v0 in range(0, V, chunk):
            v1 = min(V, v0 + chunk)
            Wc = mod.bf16_bits_to_f64(W_bits[v0:v1 - 1])             # last column of the chunk lost
            Z[:, v0:v1 - 1] = mod.logits_rows(H64, Wc)
        tok, m, lse, conf = mod.row_stats(Z)
        gap = mod.top2_gap(Z)
        if with_policy:
            entropy, margin = mod.row_policy_stats(Z)
            return tok, m, lse, conf, gap, entropy, margin
        return tok, m, lse, conf, gap
    return rows_stats_chunked


MUTATIONS = {
    "top2_gap_always_zero": ("top2_gap", _top2_gap_zero),
    "chunk_drops_last_column": ("rows_stats_chunked", _make_chunked_drops_last_column),
    "entropy_drops_mean_term": ("row_policy_stats", _policy_entropy_no_mean),
    "threshold_ignores_min_sel": ("select_unmask_threshold", _threshold_no_floor),
    "partial_argmax_not_global": ("partial_stats", _partial_local_argmax),
    "compact_positions_not_flattened": ("mask_compact", _mask_compact_not_flattened),
    "block_window_closed": ("window_mask", _window_mask_closed),
    "block_window_first_seq_only": ("window_mask", _window_mask_ignores_seq),
    "entropy_log2": ("row_policy_stats", _policy_entropy_log2),
    "margin_of_logits": ("row_policy_stats", _policy_margin_of_logits),
    "threshold_strict": ("select_unmask_threshold", _threshold_strict),
    "argmin_for_argmax": ("row_stats", _row_stats_argmin),
    "lse_drops_max": ("row_stats", _row_stats_drop_m),
    "conf_wrong_sign": ("row_stats", _row_stats_sign),
    "softmax_not_shifted": ("row_stats", _row_stats_no_shift),
    "argmax_last_on_ties": ("row_stats", _row_stats_last_argmax),
    "logits_transposed": ("logits_rows", _logits_transposed),
    "bf16_decode_wrong_shift": ("bf16_bits_to_f64", _bf16_shift15),
    "merge_drops_rescale": ("lse_merge", _lse_merge_no_rescale),
    "seq_off_shifted": ("mask_compact", _mask_compact_bad_offsets),
    "topk_tie_break_reversed": ("select_unmask", _make_select("tie_desc")),
    "topk_ascending": ("select_unmask", _make_select("ascending")),
    "topk_position_not_rebased": ("select_unmask", _make_select("no_seq_base")),
    "window_closed_interval": ("select_unmask", _make_select("closed_window")),
}


FACTORY_MUTATIONS = {"chunk_drops_last_column"}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name):
    attr, bad = MUTATIONS[name]
    mod = _fresh_copy()
    P.ALL_CHECKS[0](mod)            # the unmodified copy passes
    if name in FACTORY_MUTATIONS:   # mutants that call back into the copy they replace
        bad = bad(mod)
    setattr(mod, attr, bad)
    caught = []
    for check in P.ALL_CHECKS:
        try:
            check(mod)
        except Exception as e:       # noqa: BLE001 - any failure counts as detection
            caught.append((check.__name__, type(e).__name__))
    assert caught, f"no pin caught mutation {name}"
