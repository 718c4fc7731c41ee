"""Property tests of the oracle against the pure-Python brute force, over many random small
inputs (hypothesis): compaction with and without windows, top-k and threshold selection
(with exact ties), per-row statistics, and the split-vocabulary merge over any partition.
CPU only; the brute force shares no code with the oracle."""
import math

import numpy as np
from hypothesis import given, settings, strategies as st

import oracle.brute as BR
import oracle.oracle as O

SETTINGS = settings(max_examples=150, deadline=None, derandomize=True)


@st.composite
def masks(draw, max_b=4, max_l=24):
    B = draw(st.integers(1, max_b))
    L = draw(st.integers(1, max_l))
    rows = [[draw(st.integers(0, 1)) for _ in range(L)] for _ in range(B)]
    return rows


@st.composite
def masks_and_windows(draw):
    rows = draw(masks())
    L = len(rows[0])
    lo = [draw(st.integers(-3, L + 3)) for _ in rows]
    hi = [draw(st.integers(-3, L + 3)) for _ in rows]
    return rows, lo, hi


@SETTINGS
@given(masks())
def test_compaction(rows):
    row_idx, seq_off, count = O.mask_compact(np.array(rows, dtype=np.uint8))
    b_idx, b_off = BR.compact(rows)
    assert row_idx.tolist() == b_idx and seq_off.tolist() == b_off and count == len(b_idx)


@SETTINGS
@given(masks_and_windows())
def test_windowed_compaction(mw):
    rows, lo, hi = mw
    Mw = O.window_mask(np.array(rows, dtype=np.uint8), lo, hi)
    row_idx, seq_off, _ = O.mask_compact(Mw)
    b_idx, b_off = BR.compact_window(rows, lo, hi)
    assert row_idx.tolist() == b_idx and seq_off.tolist() == b_off


def _scores(draw, n, ties):
    if ties:                                           # few distinct values: exact ties
        return [draw(st.integers(0, 3)) / 4.0 for _ in range(n)]
    return [draw(st.floats(-4, 4, allow_nan=False, width=32)) for _ in range(n)]


@st.composite
def selections(draw):
    rows, lo, hi = draw(masks_and_windows())
    n = sum(map(sum, rows))
    scores = _scores(draw, n, draw(st.booleans()))
    k = draw(st.integers(1, 8))
    use_win = draw(st.booleans())
    return rows, scores, k, (lo, hi) if use_win else None


def _candidates(rows, scores, win):
    L = len(rows[0])
    row_idx, seq_off = BR.compact(rows)
    per_seq = []
    for b in range(len(rows)):
        c = []
        for r in range(seq_off[b], seq_off[b + 1]):
            pos = row_idx[r] - b * L
            if win is None or win[0][b] <= pos < win[1][b]:
                c.append((scores[r], pos))
        per_seq.append(c)
    return per_seq


@SETTINGS
@given(selections())
def test_topk_selection(sel):
    rows, scores, k, win = sel
    M = np.array(rows, dtype=np.uint8)
    row_idx, seq_off, _ = O.mask_compact(M)
    idx, n_sel = O.select_unmask(np.array(scores, dtype=np.float64), row_idx, seq_off, M.shape[1],
                                 k, None if win is None else win[0], None if win is None else win[1])
    for b, cands in enumerate(_candidates(rows, scores, win)):
        want = BR.topk(cands, k)
        assert n_sel[b] == len(want)
        assert idx[b].tolist() == want + [-1] * (k - len(want))


@SETTINGS
@given(selections(), st.sampled_from([-1.0, 0.0, 0.25, 0.5, 0.75, 2.0]), st.integers(0, 4))
def test_threshold_selection(sel, tau, min_sel):
    rows, scores, k, win = sel
    M = np.array(rows, dtype=np.uint8)
    row_idx, seq_off, _ = O.mask_compact(M)
    idx, n_sel = O.select_unmask_threshold(np.array(scores, dtype=np.float64), row_idx, seq_off,
                                           M.shape[1], k, tau, min_sel,
                                           None if win is None else win[0],
                                           None if win is None else win[1])
    for b, cands in enumerate(_candidates(rows, scores, win)):
        want = BR.select_threshold(cands, k, tau, min_sel)
        assert n_sel[b] == len(want)
        assert idx[b].tolist() == want + [-1] * (k - len(want))


@st.composite
def logit_rows(draw):
    n = draw(st.integers(1, 4))
    V = draw(st.integers(1, 40))
    ties = draw(st.booleans())
    if ties:
        Z = [[draw(st.integers(-3, 3)) * 0.5 for _ in range(V)] for _ in range(n)]
    else:
        Z = [[draw(st.floats(-30, 30, allow_nan=False)) for _ in range(V)] for _ in range(n)]
    return Z


@SETTINGS
@given(logit_rows())
def test_row_statistics(Z):
    tok, m, lse, conf = O.row_stats(np.array(Z, dtype=np.float64))
    ent, mar = O.row_policy_stats(np.array(Z, dtype=np.float64))
    for i, z in enumerate(Z):
        bt, bm, blse, bconf = BR.stats(z)
        be, bmar = BR.policy_stats(z)
        assert tok[i] == bt and m[i] == bm
        assert math.isclose(lse[i], blse, rel_tol=1e-12, abs_tol=1e-12)
        assert math.isclose(conf[i], bconf, rel_tol=1e-12)
        assert math.isclose(ent[i], be, rel_tol=1e-9, abs_tol=1e-12)
        assert math.isclose(mar[i], bmar, rel_tol=1e-9, abs_tol=1e-12)


@SETTINGS
@given(logit_rows(), st.data())
def test_merge_over_any_vocabulary_partition(Z, data):
    Z = np.array(Z, dtype=np.float64)
    V = Z.shape[1]
    cuts = sorted(set(data.draw(st.lists(st.integers(1, max(1, V - 1)), max_size=5)))) if V > 1 else []
    bounds = [0] + [c for c in cuts if 0 < c < V] + [V]
    parts = [O.partial_stats(Z, a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    tok, _, lse, conf = O.lse_merge(parts)
    for i, z in enumerate(Z.tolist()):
        bt, _, blse, bconf = BR.stats(z)
        assert tok[i] == bt                               # lowest token wins across splits
        assert math.isclose(lse[i], blse, rel_tol=1e-12, abs_tol=1e-12)
        assert math.isclose(conf[i], bconf, rel_tol=1e-12)
