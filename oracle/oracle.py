"""CPU oracle for the diffusion-LLM decode step: mask-only logits, then confidence unmasking.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module.  The library (``mask_only_logits_b200``) never
does, and this module imports nothing from it.

Plain and slow on purpose: fp64 NumPy, one library matmul per chunk of the vocabulary, no
fusion, no blocking beyond that chunking, no online softmax.  What it computes:

* The subject page (Mosaic, "Mosaic: Unlocking Long-Context Inference for Diffusion LLMs
  via Global Memory Planning and Dynamic Peak Taming", TL;DR and Abstract) names a
  mask-only logits kernel that removes the redundant LM-head work of a dLLM step: logits
  are needed only at masked positions.  The definition written out here is the plain one:
  compute the full logits Z = H W^T for every position, then gather the masked rows.  The
  result for a row does not depend on any other row, so computing only the rows under test
  is exactly "full, then gather" for those rows (``full_then_gather`` checks that
  identity on small inputs).
* Per masked row: the predicted token is argmax_v Z (lowest v on ties), lse = log sum_v
  exp(Z_v), and the confidence is the largest softmax probability, exp(max - lse).  The
  pages only speak of "confidence/entropy-driven unmasking" (dLLM inference survey page,
  "Main Findings"); the max-probability reading is the plainest one.
* Per sequence: the k masked positions of highest confidence are unmasked (ties: lower
  position first), optionally restricted to the current semi-autoregressive block
  [lo, hi) (Sparse-dLLM page, "Experiment" and "More Results": block-wise decoding needs
  the current block only; blocks of 32 tokens).

Parity: pinned by brute force (``oracle/brute.py``), closed forms, a hand-worked fixture and
library routines (see ``tests/test_oracle.py``).
"""
from __future__ import annotations

import numpy as np

V_CHUNK = 8192


# --------------------------------------------------------------------------------------
# inputs
# --------------------------------------------------------------------------------------
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 bit patterns (uint16) as float64: bf16 is the top half of fp32."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------------------
# mask compaction (Mosaic, Abstract: mask-only logits)
# --------------------------------------------------------------------------------------
def mask_compact(M: np.ndarray):
    """Masked positions of M[B, L] (nonzero = masked), flattened b*L + l, ascending.

    Returns (row_idx int32 [count], seq_off int32 [B+1], count).  seq_off[b] is the number
    of masked positions in sequences 0..b-1, so sequence b owns rows seq_off[b]:seq_off[b+1].
    """
    M = np.asarray(M)
    B = M.shape[0]
    flat = M.reshape(-1) != 0
    row_idx = np.flatnonzero(flat).astype(np.int32)
    per_seq = (M.reshape(B, -1) != 0).sum(axis=1)
    seq_off = np.concatenate([[0], np.cumsum(per_seq)]).astype(np.int32)
    return row_idx, seq_off, int(row_idx.size)


def window_mask(M: np.ndarray, win_lo, win_hi) -> np.ndarray:
    """M restricted to the current block of each sequence: position l of sequence b stays
    masked only if win_lo[b] <= l < win_hi[b].  Block-wise (semi-autoregressive) decoding
    only ever unmasks positions of the current block (Sparse-dLLM page, "Experiment"), so
    these are the only rows whose logits a block step needs."""
    M = np.asarray(M)
    l = np.arange(M.shape[1], dtype=np.int64)[None, :]
    lo = np.asarray(win_lo, dtype=np.int64)[:, None]
    hi = np.asarray(win_hi, dtype=np.int64)[:, None]
    return ((M != 0) & (l >= lo) & (l < hi)).astype(np.uint8)


# --------------------------------------------------------------------------------------
# logits and per-row statistics
# --------------------------------------------------------------------------------------
def logits_rows(H64: np.ndarray, W64: np.ndarray) -> np.ndarray:
    """Z = H W^T in fp64 for the given rows of H (no bias, no scaling, temperature 1)."""
    return H64 @ W64.T


def row_stats(Z: np.ndarray):
    """Per row of Z [n, V]: (tok, m, lse, conf).

    m = max_v Z; tok = the first v attaining m; lse = m + log sum_v exp(Z - m);
    conf = exp(m - lse), the largest softmax probability.
    """
    Z = np.asarray(Z, dtype=np.float64)
    m = Z.max(axis=1)
    tok = Z.argmax(axis=1).astype(np.int32)
    s = np.exp(Z - m[:, None]).sum(axis=1)
    lse = m + np.log(s)
    conf = np.exp(m - lse)
    return tok, m, lse, conf


def row_policy_stats(Z: np.ndarray):
    """Per row of Z [n, V]: (entropy, margin) of the softmax p = softmax(Z).

    entropy = -sum_v p_v ln p_v (natural log); margin = p_(1) - p_(2), the gap between the
    largest and second-largest probability (0 when the maximum is attained twice; p_(1) when
    V = 1).  These are the alternative certainty scores of entropy- and margin-driven
    unmasking (dLLM inference survey page, "Main Findings": confidence/entropy-driven
    unmasking).
    """
    Z = np.asarray(Z, dtype=np.float64)
    m = Z.max(axis=1, keepdims=True)
    e = np.exp(Z - m)
    p = e / e.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        plogp = np.where(p > 0, p * np.log(p), 0.0)
    entropy = -plogp.sum(axis=1)
    if Z.shape[1] < 2:
        margin = p[:, 0].copy()
    else:
        top2 = np.partition(p, Z.shape[1] - 2, axis=1)[:, -2:]
        margin = top2[:, 1] - top2[:, 0]
    return entropy, margin


def rows_stats_chunked(H_rows_bits: np.ndarray, W_bits: np.ndarray, chunk: int = V_CHUNK,
                       with_policy: bool = False, W64: np.ndarray | None = None):
    """(tok, m, lse, conf, top2_gap) for rows of H given as bf16 bits, W as bf16 bits.

    Logits are formed chunk by chunk over the vocabulary and kept whole per row before the
    statistics are taken (the statistics are those of ``row_stats`` on the full row); the
    chunking only bounds the fp64 copy of W held at once.  top2_gap = m - (second largest
    logit), used to exempt near-ties from exact argmax comparison.  W64, when given, is
    bf16_bits_to_f64(W_bits) computed once by the caller (the same values; callers that run
    many row sets against one W skip converting it every time).
    """
    H64 = bf16_bits_to_f64(H_rows_bits)
    n = H64.shape[0]
    V = W_bits.shape[0]
    Z = np.empty((n, V), dtype=np.float64)
    for v0 in range(0, V, chunk):
        v1 = min(V, v0 + chunk)
        Wc = W64[v0:v1] if W64 is not None else bf16_bits_to_f64(W_bits[v0:v1])
        Z[:, v0:v1] = logits_rows(H64, Wc)
    tok, m, lse, conf = row_stats(Z)
    gap = top2_gap(Z)
    if with_policy:
        entropy, margin = row_policy_stats(Z)
        return tok, m, lse, conf, gap, entropy, margin
    return tok, m, lse, conf, gap


def top2_gap(Z: np.ndarray) -> np.ndarray:
    """max - second max of each row (0 when the maximum is attained twice); inf if V == 1."""
    if Z.shape[1] < 2:
        return np.full(Z.shape[0], np.inf)
    part = np.partition(Z, Z.shape[1] - 2, axis=1)
    return part[:, -1] - part[:, -2]


# --------------------------------------------------------------------------------------
# split-vocabulary partials and their merge (helper pinned by split invariance)
# --------------------------------------------------------------------------------------
def partial_stats(Z: np.ndarray, v0: int, v1: int):
    """(m, s, a) of Z[:, v0:v1]: max, sum exp(Z - m) and first argmax (as a global index)."""
    Zs = Z[:, v0:v1]
    m = Zs.max(axis=1)
    s = np.exp(Zs - m[:, None]).sum(axis=1)
    a = (Zs.argmax(axis=1) + v0).astype(np.int32)
    return m, s, a


def lse_merge(parts):
    """Merge partials [(m_j, s_j, a_j)] of consecutive vocabulary ranges (ascending).

    m* = max_j m_j; s* = sum_j s_j exp(m_j - m*); tok = a_j of the first j with m_j = m*;
    lse = m* + log s*; conf = exp(m* - lse).
    """
    ms = np.stack([p[0] for p in parts])
    ss = np.stack([p[1] for p in parts])
    aa = np.stack([p[2] for p in parts])
    m = ms.max(axis=0)
    s = (ss * np.exp(ms - m[None, :])).sum(axis=0)
    first = (ms == m[None, :]).argmax(axis=0)
    tok = aa[first, np.arange(aa.shape[1])].astype(np.int32)
    lse = m + np.log(s)
    conf = np.exp(m - lse)
    return tok, m, lse, conf


# --------------------------------------------------------------------------------------
# unmask selection (dLLM survey page, "Main Findings": confidence-driven unmasking)
# --------------------------------------------------------------------------------------
def select_unmask(conf, row_idx, seq_off, L: int, k: int, win_lo=None, win_hi=None):
    """Per sequence b, the k candidate positions of highest confidence.

    Candidates are sequence b's masked positions l (row_idx - b*L), restricted to
    [win_lo[b], win_hi[b]) when a window is given.  Order: confidence descending, then
    position ascending.  Returns idx int32 [B, k] (positions in [0, L), -1 past n_sel)
    and n_sel int32 [B] = min(k, number of candidates).

    ``conf`` is compared in the precision it is given in (float32 when checking a GPU
    selection on the GPU's own confidences, float64 for end-to-end oracle runs).
    """
    conf = np.asarray(conf)
    row_idx = np.asarray(row_idx, dtype=np.int64)
    seq_off = np.asarray(seq_off, dtype=np.int64)
    B = seq_off.size - 1
    idx = np.full((B, k), -1, dtype=np.int32)
    n_sel = np.zeros(B, dtype=np.int32)
    for b in range(B):
        r0, r1 = seq_off[b], seq_off[b + 1]
        pos = row_idx[r0:r1] - b * L
        c = conf[r0:r1]
        if win_lo is not None:
            keep = (pos >= win_lo[b]) & (pos < win_hi[b])
            pos, c = pos[keep], c[keep]
        order = np.lexsort((pos, -c))         # primary: -conf ascending; secondary: pos
        take = order[:k]
        n_sel[b] = take.size
        idx[b, :take.size] = pos[take]
    return idx, n_sel


# --------------------------------------------------------------------------------------
# the whole step
# --------------------------------------------------------------------------------------
def select_unmask_threshold(score, row_idx, seq_off, L: int, k: int, threshold: float,
                            min_sel: int = 1, win_lo=None, win_hi=None):
    """Threshold-based parallel unmasking (dLLM pages: decoding thresholds): per sequence,
    every candidate whose score is at least `threshold` is unmasked, at most k of them, and
    at least min(min_sel, number of candidates) (the best ones) so that decoding always
    advances.  Order and ties as in ``select_unmask`` (score descending, position
    ascending).  threshold = -inf gives plain top-k.
    """
    score = np.asarray(score)
    row_idx = np.asarray(row_idx, dtype=np.int64)
    seq_off = np.asarray(seq_off, dtype=np.int64)
    B = seq_off.size - 1
    idx = np.full((B, k), -1, dtype=np.int32)
    n_sel = np.zeros(B, dtype=np.int32)
    for b in range(B):
        r0, r1 = seq_off[b], seq_off[b + 1]
        pos = row_idx[r0:r1] - b * L
        c = score[r0:r1]
        if win_lo is not None:
            keep = (pos >= win_lo[b]) & (pos < win_hi[b])
            pos, c = pos[keep], c[keep]
        n_q = int((c >= threshold).sum())
        n_take = min(k, max(min(min_sel, c.size), n_q))
        order = np.lexsort((pos, -c))[:n_take]
        n_sel[b] = n_take
        idx[b, :n_take] = pos[order]
    return idx, n_sel


def oracle_rows(H_bits, W_bits, M, rows=None):
    """Mask-only logits statistics for masked rows (all, or the given compacted rows).

    Returns dict(row_idx, seq_off, count, rows, tok, m, lse, conf, gap) with the per-row
    arrays aligned with ``rows`` (compacted row numbers).
    """
    row_idx, seq_off, count = mask_compact(M)
    if rows is None:
        rows = np.arange(count, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    H_sel = np.asarray(H_bits)[row_idx[rows]]
    tok, m, lse, conf, gap, entropy, margin = rows_stats_chunked(H_sel, np.asarray(W_bits),
                                                                 with_policy=True)
    return dict(row_idx=row_idx, seq_off=seq_off, count=count, rows=rows,
                tok=tok, m=m, lse=lse, conf=conf, gap=gap, entropy=entropy, margin=margin)


def oracle_step(H_bits, W_bits, M, k, win_lo=None, win_hi=None):
    """One full decode step on every masked row: compaction, logits statistics, selection."""
    M = np.asarray(M)
    out = oracle_rows(H_bits, W_bits, M)
    L = M.shape[1]
    idx, n_sel = select_unmask(out["conf"], out["row_idx"], out["seq_off"], L, k,
                               win_lo, win_hi)
    out.update(idx=idx, n_sel=n_sel)
    return out


def oracle_block_step(H_bits, W_bits, M, k, win_lo, win_hi):
    """A decode step with current-block-only logits: statistics for the masked rows inside
    the windows only, then the same windowed selection as ``oracle_step``."""
    return oracle_step(H_bits, W_bits, window_mask(M, win_lo, win_hi), k, win_lo, win_hi)


def full_then_gather(H_bits, W_bits, M):
    """The literal definition: logits for EVERY position, statistics, then gather masked rows.

    Feasible only for small inputs; used to check that mask-only results equal it.
    """
    H64 = bf16_bits_to_f64(H_bits)
    W64 = bf16_bits_to_f64(W_bits)
    Z_full = logits_rows(H64, W64)
    tok, m, lse, conf = row_stats(Z_full)
    row_idx, seq_off, count = mask_compact(M)
    return dict(row_idx=row_idx, seq_off=seq_off, count=count, tok=tok[row_idx],
                m=m[row_idx], lse=lse[row_idx], conf=conf[row_idx], Z_full=Z_full)
