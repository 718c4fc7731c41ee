"""Pure-Python brute force for tiny inputs: explicit loops, ``math.fsum``, ``sorted``.

TEST INFRASTRUCTURE ONLY (see ``oracle/oracle.py``).  Independent of the NumPy oracle: no
NumPy arithmetic, no shared helpers; it exists to pin the oracle on inputs small enough to
loop over.  The quantities are those of the Mosaic page's mask-only logits step and the
confidence-driven unmasking of the dLLM survey page ("Main Findings").
"""
from __future__ import annotations

import math
import struct


def bf16_to_float(bits: int) -> float:
    """bfloat16 bit pattern -> Python float (exact): it is the upper 16 bits of a float32."""
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def compact(mask_rows):
    """mask_rows: list of B lists of 0/1 -> (row_idx, seq_off) by explicit enumeration."""
    row_idx, seq_off = [], [0]
    L = len(mask_rows[0]) if mask_rows else 0
    for b, row in enumerate(mask_rows):
        for l, v in enumerate(row):
            if v:
                row_idx.append(b * L + l)
        seq_off.append(len(row_idx))
    return row_idx, seq_off


def compact_window(mask_rows, win_lo, win_hi):
    """Like ``compact`` but only positions l of sequence b with win_lo[b] <= l < win_hi[b]."""
    row_idx, seq_off = [], [0]
    L = len(mask_rows[0]) if mask_rows else 0
    for b, row in enumerate(mask_rows):
        for l, v in enumerate(row):
            if v and win_lo[b] <= l < win_hi[b]:
                row_idx.append(b * L + l)
        seq_off.append(len(row_idx))
    return row_idx, seq_off


def dot(h, w):
    """Correctly rounded dot product of two float lists (math.fsum of exact products)."""
    return math.fsum(a * b for a, b in zip(h, w))


def row_logits(h, W):
    return [dot(h, w) for w in W]


def stats(z):
    """(tok, m, lse, conf) of one logit row z by definition."""
    m = max(z)
    tok = next(i for i, x in enumerate(z) if x == m)
    s = math.fsum(math.exp(x - m) for x in z)
    lse = m + math.log(s)
    conf = math.exp(m - lse)
    return tok, m, lse, conf


def top2_gap(z):
    """Largest logit minus the second largest, by sorting the row (0 when the maximum occurs
    twice; infinite for a one-entry row, which has no second logit)."""
    if len(z) < 2:
        return math.inf
    zs = sorted(z, reverse=True)
    return zs[0] - zs[1]


def policy_stats(z):
    """(entropy, margin) of softmax(z) by definition: -sum p ln p and p_(1) - p_(2)."""
    m = max(z)
    e = [math.exp(x - m) for x in z]
    s = math.fsum(e)
    p = [x / s for x in e]
    ent = -math.fsum(q * math.log(q) for q in p if q > 0)
    ps = sorted(p, reverse=True)
    margin = ps[0] - ps[1] if len(ps) > 1 else ps[0]
    return ent, margin


def select_threshold(cands, k, threshold, min_sel=1):
    """cands: list of (score, pos); all with score >= threshold (at most k, at least
    min(min_sel, len(cands))), best first."""
    ranked = sorted(cands, key=lambda cp: (-cp[0], cp[1]))
    n_q = sum(1 for c, _ in cands if c >= threshold)
    n_take = min(k, max(min(min_sel, len(cands)), n_q))
    return [p for _, p in ranked[:n_take]]


def topk(cands, k):
    """cands: list of (conf, pos); the k best by (conf desc, pos asc)."""
    return [p for _, p in sorted(cands, key=lambda cp: (-cp[0], cp[1]))[:k]]


def step(H, W, mask_rows, k, win=None):
    """Whole decode step on lists: H [B*L][d] floats, W [V][d] floats, mask [B][L] 0/1."""
    B = len(mask_rows)
    L = len(mask_rows[0])
    row_idx, seq_off = compact(mask_rows)
    per_row = [stats(row_logits(H[p], W)) for p in row_idx]
    idx, n_sel = [], []
    for b in range(B):
        cands = []
        for r in range(seq_off[b], seq_off[b + 1]):
            pos = row_idx[r] - b * L
            if win is None or (win[0][b] <= pos < win[1][b]):
                cands.append((per_row[r][3], pos))
        sel = topk(cands, k)
        n_sel.append(len(sel))
        idx.append(sel + [-1] * (k - len(sel)))
    return dict(row_idx=row_idx, seq_off=seq_off,
                tok=[s[0] for s in per_row], m=[s[1] for s in per_row],
                lse=[s[2] for s in per_row], conf=[s[3] for s in per_row],
                idx=idx, n_sel=n_sel)
