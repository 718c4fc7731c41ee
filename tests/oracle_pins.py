"""Pin checks for the CPU oracle, written against an oracle-like namespace.

Each check raises AssertionError when the oracle disagrees with something fixed outside it:
a hand-worked fixture, a closed form, a library routine, an invariant or brute force.  The
checks take the namespace as an argument so that ``test_oracle_mutations.py`` can run them
against copies of the oracle with a planted mistake and show that some check fails.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import scipy.special
import torch

from oracle import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bits(a) -> np.ndarray:
    """Exact bf16 bit patterns of small float arrays (values chosen bf16-representable)."""
    t = torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(a, dtype=np.float32))), "not bf16-exact"
    return t.view(torch.int16).numpy().view(np.uint16)


def _rand_bits(rng: np.random.Generator, shape, scale=1.0) -> np.ndarray:
    x = torch.tensor(rng.standard_normal(shape).astype(np.float32) * scale).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


def _bf16_list(bits) -> list:
    return [[brute.bf16_to_float(b) for b in row] for row in np.asarray(bits)]


# ----------------------------------------------------------------------------------------
def check_handworked(o):
    g = json.load(open(os.path.join(GOLDEN, "handworked_step.json")))
    H, W, M = _bits(g["H"]), _bits(g["W"]), np.array(g["M"], dtype=np.uint8)
    out = o.oracle_step(H, W, M, g["k"])
    assert out["row_idx"].tolist() == g["row_idx"]
    assert out["seq_off"].tolist() == g["seq_off"]
    assert out["tok"].tolist() == g["tok"]
    np.testing.assert_allclose(out["m"], g["m"], rtol=0, atol=0)
    np.testing.assert_allclose(out["lse"], g["lse"], rtol=1e-14)
    np.testing.assert_allclose(out["conf"], g["conf"], rtol=1e-14)
    assert out["idx"].tolist() == g["idx"]
    assert out["n_sel"].tolist() == g["n_sel"]
    out1 = o.oracle_step(H, W, M, 1)
    assert out1["idx"].tolist() == g["k1_idx"]
    lo, hi = np.array(g["window_lo"]), np.array(g["window_hi"])
    outw = o.oracle_step(H, W, M, 2, lo, hi)
    assert outw["idx"].tolist() == g["window_k2_idx"]
    assert outw["n_sel"].tolist() == g["window_k2_n_sel"]
    # the logits themselves
    Z = o.logits_rows(o.bf16_bits_to_f64(H[out["row_idx"]]), o.bf16_bits_to_f64(W))
    np.testing.assert_array_equal(Z, np.array(g["logits"], dtype=np.float64))


def check_topk_ties(o):
    g = json.load(open(os.path.join(GOLDEN, "topk_ties.json")))
    M = np.array(g["M"], dtype=np.uint8)
    row_idx, seq_off, count = o.mask_compact(M)
    assert row_idx.tolist() == g["positions"]
    for dt in (np.float32, np.float64):
        conf = np.array(g["conf"], dtype=dt)
        for c in g["cases"]:
            lo = np.array([c["lo"]]) if "lo" in c else None
            hi = np.array([c["hi"]]) if "hi" in c else None
            idx, n_sel = o.select_unmask(conf, row_idx, seq_off, g["L"], c["k"], lo, hi)
            assert idx[0].tolist() == c["idx"], (c, idx)
            assert int(n_sel[0]) == c["n_sel"]


def check_compact(o, seeds=range(8)):
    rng = np.random.default_rng(123)
    cases = [np.zeros((1, 5), np.uint8), np.ones((2, 3), np.uint8),
             np.array([[0, 7, 0, 255, 1]], np.uint8)]
    for s in seeds:
        B, L = int(rng.integers(1, 5)), int(rng.integers(1, 40))
        cases.append((rng.random((B, L)) < rng.random()).astype(np.uint8))
    for M in cases:
        row_idx, seq_off, count = o.mask_compact(M)
        r2, s2 = brute.compact([[1 if v else 0 for v in row] for row in M.tolist()])
        assert row_idx.tolist() == r2 and seq_off.tolist() == s2 and count == len(r2)
        assert row_idx.dtype == np.int32 and seq_off.dtype == np.int32


def check_brute_random(o, n_cases=12):
    rng = np.random.default_rng(7)
    for _ in range(n_cases):
        B, L = int(rng.integers(1, 3)), int(rng.integers(1, 17))
        d, V = int(rng.integers(1, 9)), int(rng.integers(1, 33))
        k = int(rng.integers(1, 6))
        H, W = _rand_bits(rng, (B * L, d)), _rand_bits(rng, (V, d), 0.5)
        M = (rng.random((B, L)) < 0.6).astype(np.uint8)
        win = None
        if rng.random() < 0.5:
            lo = rng.integers(0, L, size=B)
            hi = np.minimum(L, lo + rng.integers(1, L + 1, size=B))
            win = (lo, hi)
        out = o.oracle_step(H, W, M, k, *(win if win else (None, None)))
        ref = brute.step(_bf16_list(H), _bf16_list(W), M.tolist(), k,
                         (win[0].tolist(), win[1].tolist()) if win else None)
        assert out["row_idx"].tolist() == ref["row_idx"]
        assert out["seq_off"].tolist() == ref["seq_off"]
        assert out["tok"].tolist() == ref["tok"]
        np.testing.assert_allclose(out["m"], ref["m"], rtol=1e-13, atol=1e-300)
        np.testing.assert_allclose(out["lse"], ref["lse"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(out["conf"], ref["conf"], rtol=1e-12)
        assert out["idx"].tolist() == ref["idx"]
        assert out["n_sel"].tolist() == ref["n_sel"]


def check_closed_forms(o):
    # (1) all vocabulary rows equal -> all logits equal: tok 0, conf 1/V, lse = z + ln V
    rng = np.random.default_rng(3)
    d, V = 16, 37
    w = _rand_bits(rng, (1, d))
    W = np.repeat(w, V, axis=0)
    H = _rand_bits(rng, (5, d))
    M = np.ones((1, 5), np.uint8)
    out = o.oracle_rows(H, W, M)
    z = o.bf16_bits_to_f64(H) @ o.bf16_bits_to_f64(w)[0]
    assert out["tok"].tolist() == [0] * 5
    np.testing.assert_allclose(out["conf"], 1.0 / V, rtol=1e-13)
    np.testing.assert_allclose(out["lse"], z + math.log(V), rtol=1e-13, atol=1e-13)
    # (2) W = [I_d; 0], H = c e_j -> tok j, lse = log(e^c + V - 1), conf = e^c / (e^c + V - 1)
    d, V = 8, 20
    Wf = np.zeros((V, d), np.float32)
    Wf[:d, :d] = np.eye(d)
    for j, c in [(0, 3.0), (5, 1.5), (7, 8.0), (3, 0.25)]:
        Hf = np.zeros((1, d), np.float32)
        Hf[0, j] = c
        out = o.oracle_rows(_bits(Hf), _bits(Wf), np.ones((1, 1), np.uint8))
        assert out["tok"].tolist() == [j]
        np.testing.assert_allclose(out["lse"], [math.log(math.exp(c) + V - 1)], rtol=1e-14)
        np.testing.assert_allclose(out["conf"], [math.exp(c) / (math.exp(c) + V - 1)], rtol=1e-14)
    # (3) V = 1 -> conf 1, lse = the single logit, tok 0
    H = _rand_bits(rng, (4, 8))
    W = _rand_bits(rng, (1, 8))
    out = o.oracle_rows(H, W, np.ones((1, 4), np.uint8))
    np.testing.assert_allclose(out["conf"], 1.0, rtol=0, atol=0)
    np.testing.assert_allclose(out["lse"], o.bf16_bits_to_f64(H) @ o.bf16_bits_to_f64(W)[0],
                               rtol=1e-15)
    assert out["tok"].tolist() == [0] * 4


def check_library_routines(o):
    """lse against scipy.special.logsumexp, conf against max of scipy.special.softmax,
    tok against torch.argmax, the bf16 decoding against torch's bf16 -> float64 cast."""
    rng = np.random.default_rng(11)
    H, W = _rand_bits(rng, (24, 64)), _rand_bits(rng, (300, 64), 0.3)
    M = np.ones((2, 12), np.uint8)
    out = o.oracle_rows(H, W, M)
    Ht = torch.from_numpy(H.view(np.int16)).view(torch.bfloat16).double()
    Wt = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).double()
    np.testing.assert_array_equal(o.bf16_bits_to_f64(H), Ht.numpy())
    Z = (Ht @ Wt.T).numpy()
    np.testing.assert_allclose(out["lse"], scipy.special.logsumexp(Z, axis=1), rtol=1e-12)
    np.testing.assert_allclose(out["conf"], scipy.special.softmax(Z, axis=1).max(axis=1),
                               rtol=1e-12)
    assert out["tok"].tolist() == torch.argmax(torch.from_numpy(Z), dim=1).tolist()


def check_invariants(o):
    rng = np.random.default_rng(5)
    H, W = _rand_bits(rng, (64, 32)), _rand_bits(rng, (500, 32), 0.5)
    M = (rng.random((2, 32)) < 0.5).astype(np.uint8)
    out = o.oracle_rows(H, W, M)
    V = W.shape[0]
    conf, m, lse = out["conf"], out["m"], out["lse"]
    assert np.all(conf >= 1.0 / V * (1 - 1e-12)) and np.all(conf <= 1.0 + 1e-15)
    assert np.all(m <= lse + 1e-12) and np.all(lse <= m + math.log(V) + 1e-12)
    Z = o.bf16_bits_to_f64(H[out["row_idx"]]) @ o.bf16_bits_to_f64(W).T
    np.testing.assert_allclose(np.exp(Z - lse[:, None]).sum(axis=1), 1.0, rtol=1e-12)
    np.testing.assert_allclose(conf * np.exp(Z - m[:, None]).sum(axis=1), 1.0, rtol=1e-12)
    np.testing.assert_array_equal(m, Z.max(axis=1))


def check_mask_only_equals_full(o):
    rng = np.random.default_rng(9)
    for B, L, d, V in [(1, 40, 16, 70), (3, 9, 8, 33)]:
        H, W = _rand_bits(rng, (B * L, d)), _rand_bits(rng, (V, d))
        M = (rng.random((B, L)) < 0.5).astype(np.uint8)
        a = o.oracle_rows(H, W, M)
        b = o.full_then_gather(H, W, M)
        for key in ("tok", "m", "lse", "conf"):
            np.testing.assert_array_equal(a[key], b[key])


def check_merge_split_invariance(o):
    rng = np.random.default_rng(13)
    Z = rng.standard_normal((20, 257)) * 3
    Z[3, 10] = Z[3, 200] = Z[3].max() + 1.0        # an exact tie across splits
    tok0, m0, lse0, conf0 = o.row_stats(Z)
    V = Z.shape[1]
    for n_split in (1, 2, 3, 7, 64, 257):
        cuts = np.sort(rng.choice(np.arange(1, V), size=n_split - 1, replace=False))
        bounds = np.concatenate([[0], cuts, [V]])
        parts = [o.partial_stats(Z, int(a), int(b)) for a, b in zip(bounds[:-1], bounds[1:])]
        tok, m, lse, conf = o.lse_merge(parts)
        assert tok.tolist() == tok0.tolist()
        np.testing.assert_array_equal(m, m0)
        np.testing.assert_allclose(lse, lse0, rtol=1e-13)
        np.testing.assert_allclose(conf, conf0, rtol=1e-12)
    assert tok0[3] == 10


def check_policy_closed_forms(o):
    """Entropy / margin of softmax: uniform -> (ln V, 0); one logit c above V-1 zeros ->
    (ln S - c e^c / S, (e^c - 1) / S) with S = e^c + V - 1; V = 1 -> (0, 1)."""
    rng = np.random.default_rng(21)
    d, V = 8, 50
    w = _rand_bits(rng, (1, d))
    H = _rand_bits(rng, (3, d))
    out = o.oracle_rows(H, np.repeat(w, V, axis=0), np.ones((1, 3), np.uint8))
    np.testing.assert_allclose(out["entropy"], math.log(V), rtol=1e-13)
    np.testing.assert_allclose(out["margin"], 0.0, atol=1e-15)
    Wf = np.zeros((V, d), np.float32)
    Wf[:d, :d] = np.eye(d)
    for j, c in [(0, 3.0), (4, 0.5), (7, 9.0)]:
        Hf = np.zeros((1, d), np.float32)
        Hf[0, j] = c
        out = o.oracle_rows(_bits(Hf), _bits(Wf), np.ones((1, 1), np.uint8))
        S = math.exp(c) + V - 1
        np.testing.assert_allclose(out["entropy"], [math.log(S) - c * math.exp(c) / S], rtol=1e-12)
        np.testing.assert_allclose(out["margin"], [(math.exp(c) - 1) / S], rtol=1e-12)
    out = o.oracle_rows(_rand_bits(rng, (2, 8)), _rand_bits(rng, (1, 8)), np.ones((1, 2), np.uint8))
    np.testing.assert_allclose(out["entropy"], 0.0, atol=0)
    np.testing.assert_allclose(out["margin"], 1.0, atol=0)


def check_policy_library_and_brute(o):
    """Entropy against scipy.stats.entropy of the softmax, margin against a full sort, both
    against the pure-Python brute force."""
    import scipy.stats
    rng = np.random.default_rng(23)
    H, W = _rand_bits(rng, (12, 32)), _rand_bits(rng, (200, 32), 0.4)
    out = o.oracle_rows(H, W, np.ones((1, 12), np.uint8))
    Z = o.bf16_bits_to_f64(H) @ o.bf16_bits_to_f64(W).T
    P = scipy.special.softmax(Z, axis=1)
    np.testing.assert_allclose(out["entropy"], scipy.stats.entropy(P, axis=1), rtol=1e-12)
    Ps = np.sort(P, axis=1)
    np.testing.assert_allclose(out["margin"], Ps[:, -1] - Ps[:, -2], rtol=1e-12, atol=1e-15)
    Hl, Wl = _bf16_list(H), _bf16_list(W)
    for i in range(4):
        ent, mar = brute.policy_stats(brute.row_logits(Hl[i], Wl))
        np.testing.assert_allclose(out["entropy"][i], ent, rtol=1e-12)
        np.testing.assert_allclose(out["margin"][i], mar, rtol=1e-12, atol=1e-15)


def check_threshold_select(o):
    g = json.load(open(os.path.join(GOLDEN, "threshold_select.json")))
    M = np.array(g["M"], dtype=np.uint8)
    row_idx, seq_off, _ = o.mask_compact(M)
    for dt in (np.float32, np.float64):
        score = np.array(g["score"], dtype=dt)
        for c in g["cases"]:
            lo = np.array([c["lo"]]) if "lo" in c else None
            hi = np.array([c["hi"]]) if "hi" in c else None
            idx, n_sel = o.select_unmask_threshold(score, row_idx, seq_off, g["L"], c["k"],
                                                   c["threshold"], c["min_sel"], lo, hi)
            assert idx[0].tolist() == c["idx"], (c, idx)
            assert int(n_sel[0]) == c["n_sel"]
    # brute force on random inputs; -inf threshold is plain top-k
    rng = np.random.default_rng(29)
    for _ in range(20):
        B, L = int(rng.integers(1, 4)), int(rng.integers(1, 30))
        M = (rng.random((B, L)) < 0.7).astype(np.uint8)
        row_idx, seq_off, count = o.mask_compact(M)
        score = (rng.integers(0, 8, size=count) / 8.0).astype(np.float64)
        k = int(rng.integers(1, 8))
        tau = float(rng.choice([-np.inf, 0.25, 0.5, 0.875, 2.0]))
        ms = int(rng.integers(0, 3))
        idx, n_sel = o.select_unmask_threshold(score, row_idx, seq_off, L, k, tau, ms)
        for b in range(B):
            cands = [(score[r], int(row_idx[r]) - b * L) for r in range(seq_off[b], seq_off[b + 1])]
            ref = brute.select_threshold(cands, k, tau, ms)
            assert idx[b, :n_sel[b]].tolist() == ref and int(n_sel[b]) == len(ref)
        if tau == -np.inf:
            t_idx, t_n = o.select_unmask(score, row_idx, seq_off, L, k)
            assert np.array_equal(t_idx, idx) and np.array_equal(t_n, n_sel)


def check_block_step(o):
    """Current-block-only logits: the windowed mask equals brute-force windowed compaction
    (including empty, inverted and out-of-range windows), and the block step selects exactly
    what the full step selects with the same windows, with per-row statistics equal to the
    full step's rows at the same positions."""
    rng = np.random.default_rng(21)
    for case in range(10):
        B, L = int(rng.integers(1, 4)), int(rng.integers(1, 40))
        M = (rng.random((B, L)) < 0.6).astype(np.uint8)
        lo = rng.integers(-3, L + 2, size=B)
        hi = lo + rng.integers(-2, L + 3, size=B)
        if case == 0:                                          # window edges on masked cells
            M[:] = 1
            lo[:] = 1
            hi[:] = max(2, L - 1)
        Mw = o.window_mask(M, lo, hi)
        r1, s1, c1 = o.mask_compact(Mw)
        r2, s2 = brute.compact_window(M.tolist(), lo.tolist(), hi.tolist())
        assert r1.tolist() == r2 and s1.tolist() == s2 and c1 == len(r2), (M, lo, hi)
        d, V, k = int(rng.integers(1, 6)), int(rng.integers(1, 20)), int(rng.integers(1, 5))
        H, W = _rand_bits(rng, (B * L, d)), _rand_bits(rng, (V, d), 0.5)
        blk = o.oracle_block_step(H, W, M, k, lo, hi)
        full = o.oracle_step(H, W, M, k, lo, hi)
        assert np.array_equal(blk["idx"], full["idx"]) and np.array_equal(blk["n_sel"], full["n_sel"])
        where = {int(p): i for i, p in enumerate(full["row_idx"])}
        sel = [where[int(p)] for p in blk["row_idx"]]
        for key in ("tok", "m", "lse", "conf"):
            assert np.array_equal(blk[key], np.asarray(full[key])[sel]), key


def check_top2_gap(o):
    """The near-tie exemption of the parity tests rests on top2_gap: pinned against a sorted
    brute force, exactly 0 on a repeated maximum, infinite when a row has one logit."""
    rng = np.random.default_rng(17)
    for V in (1, 2, 3, 9, 64):
        Z = rng.standard_normal((6, V)) * 2.0
        if V >= 2:
            Z[1, 0] = Z[1, V - 1] = Z[1].max() + 1.0  # the maximum twice: gap exactly 0
            Z[2, :] = 0.5                            # every entry tied
        if V >= 3:
            top = Z[3].max() + 1.0
            Z[3, 0] = top                            # unique maximum ...
            Z[3, 1] = Z[3, 2] = top - 0.25           # ... over a repeated second: gap 0.25
        got = o.top2_gap(Z)
        want = [brute.top2_gap(row) for row in Z.tolist()]
        assert got.shape == (Z.shape[0],)
        assert got.tolist() == want, (V, got, want)
        if V == 1:
            assert np.all(np.isinf(got))
        else:
            assert got[1] == 0.0 and got[2] == 0.0
        if V >= 3:
            assert got[3] == 0.25


def _onehot_case(V, d, targets, rng):
    """Rows of H that are unit vectors e_r, so that row r's logits are column r of W; W's
    column r gets its maximum at vocabulary entry targets[r].  Further rows are random."""
    n_hot = len(targets)
    H = np.zeros((n_hot + 3, d), np.float32)
    H[:n_hot, :n_hot] = np.eye(n_hot)
    H[n_hot:] = rng.standard_normal((3, d))
    W = (rng.standard_normal((V, d)) * 0.25).astype(np.float32)
    for r, t in enumerate(targets):
        W[:, r] = np.clip(W[:, r], -1.0, 1.0)
        W[t, r] = 4.0
    return _bits(torch.tensor(H).bfloat16().float().numpy()), \
        _bits(torch.tensor(W).bfloat16().float().numpy())


def check_chunked_rows(o):
    """rows_stats_chunked, the path of every full-vocabulary parity check, against the brute
    force per row, with the maximum planted on the last and first columns of chunks: small
    chunks (1, 5, 7) on V = 33 and the default chunk at V = 8193 and V = 16385."""
    rng = np.random.default_rng(19)
    cases = [(33, 1, [0, 32, 16]), (33, 5, [4, 5, 32, 29]), (33, 7, [6, 13, 7, 32]),
             (33, 64, [32, 0]),
             (8193, o.V_CHUNK, [8191, 8192, 0]), (16385, o.V_CHUNK, [8191, 8192, 16383, 16384])]
    for V, chunk, targets in cases:
        d = 8
        Hb, Wb = _onehot_case(V, d, targets, rng)
        tok, m, lse, conf, gap = o.rows_stats_chunked(Hb, Wb, chunk=chunk)
        Hl, Wl = _bf16_list(Hb), _bf16_list(Wb)
        for r in range(Hb.shape[0]):
            z = brute.row_logits(Hl[r], Wl)
            t, mm, ll, cc = brute.stats(z)
            assert int(tok[r]) == t, (V, chunk, r, int(tok[r]), t)
            if r < len(targets):
                assert t == targets[r]
            np.testing.assert_allclose(m[r], mm, rtol=1e-13)
            np.testing.assert_allclose(lse[r], ll, rtol=1e-12)
            np.testing.assert_allclose(conf[r], cc, rtol=1e-12)
            np.testing.assert_allclose(gap[r], brute.top2_gap(z), rtol=1e-12, atol=1e-12 * abs(mm))
        # the same rows unchunked: one matmul over the whole vocabulary
        Z = o.logits_rows(o.bf16_bits_to_f64(Hb), o.bf16_bits_to_f64(Wb))
        t2, m2, l2, c2 = o.row_stats(Z)
        assert tok.tolist() == t2.tolist()
        np.testing.assert_allclose(lse, l2, rtol=1e-13)
        np.testing.assert_allclose(conf, c2, rtol=1e-13)


ALL_CHECKS = [check_handworked, check_topk_ties, check_compact, check_brute_random,
              check_closed_forms, check_library_routines, check_invariants,
              check_mask_only_equals_full, check_merge_split_invariance,
              check_policy_closed_forms, check_policy_library_and_brute, check_threshold_select,
              check_block_step, check_top2_gap, check_chunked_rows]
