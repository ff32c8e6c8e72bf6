"""Pins of the fp64 oracle against what the HiLS pages and mathematics fix.

None of these tests re-types the oracle's own formulas: each checks a
consequence (an identity, a special case, a bound, a brute-force search or a
printed worked example) that a plausible mistake in the oracle would break.
"""
import itertools
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp

from oracle.oracle import Oracle, Rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(rng, *shape):
    return rng.standard_normal(shape).astype(np.float32)


def dense_causal(Q, K, V, G):
    """Brute-force dense causal softmax attention, fp64 (textbook definition)."""
    B, Hq, N, d = Q.shape
    out = np.zeros((B, Hq, N, d))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            s = (Q[b, hq].astype(np.float64) @ K[b, h].astype(np.float64).T) / math.sqrt(d)
            s[np.triu_indices(N, 1)] = -np.inf
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            out[b, hq] = p @ V[b, h].astype(np.float64)
    return out


def test_pin_landmark_query_gives_exact_chunk_lse():
    """Pin (1): a query equal to the chunk's landmark query scores exactly the
    log-sum-exp of its logits over the chunk (Taylor surrogate exact at q = lq)."""
    rng = np.random.default_rng(11)
    for d, G in ((64, 1), (128, 2), (16, 4)):
        B, Hkv, N, C = 2, 2, 256, 64
        Hq = Hkv * G
        K = rand(rng, B, Hkv, N, d)
        LQ = rand(rng, B, Hkv, N // C, d) * 1.7
        o = Oracle(B, Hq, Hkv, N, d, C, 3)
        kp, bp = o.summary(K, LQ)
        rb, rhq, rpos, qs, want = [], [], [], [], []
        for b in range(B):
            for hq in range(Hq):
                h = hq // G
                for c in range(3):
                    rb.append(b); rhq.append(hq); rpos.append(N - 1); qs.append(LQ[b, h, c])
                    logits = K[b, h, c * C:(c + 1) * C].astype(np.float64) @ LQ[b, h, c].astype(np.float64)
                    want.append((c, logsumexp(logits / math.sqrt(d))))
        S = o.scores(kp, bp, Rows(rb, rhq, rpos, np.stack(qs)))
        for r, (c, lse) in enumerate(want):
            assert abs(S[r, c] - lse) < 1e-12 * max(1.0, abs(lse))


def test_pin_worked_example():
    """Pin (2): the pages' worked example, read from tests/golden."""
    vals = {}
    with open(os.path.join(GOLDEN, "worked_example.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                vals[k] = float(v)
    d = int(vals["head_dim"])
    rng = np.random.default_rng(3)
    q = rand(rng, d)
    v = rng.standard_normal(d)
    kp_vec = v * (vals["scaled_dot"] * math.sqrt(d) / float(np.dot(q.astype(np.float64), v)))
    N, C = 128, 64
    o = Oracle(1, 1, 1, N, d, C, 1)
    kp = np.zeros((1, 1, 2, d)); kp[0, 0, 0] = kp_vec
    bp = np.zeros((1, 1, 2)); bp[0, 0, 0] = vals["entropy_bias"]
    S = o.scores(kp, bp, Rows([0], [0], [N - 1], q[None]))
    assert abs(S[0, 0] - vals["score"]) < 1e-12
    assert round(math.exp(S[0, 0]), 1) == vals["exp_score_1dp"]
    assert S[0, 1] == -np.inf          # the own chunk is not a candidate


@pytest.mark.parametrize("B,Hq,Hkv,d", [(1, 1, 1, 16), (2, 4, 2, 16), (1, 3, 1, 8)])
def test_pin_dense_equivalence(B, Hq, Hkv, d):
    """Pin (3): with every past chunk kept and exact chunk log-sum-exps in
    place of the surrogate, the hierarchical output equals dense causal
    attention (hierarchical factorisation of the softmax)."""
    rng = np.random.default_rng(5 + d + Hq)
    N, C = 512, 64
    nc = N // C
    G = Hq // Hkv
    Q, K, V = rand(rng, B, Hq, N, d), rand(rng, B, Hkv, N, d), rand(rng, B, Hkv, N, d)
    LQ = rand(rng, B, Hkv, nc, d)
    o = Oracle(B, Hq, Hkv, N, d, C, nc)
    kp, bp = o.summary(K, LQ)
    flat = np.arange(B * Hq * N)
    rows = Rows.from_prefill(Q, flat)
    ids = np.full((len(rows), nc), -1, np.int32)
    for r in range(len(rows)):
        own = rows.pos[r] // C
        ids[r, :own] = np.arange(own)
    O, _ = o.attend(K, V, kp, bp, rows, ids, score_mode=1)
    ref = dense_causal(Q, K, V, G).reshape(-1, d)
    assert np.max(np.abs(O - ref)) < 1e-12
    # the surrogate scores give a different (approximate) answer
    O2, _ = o.attend(K, V, kp, bp, rows, ids, score_mode=0)
    assert np.max(np.abs(O2 - ref)) > 1e-6


def test_pin_surrogate_fusion_exact_when_query_is_every_landmark():
    """Pins (1) and (3) together on the surrogate path: if every chunk's
    landmark query equals the row's query, every surrogate score is that
    chunk's exact log-sum-exp, so keeping all past chunks reproduces dense
    causal attention with the surrogate-weighted fusion."""
    rng = np.random.default_rng(15)
    B, H, N, d, C = 1, 1, 512, 16, 64
    nc = N // C
    Q, K, V = rand(rng, B, H, N, d), rand(rng, B, H, N, d), rand(rng, B, H, N, d)
    ref = dense_causal(Q, K, V, 1)
    o = Oracle(B, H, H, N, d, C, nc)
    for i in (70, 200, 321, 511):
        LQ = np.broadcast_to(Q[:, :, i:i + 1, :], (B, H, nc, d)).copy()
        kp, bp = o.summary(K, LQ)
        rows = Rows([0], [0], [i], Q[0, 0, i][None])
        ids = np.full((1, nc), -1, np.int32)
        ids[0, :i // C] = np.arange(i // C)
        O, _ = o.attend(K, V, kp, bp, rows, ids, score_mode=0)
        assert np.max(np.abs(O[0] - ref[0, 0, i])) < 1e-12


def test_zero_landmark_is_mean_pooling():
    """lq = 0 gives a uniform intra-chunk distribution: k' is the mean key
    (the mean-pooling summary of earlier sparse methods) and b' = log C."""
    rng = np.random.default_rng(1)
    B, H, N, d, C = 1, 2, 256, 32, 64
    K = rand(rng, B, H, N, d)
    kp, bp = Oracle(B, H, H, N, d, C, 1).summary(K, np.zeros((B, H, N // C, d), np.float32))
    mean = K.astype(np.float64).reshape(B, H, N // C, C, d).mean(axis=3)
    assert np.max(np.abs(kp - mean)) < 1e-12
    assert np.max(np.abs(bp - math.log(C))) < 1e-12


def test_equal_keys():
    """A chunk whose keys are all equal summarises to that key, with b' = log C."""
    rng = np.random.default_rng(2)
    B, H, N, d, C = 1, 1, 128, 16, 64
    K = np.repeat(rand(rng, B, H, N // C, 1, d), C, axis=3).reshape(B, H, N, d)
    kp, bp = Oracle(B, H, H, N, d, C, 1).summary(K, rand(rng, B, H, N // C, d) * 3)
    assert np.max(np.abs(kp - K[:, :, ::C, :])) < 1e-12
    assert np.max(np.abs(bp - math.log(C))) < 1e-12


def test_entropy_bounds_and_convex_hull():
    rng = np.random.default_rng(3)
    B, H, N, d, C = 2, 3, 1024, 64, 64
    K = rand(rng, B, H, N, d)
    LQ = rand(rng, B, H, N // C, d) * 4.0          # sharp distributions too
    kp, bp = Oracle(B, H, H, N, d, C, 1).summary(K, LQ)
    assert bp.min() >= -1e-12 and bp.max() <= math.log(C) + 1e-12
    Kc = K.reshape(B, H, N // C, C, d)
    assert np.all(kp <= Kc.max(axis=3) + 1e-12) and np.all(kp >= Kc.min(axis=3) - 1e-12)


def test_entropy_equals_definition():
    """b' is the Shannon entropy -sum p log p of the landmark's distribution
    (the oracle evaluates it through a log-sum-exp rewrite)."""
    rng = np.random.default_rng(4)
    B, H, N, d, C = 1, 1, 256, 64, 64
    K, LQ = rand(rng, B, H, N, d), rand(rng, B, H, N // C, d) * 2
    kp, bp = Oracle(B, H, H, N, d, C, 1).summary(K, LQ)
    for c in range(N // C):
        z = K[0, 0, c * C:(c + 1) * C].astype(np.float64) @ LQ[0, 0, c].astype(np.float64) / math.sqrt(d)
        p = np.exp(z - logsumexp(z))
        assert abs(bp[0, 0, c] - float(-(p * np.log(p)).sum())) < 1e-12


def test_needle_shift_invariance():
    """Shifting every key of a chunk by v leaves the landmark distribution and
    b' unchanged and moves k' by exactly v."""
    rng = np.random.default_rng(6)
    B, H, N, d, C = 1, 2, 512, 64, 64
    # values on a 2^-10 grid so that the fp32 shift below is exact
    K = np.round(rand(rng, B, H, N, d) * 1024) / 1024
    LQ = rand(rng, B, H, N // C, d)
    o = Oracle(B, H, H, N, d, C, 1)
    kp0, bp0 = o.summary(K, LQ)
    v = (np.round(rand(rng, d) * 1.5 * 1024) / 1024).astype(np.float32)
    K2 = K.copy()
    K2[0, 1, 3 * C:4 * C] += v
    assert np.array_equal(K2[0, 1, 3 * C:4 * C] - K[0, 1, 3 * C:4 * C], np.broadcast_to(v, (C, d)))
    kp1, bp1 = o.summary(K2, LQ)
    assert np.max(np.abs(bp1 - bp0)) < 1e-12
    assert np.max(np.abs(kp1[0, 1, 3] - kp0[0, 1, 3] - v)) < 1e-12
    mask = np.ones(kp0.shape[:3], bool); mask[0, 1, 3] = False
    assert np.array_equal(kp0[mask], kp1[mask])


def test_surrogate_is_a_lower_bound_of_chunk_lse():
    """LSE is convex, so its tangent plane at lq never exceeds it:
    s^_{i,c} <= log sum_j exp(q_i.k_j/sqrt(d)) for every query."""
    rng = np.random.default_rng(7)
    B, H, N, d, C = 1, 2, 1024, 64, 64
    K, LQ = rand(rng, B, H, N, d), rand(rng, B, H, N // C, d)
    o = Oracle(B, H, H, N, d, C, 4)
    kp, bp = o.summary(K, LQ)
    Q = rand(rng, B, H, N, d)
    rows = Rows.from_prefill(Q, np.arange(B * H * N)[::7])
    S = o.scores(kp, bp, rows)
    for r in range(len(rows)):
        h = rows.hq[r]
        for c in range(rows.pos[r] // C):
            lse = logsumexp(K[0, h, c * C:(c + 1) * C].astype(np.float64) @ rows.q[r].astype(np.float64)
                            / math.sqrt(d))
            assert S[r, c] <= lse + 1e-12


def _brute_topk(scores, K):
    """The K-subset with the largest score sum; ties -> lexicographically
    smallest id tuple (equivalent to 'lower id wins')."""
    n = len(scores)
    if n <= K:
        return list(range(n))
    best, best_ids = -np.inf, None
    for sub in itertools.combinations(range(n), K):
        s = sum(scores[i] for i in sub)
        if s > best + 1e-15:
            best, best_ids = s, list(sub)
    return best_ids


def test_selection_brute_force_with_ties():
    rng = np.random.default_rng(8)
    B, H, N, d, C, K = 1, 2, 640, 16, 64, 3
    nc = N // C
    Kt, LQ = rand(rng, B, H, N, d), rand(rng, B, H, nc, d)
    # plant exact ties: chunks 2 and 5 (and 1 and 7 of head 1) identical
    Kt[0, 0, 5 * C:6 * C] = Kt[0, 0, 2 * C:3 * C]; LQ[0, 0, 5] = LQ[0, 0, 2]
    Kt[0, 1, 7 * C:8 * C] = Kt[0, 1, 1 * C:2 * C]; LQ[0, 1, 7] = LQ[0, 1, 1]
    o = Oracle(B, H, H, N, d, C, K)
    kp, bp = o.summary(Kt, LQ)
    Q = rand(rng, B, H, N, d)
    rows = Rows.from_prefill(Q, np.arange(B * H * N)[::5])
    S = o.scores(kp, bp, rows)
    ids, sel, gap = o.select(kp, bp, rows)
    n_tie_rows = 0
    for r in range(len(rows)):
        own = rows.pos[r] // C
        want = _brute_topk(list(S[r, :own]), K)
        got = [int(c) for c in ids[r] if c >= 0]
        assert got == sorted(want)
        assert list(ids[r, len(got):]) == [-1] * (K - len(got))
        assert np.allclose(sel[r, :len(got)], S[r, got], rtol=0, atol=0)
        assert (gap[r] == np.inf) == (own <= K)
        if own > K:
            assert gap[r] >= 0
            srt = np.sort(S[r, :own])[::-1]
            n_tie_rows += srt[K - 1] == srt[K]
    # the planted copies tie at the K-th / (K+1)-th boundary on some rows, so
    # the brute force above really decided ties there (20 of 256 rows here)
    assert n_tie_rows > 0


def test_selection_ties_go_to_lower_ids():
    """Reading of the selection rule: among equal scores the lower chunk ids
    are kept.  With every chunk a copy of chunk 0 (keys and landmark query),
    all surrogate scores of a row are exactly equal, so every row with more
    than K candidates keeps chunks 0 .. K-1 and its K-th/(K+1)-th gap is 0."""
    rng = np.random.default_rng(21)
    B, H, N, d, C, K = 1, 1, 640, 16, 64, 3
    nc = N // C
    Kt = np.tile(rand(rng, 1, 1, C, d), (1, 1, nc, 1))
    LQ = np.tile(rand(rng, 1, 1, 1, d), (1, 1, nc, 1))
    o = Oracle(B, H, H, N, d, C, K)
    kp, bp = o.summary(Kt, LQ)
    Q = rand(rng, B, H, N, d)
    rows = Rows.from_prefill(Q, np.arange(C * (K + 1), N, 7))
    S = o.scores(kp, bp, rows)
    ids, _, gap = o.select(kp, bp, rows)
    for r in range(len(rows)):
        own = rows.pos[r] // C
        assert np.all(S[r, :own] == S[r, 0])
        assert list(ids[r]) == list(range(K))
        assert gap[r] == 0


def test_rows_in_first_chunk_are_plain_causal_attention():
    """A query in chunk 0 has no candidate chunk: its output is causal softmax
    attention over keys 0..i; row 0 returns v_0."""
    rng = np.random.default_rng(9)
    B, H, N, d, C = 1, 1, 256, 32, 64
    Q, K, V, LQ = rand(rng, B, H, N, d), rand(rng, B, H, N, d), rand(rng, B, H, N, d), rand(rng, B, H, N // C, d)
    o = Oracle(B, H, H, N, d, C, 3)
    kp, bp = o.summary(K, LQ)
    res = o.prefill_rows(Q, K, V, kp, bp, np.arange(C))
    ref = dense_causal(Q, K, V, 1)[0, 0, :C]
    assert np.max(np.abs(res["O"] - ref)) < 1e-12
    assert np.max(np.abs(res["O"][0] - V[0, 0, 0])) < 1e-15
    assert np.all(res["ids"] == -1)


def test_fewer_candidates_than_k():
    rng = np.random.default_rng(10)
    B, H, N, d, C, K = 1, 1, 256, 16, 64, 3
    Q, K_, LQ = rand(rng, B, H, N, d), rand(rng, B, H, N, d), rand(rng, B, H, N // C, d)
    o = Oracle(B, H, H, N, d, C, K)
    kp, bp = o.summary(K_, LQ)
    ids, _, gap = o.select(kp, bp, Rows.from_prefill(Q, np.array([70, 130, 250])))
    assert list(ids[0]) == [0, -1, -1]
    assert list(ids[1]) == [0, 1, -1]
    assert list(ids[2]) == [0, 1, 2]
    assert np.all(np.isinf(gap))


def test_identical_query_heads_give_identical_outputs():
    rng = np.random.default_rng(12)
    B, Hq, Hkv, N, d, C, K = 1, 4, 1, 512, 16, 64, 3
    q1 = rand(rng, B, 1, N, d)
    Q = np.repeat(q1, Hq, axis=1)
    Kt, V, LQ = rand(rng, B, Hkv, N, d), rand(rng, B, Hkv, N, d), rand(rng, B, Hkv, N // C, d)
    o = Oracle(B, Hq, Hkv, N, d, C, K)
    kp, bp = o.summary(Kt, LQ)
    res = o.prefill_rows(Q, Kt, V, kp, bp, np.arange(B * Hq * N))
    O = res["O"].reshape(Hq, N, d)
    for g in range(1, Hq):
        assert np.array_equal(O[g], O[0])


def test_decode_equals_last_prefill_row():
    from chunk_wise_sparse_b200.inputs import custom, generate
    w = custom(B=2, Hq=4, Hkv=2, d=32, N=1024, K=3, seed=21, dtype="bf16", needles=2,
               needle_mode="random", kind="prefill+decode")
    inp = generate(w)
    o = Oracle.for_workload(w)
    kp, bp = o.summary(inp.k_f32, inp.lq_f32)
    dec = o.decode(inp.decode_query(), inp.k_f32, inp.v_f32, kp, bp, inp.seqlens)
    B, Hq, N = w.B, w.Hq, w.N
    flat = np.array([(b * Hq + h) * N + N - 1 for b in range(B) for h in range(Hq)])
    pre = o.prefill_rows(inp.q_f32, inp.k_f32, inp.v_f32, kp, bp, flat)
    assert np.array_equal(dec["O"].reshape(-1, w.d), pre["O"])
    assert np.array_equal(dec["ids"].reshape(-1, w.K), pre["ids"])


def test_partial_summary_range():
    """Summarising a chunk range touches only those chunks (decode appends)."""
    rng = np.random.default_rng(13)
    B, H, N, d, C = 1, 1, 512, 16, 64
    K, LQ = rand(rng, B, H, N, d), rand(rng, B, H, N // C, d)
    o = Oracle(B, H, H, N, d, C, 1)
    kp, bp = o.summary(K, LQ)
    kp2, bp2 = o.summary(K, LQ, 3, 5)
    assert np.array_equal(kp2[:, :, 3:5], kp[:, :, 3:5]) and np.array_equal(bp2[:, :, 3:5], bp[:, :, 3:5])
    assert not kp2[:, :, :3].any() and not kp2[:, :, 5:].any()


@pytest.mark.parametrize("W", [64, 128, 320, 512])
def test_pin_window_plus_all_exact_chunks_is_dense_attention(W):
    """Local window (aitrends.kr article, section "기술 상세": sliding window
    512; read as chunk-aligned, the own chunk and the W/C - 1 chunks before it,
    one fusion branch scored by its exact log-sum-exp).  Keeping every
    candidate (the chunks before the window) with exact chunk log-sum-exps
    must reproduce dense causal attention for any W: window and candidates
    cover every past key exactly once."""
    rng = np.random.default_rng(31 + W)
    B, Hq, Hkv, N, d, C = 1, 2, 1, 768, 16, 64
    nc = N // C
    Q, K, V = rand(rng, B, Hq, N, d), rand(rng, B, Hkv, N, d), rand(rng, B, Hkv, N, d)
    LQ = rand(rng, B, Hkv, nc, d)
    o = Oracle(B, Hq, Hkv, N, d, C, nc, W)
    kp, bp = o.summary(K, LQ)
    rows = Rows.from_prefill(Q, np.arange(B * Hq * N))
    ids, _, _ = o.select(kp, bp, rows)
    wc = W // C
    for r in range(len(rows)):
        # candidates: the chunks before the window, all kept (K = nc)
        n_cand = max(0, rows.pos[r] // C - (wc - 1))
        assert np.array_equal(ids[r, :n_cand], np.arange(n_cand))
        assert np.all(ids[r, n_cand:] == -1)
    O, lse_w = o.attend(K, V, kp, bp, rows, ids, score_mode=1)
    assert np.max(np.abs(O - dense_causal(Q, K, V, Hq // Hkv).reshape(-1, d))) < 1e-12
    # the window branch's score is the exact log-sum-exp over its keys
    for r in (0, 100, 700, 767 + 768):
        i, h = rows.pos[r], rows.hq[r] // (Hq // Hkv)
        w0 = max(0, (i // C - (wc - 1)) * C)
        s = (K[0, h, w0:i + 1].astype(np.float64) @ Q[0, rows.hq[r], i].astype(np.float64)) / math.sqrt(d)
        assert abs(lse_w[r] - logsumexp(s)) < 1e-12


def test_pin_window_over_the_whole_sequence_is_dense_attention():
    """A window that covers every past key leaves no candidates: the output is
    dense causal attention whatever the summaries and K."""
    rng = np.random.default_rng(37)
    B, H, N, d, C = 1, 1, 512, 16, 64
    Q, K, V = rand(rng, B, H, N, d), rand(rng, B, H, N, d), rand(rng, B, H, N, d)
    LQ = rand(rng, B, H, N // C, d)
    o = Oracle(B, H, H, N, d, C, 3, N)
    kp, bp = o.summary(K, LQ)
    rows = Rows.from_prefill(Q, np.arange(N))
    ids, _, _ = o.select(kp, bp, rows)
    assert np.all(ids == -1)
    O, _ = o.attend(K, V, kp, bp, rows, ids, score_mode=0)
    assert np.max(np.abs(O - dense_causal(Q, K, V, 1).reshape(-1, d))) < 1e-12


# ---------------------------------------------------------------- Q-Cal
# aitrends.kr article, section "방법론" and glossary entry "저계수 쿼리 보정":
# a low-rank down/up projection of the query gives the calibrated query that
# scores the chunks.

def test_pin_qcal_hand_built_projection():
    """W_down picks q0 and 2 q2, W_up sends them to dims 1 and 4 with factors
    3 and -1: q^ = q + (0, 3 q0, 0, 0, -2 q2, 0), worked out by hand."""
    from oracle.oracle import qcal
    wd = np.zeros((1, 2, 6), np.float32)
    wd[0, 0, 0], wd[0, 1, 2] = 1.0, 2.0
    wu = np.zeros((1, 6, 2), np.float32)
    wu[0, 1, 0], wu[0, 4, 1] = 3.0, -1.0
    q = np.array([[0.5, -1.0, 2.0, 0.25, 4.0, -3.0], [1.0, 1.0, -1.5, 0.0, 0.5, 2.0]], np.float32)
    out = qcal(q, np.zeros(2, np.int32), wd, wu)
    want = q.astype(np.float64).copy()
    want[:, 1] += 3.0 * want[:, 0]
    want[:, 4] += -2.0 * q[:, 2]
    assert np.array_equal(out, want)


def test_pin_qcal_orthogonal_projection_per_head():
    """With orthonormal rows U_h^T as W_down and -U_h as W_up, q^ is q with its
    component in span(U_h) removed: U_h^T q^ = 0, and calibrating q^ again
    changes nothing (a projection is idempotent).  Heads use their own U_h."""
    from oracle.oracle import qcal
    rng = np.random.default_rng(23)
    Hq, d, r, n = 3, 16, 4, 40
    U = np.stack([np.linalg.qr(rng.standard_normal((d, r)))[0] for _ in range(Hq)])   # [Hq, d, r]
    wd = np.ascontiguousarray(U.transpose(0, 2, 1)).astype(np.float32)
    wu = (-U).astype(np.float32)
    hq = rng.integers(0, Hq, n).astype(np.int32)
    q = rand(rng, n, d)
    out = qcal(q, hq, wd, wu)
    Uf = U.astype(np.float32).astype(np.float64)
    for i in range(n):
        assert np.max(np.abs(Uf[hq[i]].T @ out[i])) < 1e-6
    assert np.max(np.abs(out - q)) > 0.1
    again = qcal(out.astype(np.float32), hq, wd, wu)
    assert np.max(np.abs(again - out)) < 1e-5


def test_pin_scoring_query_steers_only_the_fusion():
    """A scoring query pushed far along k'_c makes chunk c's fusion weight 1,
    so O is chunk c's own softmax attention computed with the attending query
    q (a textbook softmax over 64 keys), not with the scoring query."""
    rng = np.random.default_rng(29)
    B, Hq, Hkv, N, d, C = 1, 2, 1, 512, 32, 64
    K, V = rand(rng, B, Hkv, N, d), rand(rng, B, Hkv, N, d)
    LQ = rand(rng, B, Hkv, N // C, d)
    o = Oracle(B, Hq, Hkv, N, d, C, 1)
    kp, bp = o.summary(K, LQ)
    c, pos = 3, 7 * C + 20
    q = rand(rng, 2, d)
    qs = q + 400.0 * (kp[0, 0, c] / np.linalg.norm(kp[0, 0, c])).astype(np.float32)
    rows = Rows([0, 0], [0, 1], [pos, pos], q)
    ids = np.array([[c], [c]], np.int32)
    O, _ = o.attend(K, V, kp, bp, rows, ids, qscore=qs)
    keys = K[0, 0, c * C:(c + 1) * C].astype(np.float64)
    for r in range(2):
        s = keys @ q[r].astype(np.float64) / math.sqrt(d)
        p = np.exp(s - s.max())
        want = (p / p.sum()) @ V[0, 0, c * C:(c + 1) * C].astype(np.float64)
        assert np.max(np.abs(O[r] - want)) < 1e-9
    # the same rows without the scoring query mix in the own chunk
    O2, _ = o.attend(K, V, kp, bp, rows, ids)
    assert np.max(np.abs(O2 - O)) > 1e-3
