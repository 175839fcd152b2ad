"""Pins for the fp64 oracle against facts the paper and the mathematics fix (no GPU).

Paper: "Hierarchical Sparse Attention Done Right: Toward Infinite Context Modeling" (arXiv 2607.02980).
Each test names the definition it pins and the mistake it would catch.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from oracle import Geometry

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))


def rng(seed=0):
    return np.random.default_rng(seed)


def rand_problem(g: Geometry, seed=0, scale=1.0):
    r = rng(seed)
    return dict(
        q=r.standard_normal((g.B, g.Hq, g.T, g.d)) * scale,
        k=r.standard_normal((g.B, g.Hkv, g.L, g.d)) * scale,
        v=r.standard_normal((g.B, g.Hkv, g.L, g.d)),
        q_land=r.standard_normal((g.B, g.Hq, g.Nc, g.d)),
        q_hat=r.standard_normal((g.B, g.Hq, g.T, g.d)) * scale,
    )


# ---------------------------------------------------------------- Eq. 8 summaries

def test_summary_golden_two_tokens():
    """Eq. 8 on a hand-derived two-token chunk (catches a wrong sign on b', missing scale, wrong p)."""
    e = GOLDEN["summary_two_tokens"]
    g = Geometry(B=1, T=1, L=2, Hq=1, Hkv=1, d=2, S=2, topk=1, W=1)
    k = np.array(e["keys"])[None, None]
    ql = np.array(e["q_land"])[None, None, None]
    ks, bs = oracle.chunk_summary(g, k, ql)
    np.testing.assert_allclose(ks[0, 0, 0], e["k_sum"], rtol=0, atol=1e-15)
    assert abs(bs[0, 0, 0] - e["b_sum"]) < 1e-15


def test_summary_S1_is_identity():
    """Eq. 8 with S = 1: k'_c = k_c and b'_c = 0 exactly."""
    g = Geometry(B=2, T=1, L=9, Hq=4, Hkv=2, d=8, S=1, topk=1, W=1)
    x = rand_problem(g)
    ks, bs = oracle.chunk_summary(g, x["k"], x["q_land"])
    kk = np.repeat(x["k"], g.G, axis=1)  # head h reads KV head h // G
    np.testing.assert_array_equal(ks, kk)
    np.testing.assert_array_equal(bs, 0.0)


def test_summary_uniform_logits():
    """Eq. 8 with q' = 0: p is uniform, so k' is the mean key and b' = log S (the entropy maximum)."""
    g = Geometry(B=1, T=1, L=48, Hq=2, Hkv=1, d=8, S=16, topk=1, W=1)
    x = rand_problem(g)
    ks, bs = oracle.chunk_summary(g, x["k"], np.zeros_like(x["q_land"]))
    mean = x["k"][0, 0].reshape(3, 16, 8).mean(axis=1)
    np.testing.assert_allclose(ks[0, 0], mean, atol=1e-14)
    np.testing.assert_allclose(bs, math.log(16), atol=1e-14)


def test_summary_entropy_bounds_and_dominant_token():
    """b' is an entropy: 0 <= b' <= log S; a dominant logit drives b' -> 0 and k' -> that key."""
    g = Geometry(B=1, T=1, L=64, Hq=1, Hkv=1, d=16, S=16, topk=1, W=1)
    x = rand_problem(g, seed=3)
    ks, bs = oracle.chunk_summary(g, x["k"], x["q_land"])
    assert np.all(bs >= 0) and np.all(bs <= math.log(16) + 1e-12)
    kk = x["k"].copy()
    ql = x["q_land"].copy()
    kk[0, 0, 5] = 0
    kk[0, 0, 5, 0] = 40.0  # token 5 of chunk 0 aligned with q'
    ql[0, 0, 0] = 0
    ql[0, 0, 0, 0] = 40.0
    ks, bs = oracle.chunk_summary(g, kk, ql)
    assert bs[0, 0, 0] < 1e-12
    np.testing.assert_allclose(ks[0, 0, 0], kk[0, 0, 5], atol=1e-12)


def test_summary_head_mapping_gqa():
    """Query head h summarises KV head h // G (catches h % Hkv)."""
    g = Geometry(B=1, T=1, L=32, Hq=4, Hkv=2, d=8, S=8, topk=1, W=1)
    x = rand_problem(g, seed=5)
    ks, bs = oracle.chunk_summary(g, x["k"], x["q_land"])
    for h in range(4):
        g1 = Geometry(B=1, T=1, L=32, Hq=1, Hkv=1, d=8, S=8, topk=1, W=1)
        k1, b1 = oracle.chunk_summary(g1, x["k"][:, h // 2:h // 2 + 1], x["q_land"][:, h:h + 1])
        np.testing.assert_array_equal(ks[:, h:h + 1], k1)
        np.testing.assert_array_equal(bs[:, h:h + 1], b1)


def test_summary_chunk_range():
    """Only chunks in [c_begin, c_end) are written; the others keep their previous contents (zero here)."""
    g = Geometry(B=1, T=1, L=64, Hq=1, Hkv=1, d=8, S=8, topk=1, W=1)
    x = rand_problem(g, seed=6)
    full_k, full_b = oracle.chunk_summary(g, x["k"], x["q_land"])
    part_k, part_b = oracle.chunk_summary(g, x["k"], x["q_land"], 2, 5)
    np.testing.assert_array_equal(part_k[:, :, 2:5], full_k[:, :, 2:5])
    np.testing.assert_array_equal(part_b[:, :, 2:5], full_b[:, :, 2:5])
    assert np.all(part_k[:, :, :2] == 0) and np.all(part_k[:, :, 5:] == 0)


def test_summary_shared_query_dominant_tokens():
    """Shared landmark query (Sec. 4): q'[h] = 40 e_h serves every chunk of every sequence. Chunk c of KV
    head g holds 40 e_h at token (c + h) mod S for each query head h of the group, so head h's summary of
    chunk c is that token's key with b' ~ 0 (catches a wrong head, chunk or batch index into q')."""
    g = Geometry(B=2, T=1, L=40, Hq=4, Hkv=2, d=8, S=8, topk=1, W=1)
    r = rng(12)
    k = r.standard_normal((2, 2, 40, 8)) * 0.5
    for b in range(2):
        for c in range(g.Nc):
            for h in range(4):
                k[b, h // 2, c * 8 + (c + h) % 8] = 0.0
                k[b, h // 2, c * 8 + (c + h) % 8, h] = 40.0
    qs = 40.0 * np.eye(8)[:4]
    ks, bs = oracle.chunk_summary_shared_query(g, k, qs)
    for b in range(2):
        for h in range(4):
            for c in range(g.Nc):
                np.testing.assert_allclose(ks[b, h, c], k[b, h // 2, c * 8 + (c + h) % 8], atol=1e-12)
                assert bs[b, h, c] < 1e-12
    # and with q' = 0 the shared form is the uniform (mean-key, log S) summary
    ks0, bs0 = oracle.chunk_summary_shared_query(g, k, np.zeros((4, 8)))
    np.testing.assert_allclose(ks0[1, 3], k[1, 1].reshape(5, 8, 8).mean(axis=1), atol=1e-14)
    np.testing.assert_allclose(bs0, math.log(8), atol=1e-14)


def test_eq7_tangency_and_lower_bound():
    """Prop. 3.1 / Eq. 7: s^ = q^.k'/sqrt(d) + b' is the tangent of the chunk LogSumExp at q^ = q'_c, so it
    equals LSE_j(q'.k_j/sqrt(d)) there, and (LSE is convex) never exceeds LSE_j(q^.k_j/sqrt(d))."""
    g = Geometry(B=1, T=1, L=128, Hq=1, Hkv=1, d=16, S=32, topk=1, W=1)
    x = rand_problem(g, seed=7)
    ks, bs = oracle.chunk_summary(g, x["k"], x["q_land"])
    tau = 1 / math.sqrt(16)
    kc = x["k"][0, 0].reshape(4, 32, 16)
    for c in range(4):
        ql = x["q_land"][0, 0, c]
        exact = logsumexp(tau * kc[c] @ ql)
        surrogate = tau * ql @ ks[0, 0, c] + bs[0, 0, c]
        assert abs(surrogate - exact) < 1e-12
        for s in range(20):
            qh = rng(100 + s).standard_normal(16) * 2
            assert tau * qh @ ks[0, 0, c] + bs[0, 0, c] <= logsumexp(tau * kc[c] @ qh) + 1e-12


# ---------------------------------------------------------------- Sec. 2 window

def test_window_golden_c1():
    """Sec. 2 window reading at the tiny config's geometry (S = 32, W = 64), hand-derived values."""
    e = GOLDEN["window_c1_geometry"]
    g = Geometry(B=1, T=512, L=512, Hq=1, Hkv=1, d=4, S=e["S"], topk=1, W=e["W"])
    left, n = oracle.window(g)
    for pos, l_exp, n_exp in zip(e["positions"], e["left"], e["n_cand"]):
        assert left[pos] == l_exp and n[pos] == n_exp


@pytest.mark.parametrize("S,W", [(1, 1), (4, 7), (32, 64), (64, 512), (16, 5)])
def test_window_properties(S, W):
    """The aligned window covers at least W tokens (all of [0,p] when p < W), starts on a chunk boundary,
    and is shorter than W + S; candidate chunks end before it."""
    g = Geometry(B=1, T=700, L=700, Hq=1, Hkv=1, d=4, S=S, topk=1, W=W)
    left, n = oracle.window(g)
    for p in range(700):
        assert left[p] % S == 0 and left[p] <= p
        assert p - left[p] + 1 >= min(W, p + 1)
        assert p - left[p] + 1 < W + S or left[p] == 0
        assert n[p] * S == left[p]


# ---------------------------------------------------------------- Sec. 3/4 selection

def _select_from_scores(b_rows, topk, position, S=1, W=1):
    """Run the oracle selection where s^ = b' (k_sum = 0) for one query at `position`."""
    b_rows = np.asarray(b_rows, dtype=np.float64)
    G, n = b_rows.shape
    L = position + 1
    g = Geometry(B=1, T=1, L=L, Hq=G, Hkv=1, d=4, S=S, topk=topk, W=W, q_pos0=position)
    ks = np.zeros((1, G, g.Nc, 4))
    bs = np.full((1, G, g.Nc), -1e3)
    bs[0, :, :n] = b_rows
    idx, gap = oracle.select_topk(g, np.zeros((1, G, 1, 4)), ks, bs)
    return idx[0, 0, 0], gap[0, 0, 0]


def test_select_golden_gqa_max():
    """Sec. 4 GQA: max over heads of the per-head normalised weights (a mean would pick chunk 1)."""
    e = GOLDEN["gqa_max_not_mean"]
    idx, gap = _select_from_scores(e["b_sum"], 1, e["position"])
    assert list(idx) == e["top1"] and abs(gap - e["gap_top1"]) < 1e-12
    idx, gap = _select_from_scores(e["b_sum"], 2, e["position"])
    assert list(idx) == e["top2"] and abs(gap - e["gap_top2"]) < 1e-12


def test_select_planted_monotone_scores():
    """G = 1: with k'_c = c * e_0 and b' = 0, s^ grows with c when q^_0 > 0, so the top-k are the last k
    candidates (ascending), and gap = tau * q^_0 (one step)."""
    g = Geometry(B=1, T=1, L=1000, Hq=1, Hkv=1, d=4, S=10, topk=5, W=30, q_pos0=999)
    ks = np.zeros((1, 1, g.Nc, 4))
    ks[0, 0, :, 0] = np.arange(g.Nc)
    qh = np.zeros((1, 1, 1, 4))
    qh[..., 0] = 0.7
    idx, gap = oracle.select_topk(g, qh, ks, np.zeros((1, 1, g.Nc)))
    n = oracle.window(g)[1][0]
    assert list(idx[0, 0, 0]) == list(range(n - 5, n))
    assert abs(gap[0, 0, 0] - 0.5 * 0.7) < 1e-12


def test_select_ties_lowest_index_and_padding():
    """Identical chunks tie: the lowest ids win. Fewer candidates than k: all are kept, -1 pads, gap = inf."""
    idx, gap = _select_from_scores(np.zeros((2, 9)), 4, 20)
    assert list(idx) == [0, 1, 2, 3] and gap == 0.0
    idx, gap = _select_from_scores(np.zeros((1, 3)), 6, 3)
    assert list(idx) == [0, 1, 2, -1, -1, -1] and math.isinf(gap)
    g = Geometry(B=1, T=4, L=4, Hq=1, Hkv=1, d=4, S=1, topk=2, W=8)
    idx, gap = oracle.select_topk(g, np.zeros((1, 1, 4, 4)), np.zeros((1, 1, 4, 4)), np.zeros((1, 1, 4)))
    assert np.all(idx == -1) and np.all(np.isinf(gap))  # no candidate inside the first W positions


def test_select_per_head_shift_invariance():
    """Per-head normalisation (Sec. 4): adding a constant to every b' of one head changes nothing
    (without the per-head LSE, the shifted head would take over the max)."""
    g = Geometry(B=1, T=64, L=400, Hq=3, Hkv=1, d=8, S=8, topk=5, W=16, q_pos0=336)
    x = rand_problem(g, seed=11)
    ks, bs = oracle.chunk_summary(g, x["k"], x["q_land"])
    idx0, gap0 = oracle.select_topk(g, x["q_hat"], ks, bs)
    bs2 = bs.copy()
    bs2[:, 1] += 25.0
    idx1, gap1 = oracle.select_topk(g, x["q_hat"], ks, bs2)
    np.testing.assert_array_equal(idx0, idx1)
    np.testing.assert_allclose(gap0, gap1, atol=1e-9)


def test_select_equals_naive_bsa_on_chunk_constant_keys():
    """With every key of a chunk equal and q^ = q, b' = log S and s^_c = log Z_{i,c} exactly, so HiLS
    selection (G = 1) is naive BSA's top-k by exact chunk mass (Sec. 2), computed here by brute force."""
    g = Geometry(B=1, T=40, L=200, Hq=1, Hkv=1, d=8, S=5, topk=3, W=10, q_pos0=160)
    r = rng(12)
    kc = r.standard_normal((g.Nc, 8))
    k = np.repeat(kc, 5, axis=0)[None, None]
    q = r.standard_normal((1, 1, g.T, 8))
    ks, bs = oracle.chunk_summary(g, k, r.standard_normal((1, 1, g.Nc, 8)))
    idx, _ = oracle.select_topk(g, q, ks, bs)
    left, n = oracle.window(g)
    for i in range(g.T):
        logits = k[0, 0] @ q[0, 0, i] / math.sqrt(8)
        mass = np.array([np.exp(logits[c * 5:(c + 1) * 5]).sum() for c in range(n[i])])
        order = sorted(range(n[i]), key=lambda c: (-mass[c], c))[:3]
        assert sorted(order) == list(idx[0, 0, i])


def test_select_head_group_mapping():
    """Selection of group g uses exactly heads g*G .. g*G+G-1: solving each group alone gives the same ids."""
    g = Geometry(B=2, T=16, L=256, Hq=4, Hkv=2, d=8, S=8, topk=4, W=16, q_pos0=240)
    x = rand_problem(g, seed=13)
    ks, bs = oracle.chunk_summary(g, x["k"], x["q_land"])
    idx, gap = oracle.select_topk(g, x["q_hat"], ks, bs)
    for grp in range(2):
        g1 = Geometry(B=2, T=16, L=256, Hq=2, Hkv=1, d=8, S=8, topk=4, W=16, q_pos0=240)
        hs = slice(2 * grp, 2 * grp + 2)
        i1, g1v = oracle.select_topk(g1, x["q_hat"][:, hs], ks[:, hs], bs[:, hs])
        np.testing.assert_array_equal(idx[:, grp:grp + 1], i1)


# ---------------------------------------------------------------- Q-Cal (Sec. 4)

def test_qcal_closed_forms():
    """q^ = q + W_up W_down q: with W_up = 0 (or W_down = 0) q^ = q; with W_down = the first r unit rows and
    W_up = a times their transpose, q^ scales the first r coordinates by 1 + a and keeps the rest (a rank-r
    projector), so the fused selection equals select_topk on that q^."""
    d, r = 16, 4
    rr = rng(41)
    q = rr.standard_normal((1, 2, 30, d))
    wd, wu = rr.standard_normal((r, d)), rr.standard_normal((d, r))
    np.testing.assert_array_equal(oracle.qcal(q, wd, np.zeros((d, r))), q)
    np.testing.assert_array_equal(oracle.qcal(q, np.zeros((r, d)), wu), q)
    e = np.eye(d)[:r]
    expect = q.copy()
    expect[..., :r] *= 1.5
    np.testing.assert_allclose(oracle.qcal(q, e, 0.5 * e.T), expect, rtol=0, atol=1e-15)
    g = Geometry(B=1, T=30, L=30, Hq=2, Hkv=1, d=d, S=4, topk=2, W=6)
    ks, bs = oracle.chunk_summary(g, rr.standard_normal((1, 1, 30, d)), rr.standard_normal((1, 2, g.Nc, d)))
    i1, g1 = oracle.select_topk_qcal(g, q, e, 0.5 * e.T, ks, bs)
    i2, g2 = oracle.select_topk(g, expect, ks, bs)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_allclose(g1, g2, rtol=1e-12)
    # the correction is linear in q and of rank <= r
    corr = oracle.qcal(q, wd, wu) - q
    assert np.linalg.matrix_rank(corr.reshape(-1, d)) <= r


# ---------------------------------------------------------------- naive BSA (Sec. 2)

def test_bsa_masses_brute_force_and_mha_topk():
    """Naive BSA on a tiny MHA case: every chunk mass equals the direct sum of exp(tau q.k_j) over the chunk's
    tokens, and the selection is the top-k of those sums by (mass desc, id asc), as Sec. 2 states."""
    g = Geometry(B=2, T=40, L=40, Hq=2, Hkv=2, d=4, S=4, topk=3, W=6, scale=0.7)
    r = rng(31)
    q = r.standard_normal((2, 2, 40, 4))
    k = r.standard_normal((2, 2, 40, 4))
    idx, gap, mass = oracle.bsa_select_topk(g, q, k)
    for b in range(2):
        for h in range(2):
            for i in range(40):
                left = max(0, i - 6 + 1) // 4 * 4
                n = left // 4
                sums = [sum(math.exp(0.7 * float(q[b, h, i] @ k[b, h, j])) for j in range(4 * c, 4 * c + 4))
                        for c in range(n)]
                np.testing.assert_allclose(np.exp(mass[b, h, i, :n]), sums, rtol=1e-12)
                assert np.all(np.isnan(mass[b, h, i, n:]))
                order = sorted(range(n), key=lambda c: (-sums[c], c))[:3]
                expect = sorted(order) + [-1] * (3 - len(order))
                assert idx[b, h, i].tolist() == expect, (b, h, i)


def test_bsa_masses_partition_the_pre_window_logits():
    """The candidate chunks tile the tokens left of the window: LSE over the chunk masses equals the LSE of
    every logit s_ij with j < l_p (catches a chunk boundary or a token dropped or counted twice)."""
    g = Geometry(B=1, T=200, L=200, Hq=4, Hkv=2, d=8, S=16, topk=4, W=40)
    x = rand_problem(g, seed=32)
    _, _, mass = oracle.bsa_select_topk(g, x["q"], x["k"])
    left, n = oracle.window(g)
    for h in range(4):
        for i in range(0, 200, 7):
            if n[i] == 0:
                continue
            s = g.tau() * x["k"][0, h // 2, :left[i]] @ x["q"][0, h, i]
            assert abs(logsumexp(mass[0, h, i, :n[i]]) - logsumexp(s)) < 1e-11


def test_bsa_equals_hils_on_chunk_constant_keys():
    """With every key of a chunk equal, the landmark summary is exact (k' = k_c, b' = log S, Prop. 3.1), so
    the HiLS selection with q^ = q is the naive BSA selection and s^ is the exact log mass."""
    g = Geometry(B=1, T=160, L=160, Hq=4, Hkv=2, d=8, S=8, topk=3, W=24)
    r = rng(33)
    kc = r.standard_normal((1, 2, g.Nc, 8))
    k = np.repeat(kc, 8, axis=2)
    q = r.standard_normal((1, 4, 160, 8))
    idx_b, gap_b, mass = oracle.bsa_select_topk(g, q, k)
    ks, bs = oracle.chunk_summary(g, k, r.standard_normal((1, 4, g.Nc, 8)))
    idx_h, gap_h = oracle.select_topk(g, q, ks, bs)
    np.testing.assert_array_equal(idx_b, idx_h)
    np.testing.assert_allclose(gap_b, gap_h, rtol=1e-9, atol=1e-12)
    left, n = oracle.window(g)
    for h in range(4):
        for i in range(0, 160, 5):
            closed = g.tau() * kc[0, h // 2, :n[i]] @ q[0, h, i] + math.log(8)
            np.testing.assert_allclose(mass[0, h, i, :n[i]], closed, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- Eq. 10 attention

def test_eq10_golden_three_tokens():
    e = GOLDEN["eq10_three_tokens"]
    g = Geometry(B=1, T=1, L=3, Hq=1, Hkv=1, d=1, S=1, topk=1, W=1, q_pos0=2, scale=1.0)
    k = np.array(e["keys"]).reshape(1, 1, 3, 1)
    v = np.array(e["values"]).reshape(1, 1, 3, 1)
    q = np.ones((1, 1, 1, 1))
    ks, bs = oracle.chunk_summary(g, k, np.zeros((1, 1, 3, 1)))
    idx, _ = oracle.select_topk(g, q, ks, bs)
    assert list(idx[0, 0, 0]) == e["idx"]
    out, lse = oracle.attn_fwd(g, q, k, v, q, ks, bs, idx)
    assert abs(out[0, 0, 0, 0] - e["out"]) < 1e-12 and abs(lse[0, 0, 0] - e["lse"]) < 1e-14


def _full_problem(g, seed, scale=1.0):
    x = rand_problem(g, seed, scale)
    ks, bs = oracle.chunk_summary(g, x["k"], x["q_land"])
    idx, gap = oracle.select_topk(g, x["q_hat"], ks, bs)
    return x, ks, bs, idx


def test_weights_sum_to_one():
    """Eq. 10: the fused weights sum to 1 over window + selected tokens, so v = 1 gives out = 1."""
    g = Geometry(B=2, T=96, L=96, Hq=4, Hkv=2, d=16, S=8, topk=3, W=16)
    x, ks, bs, idx = _full_problem(g, 21)
    out, _ = oracle.attn_fwd(g, x["q"], x["k"], np.ones_like(x["v"]), x["q_hat"], ks, bs, idx)
    np.testing.assert_allclose(out, 1.0, atol=1e-13)


def test_chunked_equals_tokenwise_eq10():
    """The chunked oracle equals Eq. 10 evaluated weight by weight (all candidates selected, and a top-k)."""
    for topk in (64, 3):
        g = Geometry(B=1, T=80, L=80, Hq=4, Hkv=2, d=8, S=4, topk=topk, W=9)
        x, ks, bs, idx = _full_problem(g, 22, scale=0.7)
        out, _ = oracle.attn_fwd(g, x["q"], x["k"], x["v"], x["q_hat"], ks, bs, idx)
        out2, wsum = oracle.eq10_tokenwise(g, x["q"], x["k"], x["v"], x["q_hat"], ks, bs, idx)
        np.testing.assert_allclose(out, out2, atol=1e-12)
        np.testing.assert_allclose(wsum, 1.0, atol=1e-12)


def test_weight_structure_one_hot_values():
    """With one-hot values (d = L, v_j = e_j), out_i is the weight row itself. Check its structure against
    logits computed here: zero outside window + selected chunks; inside the window w ~ exp(s_ij); inside a
    selected chunk w ~ exp(s_ij) and the chunk's total is exp(s^_c)/Z^_i."""
    L = 48
    g = Geometry(B=1, T=L, L=L, Hq=2, Hkv=1, d=L, S=4, topk=2, W=7, scale=0.3)
    r = rng(23)
    q = r.standard_normal((1, 2, L, L))
    k = r.standard_normal((1, 1, L, L))
    qh = r.standard_normal((1, 2, L, L))
    ks, bs = oracle.chunk_summary(g, k, r.standard_normal((1, 2, g.Nc, L)))
    idx, _ = oracle.select_topk(g, qh, ks, bs)
    v = np.eye(L)[None, None]
    w, lse = oracle.attn_fwd(g, q, k, v, qh, ks, bs, idx)
    left, n = oracle.window(g)
    for h in range(2):
        for i in range(L):
            s = 0.3 * k[0, 0] @ q[0, h, i]
            row = w[0, h, i]
            win = np.arange(left[i], i + 1)
            np.testing.assert_allclose(row[win] / row[win].sum(), np.exp(s[win]) / np.exp(s[win]).sum(), atol=1e-12)
            sel = [c for c in idx[0, 0, i] if c >= 0]
            allowed = set(win.tolist())
            for c in sel:
                toks = np.arange(c * 4, c * 4 + 4)
                allowed |= set(toks.tolist())
                shat = 0.3 * qh[0, h, i] @ ks[0, h, c] + bs[0, h, c]
                assert abs(row[toks].sum() - math.exp(shat - lse[0, h, i])) < 1e-12
                np.testing.assert_allclose(row[toks] / row[toks].sum(), np.exp(s[toks]) / np.exp(s[toks]).sum(),
                                           atol=1e-12)
            outside = [j for j in range(L) if j not in allowed]
            assert np.all(row[outside] == 0)


def test_full_causal_attention_special_case():
    """Chunk-constant keys, q^ = q and every candidate selected make s^_c the exact chunk log-mass, so HiLS
    equals exact causal softmax attention (checked against torch SDPA in fp64), lse included."""
    g = Geometry(B=2, T=96, L=96, Hq=4, Hkv=2, d=16, S=8, topk=12, W=10)
    r = rng(24)
    kc = r.standard_normal((2, 2, g.Nc, 16))
    k = np.repeat(kc, 8, axis=2)
    q = r.standard_normal((2, 4, 96, 16))
    v = r.standard_normal((2, 2, 96, 16))
    ks, bs = oracle.chunk_summary(g, k, r.standard_normal((2, 4, g.Nc, 16)))
    idx, _ = oracle.select_topk(g, q, ks, bs)
    out, lse = oracle.attn_fwd(g, q, k, v, q, ks, bs, idx)
    tq = torch.from_numpy(q)
    tk = torch.from_numpy(np.repeat(k, 2, axis=1))
    tv = torch.from_numpy(np.repeat(v, 2, axis=1))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    np.testing.assert_allclose(out, ref.numpy(), atol=1e-12)
    logits = (tq @ tk.transpose(-1, -2)) / 4.0
    logits = logits.masked_fill(torch.ones(96, 96, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(logits, -1).numpy(), atol=1e-12)


def test_sliding_window_when_no_candidates():
    """Rows whose window reaches position 0 have no candidate chunk: plain sliding-window softmax attention."""
    g = Geometry(B=1, T=40, L=40, Hq=2, Hkv=2, d=8, S=8, topk=2, W=40)
    x, ks, bs, idx = _full_problem(g, 25)
    out, lse = oracle.attn_fwd(g, x["q"], x["k"], x["v"], x["q_hat"], ks, bs, idx)
    for h in range(2):
        for i in range(40):
            s = x["k"][0, h, :i + 1] @ x["q"][0, h, i] / math.sqrt(8)
            p = np.exp(s - s.max())
            np.testing.assert_allclose(out[0, h, i], p @ x["v"][0, h, :i + 1] / p.sum(), atol=1e-12)
            assert abs(lse[0, h, i] - logsumexp(s)) < 1e-12


def test_idx_is_a_set():
    """Permuting a row of idx, padding it with -1 or ids >= n_p, or repeating an id, changes nothing."""
    g = Geometry(B=1, T=64, L=64, Hq=2, Hkv=1, d=8, S=4, topk=3, W=8)
    x, ks, bs, idx = _full_problem(g, 26)
    out, lse = oracle.attn_fwd(g, x["q"], x["k"], x["v"], x["q_hat"], ks, bs, idx)
    r = rng(27)
    idx2 = idx.copy()
    for i in range(64):
        idx2[0, 0, i] = r.permutation(idx2[0, 0, i])
    out2, lse2 = oracle.attn_fwd(g, x["q"], x["k"], x["v"], x["q_hat"], ks, bs, idx2)
    np.testing.assert_array_equal(out, out2)
    g5 = Geometry(B=1, T=64, L=64, Hq=2, Hkv=1, d=8, S=4, topk=6, W=8)
    left, n = oracle.window(g)
    idx5 = np.concatenate([idx, idx[..., :1], np.full_like(idx[..., :1], -1), (n[None, None, :, None] + 1)], -1)
    out5, lse5 = oracle.attn_fwd(g5, x["q"], x["k"], x["v"], x["q_hat"], ks, bs, idx5)
    np.testing.assert_allclose(out5, out, atol=1e-15)
    np.testing.assert_allclose(lse5, lse, atol=1e-15)


def test_gqa_equals_mha_with_repeated_kv():
    """GQA attention equals MHA with each KV head repeated G times and the group's idx row repeated."""
    g = Geometry(B=1, T=64, L=64, Hq=4, Hkv=2, d=8, S=4, topk=3, W=8)
    x, ks, bs, idx = _full_problem(g, 28)
    out, lse = oracle.attn_fwd(g, x["q"], x["k"], x["v"], x["q_hat"], ks, bs, idx)
    gm = Geometry(B=1, T=64, L=64, Hq=4, Hkv=4, d=8, S=4, topk=3, W=8)
    out2, lse2 = oracle.attn_fwd(gm, x["q"], np.repeat(x["k"], 2, 1), np.repeat(x["v"], 2, 1), x["q_hat"], ks, bs,
                                 np.repeat(idx, 2, 1))
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def test_query_offset_rows_match_full_prefill():
    """Rows solved with q_pos0 > 0 (a slice of the queries, or one decode row at L-1) equal the same rows of
    the full prefill: every row depends only on its own position."""
    g = Geometry(B=1, T=120, L=120, Hq=2, Hkv=1, d=8, S=4, topk=3, W=9)
    x = rand_problem(g, 29)
    full = oracle.forward(g, x["q"], x["k"], x["v"], x["q_hat"], x["q_land"])
    gs = Geometry(B=1, T=20, L=120, Hq=2, Hkv=1, d=8, S=4, topk=3, W=9, q_pos0=77)
    part = oracle.forward(gs, x["q"][:, :, 77:97], x["k"], x["v"], x["q_hat"][:, :, 77:97], x["q_land"])
    np.testing.assert_array_equal(part["idx"], full["idx"][:, :, 77:97])
    np.testing.assert_allclose(part["out"], full["out"][:, :, 77:97], atol=1e-14)
    gd = Geometry(B=1, T=1, L=120, Hq=2, Hkv=1, d=8, S=4, topk=3, W=9, q_pos0=119)
    o, lse, idx, gap = oracle.decode(gd, x["q"][:, :, 119:], x["q_hat"][:, :, 119:], x["k"], x["v"], full["k_sum"],
                                     full["b_sum"])
    np.testing.assert_allclose(o, full["out"][:, :, 119:], atol=1e-14)
    np.testing.assert_array_equal(idx, full["idx"][:, :, 119:])
