"""GPU parity of the prefill path (summaries, selection, attention) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from oracle import Geometry
from chunk_wise_hierarchical_summary_b200 import workloads as W
from tests.parity import (BSUM_TOL, TOL, assert_close, check_idx, check_shat, geometry, np64,
                           retrieval_group_scores, splice)

pytestmark = pytest.mark.gpu

H = None


@pytest.fixture(scope="module", autouse=True)
def hils(cuda_device):
    global H
    import chunk_wise_hierarchical_summary_b200.hils as h

    H = h
    return h


def run_case(w: W.Workload, seed=0, device="cuda", idx_override=None):
    """Whole prefill on the GPU vs the oracle on every output element."""
    x = W.prefill_inputs(w, seed=seed, device="cpu")
    g = geometry(w)
    ref = oracle.forward(g, *(np64(x[n]) for n in ("q", "k", "v", "q_hat", "q_land")))
    xd = {n: t.to(device) for n, t in x.items()}
    tol = TOL[w.dtype]
    k_sum, b_sum = H.chunk_summary(xd["k"], xd["q_land"], w.S)
    assert_close(k_sum, ref["k_sum"], tol, "k_sum")
    assert_close(b_sum, ref["b_sum"], BSUM_TOL, "b_sum")
    idx, gap = H.select_topk(xd["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                             q_pos0=w.q_pos0, with_gap=True)
    near = check_idx(idx, ref["idx"], ref["gap"],
                     scores=retrieval_group_scores(g, np64(x["q_hat"]), ref["k_sum"], ref["b_sum"]))
    finite = np.isfinite(ref["gap"])
    assert_close(gap.cpu().numpy()[finite], ref["gap"][finite], dict(atol=1e-3, rtol=1e-3), "gap")
    assert np.all(np.isinf(gap.cpu().numpy()[~finite]))
    used = splice(idx, ref["idx"], near)
    out, lse = H.attn_fwd(xd["q"], xd["k"], xd["v"], xd["q_hat"], k_sum, b_sum, used, S=w.S, window=w.W,
                          q_pos0=w.q_pos0)
    ref_out, ref_lse = ref["out"], ref["lse"]
    if near.any():
        ref_out, ref_lse = oracle.attn_fwd(g, np64(x["q"]), np64(x["k"]), np64(x["v"]), np64(x["q_hat"]),
                                           ref["k_sum"], ref["b_sum"], np64(used))
    assert_close(out, ref_out, tol, "out")
    assert_close(lse, ref_lse, tol, "lse")
    # the selection's retrieval scores of its ids, and the attention that takes them
    idx2, _, shat = H.select_topk(xd["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                                  q_pos0=w.q_pos0, with_shat=True)
    assert torch.equal(idx2, idx)
    check_shat(shat, idx, g, np64(x["q_hat"]), np64(k_sum), np64(b_sum))
    if shat_attention_takes(w):
        o_s, l_s = H.attn_fwd_shat(xd["q"], xd["k"], xd["v"], idx, shat, S=w.S, window=w.W, q_pos0=w.q_pos0)
        H.check()
        gi = idx.cpu().numpy()
        if near.any():
            ref_out, ref_lse = oracle.attn_fwd(g, np64(x["q"]), np64(x["k"]), np64(x["v"]), np64(x["q_hat"]),
                                               ref["k_sum"], ref["b_sum"], gi)
        assert_close(o_s, ref_out, tol, "out (shat)")
        assert_close(l_s, ref_lse, tol, "lse (shat)")
        if gather_attention_is_tc(w):  # same kernel, same scores: the same bits
            o_g, l_g = H.attn_fwd(xd["q"], xd["k"], xd["v"], xd["q_hat"], k_sum, b_sum, idx, S=w.S, window=w.W,
                                  q_pos0=w.q_pos0)
            assert torch.equal(o_s, o_g) and torch.equal(l_s, l_g)
    return dict(near=int(near.sum()), rows=near.size)


def shat_attention_takes(w: W.Workload) -> bool:
    """Shapes hils_attn_fwd_shat covers (the tensor-core attention)."""
    return w.dtype == "bf16" and w.d == 128 and w.S == 64 and w.topk <= 32 and 128 % w.G == 0


def gather_attention_is_tc(w: W.Workload) -> bool:
    """hils_attn_fwd runs the same tensor-core kernel (its score gather needs G <= 4 and 1..128 candidates)."""
    last = w.q_pos0 + w.T - 1
    n_max = max(0, last - w.W + 1) // w.S
    return shat_attention_takes(w) and w.G <= 4 and 1 <= n_max <= 128


def test_tiny_fp32_config():
    """The tiny fp32 workload (B1 T512 H2 d64 S32 k4 W64), every element."""
    run_case(W.TINY_FP32)


@pytest.mark.parametrize("w", [
    # bf16 GQA, several 64-token tiles and a ragged tail (T not a multiple of 64 or of S)
    W.Workload("gqa_bf16_ragged", B=2, T=1000, L=1000, Hq=8, Hkv=2, d=128, S=64, topk=4, W=128, dtype="bf16",
               recipe="scaled"),
    W.Workload("gqa_bf16_d64", B=1, T=700, L=700, Hq=4, Hkv=1, d=64, S=32, topk=6, W=100, dtype="bf16",
               recipe="scaled"),
    W.Workload("mha_fp32_tiny_recipe", B=1, T=300, L=300, Hq=3, Hkv=3, d=128, S=16, topk=5, W=40, dtype="fp32",
               recipe="tiny"),
    W.Workload("fp32_S1", B=1, T=80, L=80, Hq=2, Hkv=1, d=64, S=1, topk=7, W=5, dtype="fp32", recipe="tiny"),
    W.Workload("fp32_S128_topk64", B=1, T=900, L=900, Hq=2, Hkv=1, d=64, S=128, topk=64, W=128, dtype="fp32",
               recipe="tiny"),
    W.Workload("bf16_chunked_prefill", B=1, T=200, L=777, Hq=4, Hkv=2, d=128, S=64, topk=3, W=64, dtype="bf16",
               recipe="scaled", q_pos0=577),
    W.Workload("bf16_single_row_at_zero", B=1, T=1, L=1, Hq=4, Hkv=2, d=128, S=64, topk=3, W=64, dtype="bf16",
               recipe="scaled"),
    W.Workload("bf16_G16", B=1, T=400, L=400, Hq=16, Hkv=1, d=128, S=32, topk=2, W=32, dtype="bf16",
               recipe="scaled"),
], ids=lambda w: w.name)
def test_prefill_shapes(w):
    run_case(w)


def test_attn_fwd_shat_beyond_128_candidates():
    """The score-taking attention has no 128-candidate limit: 256 rows at the end of a 12K cache (up to 183
    candidate chunks, selected by the general kernel with its scores) against the oracle on the GPU's ids."""
    w = W.Workload("shat_long", B=1, T=256, L=12288, Hq=8, Hkv=2, d=128, S=64, topk=16, W=512, dtype="bf16",
                   recipe="scaled", q_pos0=12288 - 256)
    x = W.prefill_inputs(w, seed=21, device="cpu")
    g = geometry(w)
    xd = {n: t.cuda() for n, t in x.items()}
    k_sum, b_sum = H.chunk_summary(xd["k"], xd["q_land"], w.S)
    ks, bs = np64(k_sum), np64(b_sum)
    qh = np64(x["q_hat"])
    idx, gap, shat = H.select_topk(xd["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                                   q_pos0=w.q_pos0, with_gap=True, with_shat=True)
    ridx, rgap = oracle.select_topk(g, qh, ks, bs)
    check_idx(idx, ridx, rgap, scores=retrieval_group_scores(g, qh, ks, bs))
    check_shat(shat, idx, g, qh, ks, bs)
    out, lse = H.attn_fwd_shat(xd["q"], xd["k"], xd["v"], idx, shat, S=w.S, window=w.W, q_pos0=w.q_pos0)
    H.check()
    ro, rl = oracle.attn_fwd(g, np64(x["q"]), np64(x["k"]), np64(x["v"]), qh, ks, bs, idx.cpu().numpy())
    assert_close(out, ro, TOL["bf16"], "out")
    assert_close(lse, rl, TOL["bf16"], "lse")


def test_attn_fwd_shat_flags_non_canonical_ids():
    """Ids out of order, out of range or repeated are a reported error (HILS_ERR_INVALID_ARG at hils_check),
    not a fault; the next call with canonical ids is clean and correct."""
    w = W.Workload("shat_bad", B=1, T=512, L=512, Hq=4, Hkv=1, d=128, S=64, topk=3, W=64, dtype="bf16",
                   recipe="scaled")
    x = W.prefill_inputs(w, seed=22, device="cuda")
    k_sum, b_sum = H.chunk_summary(x["k"], x["q_land"], w.S)
    idx, _, shat = H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=1, L=w.L, S=w.S, topk=w.topk, window=w.W,
                                 with_shat=True)
    good_out, good_lse = H.attn_fwd_shat(x["q"], x["k"], x["v"], idx, shat, S=w.S, window=w.W)
    H.check()
    for mutate in ("reverse", "out_of_range", "repeat", "hole"):
        bad = idx.clone()
        row = bad[0, 0, 500]
        assert int((row >= 0).sum()) == 3
        if mutate == "reverse":
            bad[0, 0, 500] = row.flip(0)
        elif mutate == "out_of_range":
            bad[0, 0, 500, 2] = 10 ** 6
        elif mutate == "repeat":
            bad[0, 0, 500, 2] = row[1]
        else:
            bad[0, 0, 500, 1] = -1
        H.attn_fwd_shat(x["q"], x["k"], x["v"], bad, shat, S=w.S, window=w.W)
        with pytest.raises(H.HilsError, match="canonical") as e:
            H.check()
        assert e.value.status == 1
    out, lse = H.attn_fwd_shat(x["q"], x["k"], x["v"], idx, shat, S=w.S, window=w.W)
    H.check()
    assert torch.equal(out, good_out) and torch.equal(lse, good_lse)


def test_idx_read_as_a_set():
    """attn_fwd ignores -1, out-of-range and repeated ids, and the order of a row."""
    w = W.Workload("set", B=1, T=256, L=256, Hq=4, Hkv=2, d=128, S=16, topk=3, W=32, dtype="fp32", recipe="tiny")
    x = W.prefill_inputs(w, seed=3)
    g = geometry(w)
    ref = oracle.forward(g, *(np64(x[n]) for n in ("q", "k", "v", "q_hat", "q_land")))
    messy = np.concatenate([ref["idx"][..., ::-1], ref["idx"][..., :1], np.full_like(ref["idx"][..., :1], -1),
                            np.full_like(ref["idx"][..., :1], 10 ** 6)], -1).copy()
    xd = {n: t.cuda() for n, t in x.items()}
    k_sum, b_sum = H.chunk_summary(xd["k"], xd["q_land"], w.S)
    out, lse = H.attn_fwd(xd["q"], xd["k"], xd["v"], xd["q_hat"], k_sum, b_sum,
                          torch.from_numpy(messy.astype(np.int32)).cuda(), S=w.S, window=w.W)
    assert_close(out, ref["out"], TOL["fp32"], "out")
    assert_close(lse, ref["lse"], TOL["fp32"], "lse")


def test_summary_chunk_range_only_touches_range():
    w = W.Workload("rng", B=2, T=512, L=512, Hq=4, Hkv=2, d=128, S=64, topk=2, W=64, dtype="bf16", recipe="scaled")
    x = {n: t.cuda() for n, t in W.prefill_inputs(w, seed=4).items()}
    k_sum = torch.full((2, 4, 8, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    b_sum = torch.full((2, 4, 8), 7.0, device="cuda")
    H.chunk_summary(x["k"], x["q_land"], 64, c_begin=3, c_end=6, k_sum=k_sum, b_sum=b_sum)
    full_k, full_b = H.chunk_summary(x["k"], x["q_land"], 64)
    assert torch.equal(k_sum[:, :, 3:6], full_k[:, :, 3:6]) and torch.equal(b_sum[:, :, 3:6], full_b[:, :, 3:6])
    assert torch.all(k_sum[:, :, :3] == 7) and torch.all(k_sum[:, :, 6:] == 7) and torch.all(b_sum[:, :, 6:] == 7)


def test_prefill_full_size_sampled():
    """The prefill workload at full size (B4 T8192 Hq16 Hkv4 d128 S64 k16 W512): summaries of two whole
    (b, group) slices and selection + attention of three 64-row blocks each, against the oracle."""
    w = W.PREFILL_BF16
    x = W.prefill_inputs(w, seed=0, device="cuda")
    k_sum, b_sum = H.chunk_summary(x["k"], x["q_land"], w.S)
    idx, gap = H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                             with_gap=True)
    out, lse = H.attn_fwd(x["q"], x["k"], x["v"], x["q_hat"], k_sum, b_sum, idx, S=w.S, window=w.W)
    torch.cuda.synchronize()
    tol = TOL["bf16"]
    for b, grp in ((0, 0), (3, 3)):
        hs = slice(grp * w.G, (grp + 1) * w.G)
        kk = np64(x["k"][b:b + 1, grp:grp + 1])
        vv = np64(x["v"][b:b + 1, grp:grp + 1])
        ql = np64(x["q_land"][b:b + 1, hs])
        g1 = Geometry(B=1, T=64, L=w.L, Hq=w.G, Hkv=1, d=w.d, S=w.S, topk=w.topk, W=w.W)
        rk, rb = oracle.chunk_summary(g1, kk, ql)
        assert_close(k_sum[b:b + 1, hs], rk, tol, "k_sum")
        assert_close(b_sum[b:b + 1, hs], rb, BSUM_TOL, "b_sum")
        for r0 in (0, 4000, w.T - 64):
            gr = Geometry(B=1, T=64, L=w.L, Hq=w.G, Hkv=1, d=w.d, S=w.S, topk=w.topk, W=w.W, q_pos0=r0)
            rows = slice(r0, r0 + 64)
            qh = np64(x["q_hat"][b:b + 1, hs, rows])
            ridx, rgap = oracle.select_topk(gr, qh, rk, rb)
            near = check_idx(idx[b:b + 1, grp:grp + 1, rows], ridx, rgap, f"idx b{b} g{grp} r{r0}",
                             scores=retrieval_group_scores(gr, qh, rk, rb))
            used = np.where(near[..., None], ridx, idx[b:b + 1, grp:grp + 1, rows].cpu().numpy())
            ro, rl = oracle.attn_fwd(gr, np64(x["q"][b:b + 1, hs, rows]), kk, vv, qh, rk, rb, used)
            if near.any():  # recompute those rows on the GPU with the oracle's ids
                sub_idx = idx.clone()
                sub_idx[b:b + 1, grp:grp + 1, rows] = torch.from_numpy(used.astype(np.int32)).cuda()
                o2, l2 = H.attn_fwd(x["q"], x["k"], x["v"], x["q_hat"], k_sum, b_sum, sub_idx, S=w.S, window=w.W)
                assert_close(o2[b:b + 1, hs, rows], ro, tol, "out")
                assert_close(l2[b:b + 1, hs, rows], rl, tol, "lse")
            else:
                assert_close(out[b:b + 1, hs, rows], ro, tol, "out")
                assert_close(lse[b:b + 1, hs, rows], rl, tol, "lse")
    # the bench's path (selection with scores, attention on them) gives the same bits at full size
    idx_s, _, shat = H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                                   with_shat=True)
    out_s, lse_s = H.attn_fwd_shat(x["q"], x["k"], x["v"], idx_s, shat, S=w.S, window=w.W)
    H.check()
    assert torch.equal(idx_s, idx) and torch.equal(out_s, out) and torch.equal(lse_s, lse)
    # properties that hold everywhere: every row is finite, ids ascending and candidates only
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    pos = torch.arange(w.T, device="cuda")
    n = (torch.clamp(pos - w.W + 1, min=0) // w.S)
    valid = idx >= 0
    assert torch.all(idx < n[None, None, :, None]) and torch.all((idx[..., 1:] > idx[..., :-1]) | ~valid[..., 1:])
    assert torch.all(valid.sum(-1) == torch.clamp(n, max=w.topk)[None, None, :])


@pytest.mark.parametrize("dtype,Hq,Hkv,d,S,L", [
    ("bf16", 16, 4, 128, 64, 64 * 37 + 19),  # streamed tensor-core kernel, ragged tail token
    ("bf16", 8, 1, 128, 64, 64 * 20),        # G = 8
    ("fp32", 4, 2, 64, 32, 32 * 9 + 5),      # CUDA-core kernel
])
def test_chunk_summary_shared_query(dtype, Hq, Hkv, d, S, L):
    """Shared landmark query (one q' per head, Sec. 4) against the oracle, every element, plus a chunk
    range that leaves the other chunks untouched."""
    g = torch.Generator().manual_seed(77)
    B = 2
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    k = torch.randn((B, Hkv, L, d), generator=g).to(dt)
    qs = torch.randn((Hq, d), generator=g).to(dt)
    geo = Geometry(B=B, T=1, L=L, Hq=Hq, Hkv=Hkv, d=d, S=S, topk=1, W=1)
    ref_k, ref_b = oracle.chunk_summary_shared_query(geo, np64(k), np64(qs))
    ks, bs = H.chunk_summary_shared_query(k.cuda(), qs.cuda(), S)
    assert_close(ks, ref_k, TOL[dtype], "k_sum")
    assert_close(bs, ref_b, BSUM_TOL, "b_sum")
    ks2 = torch.full_like(ks, 7.0)
    bs2 = torch.full_like(bs, 7.0)
    H.chunk_summary_shared_query(k.cuda(), qs.cuda(), S, c_begin=3, c_end=7, k_sum=ks2, b_sum=bs2)
    assert torch.equal(ks2[:, :, 3:7], ks[:, :, 3:7]) and torch.equal(bs2[:, :, 3:7], bs[:, :, 3:7])
    assert bool((ks2[:, :, :3] == 7).all()) and bool((bs2[:, :, 7:] == 7).all())


@pytest.mark.parametrize("w", [
    W.Workload("qcal_g4_k16", B=2, T=1000, L=1000, Hq=8, Hkv=2, d=128, S=64, topk=4, W=128, dtype="bf16",
               recipe="scaled"),
    W.Workload("qcal_g2_k32", B=1, T=2000, L=2000, Hq=4, Hkv=2, d=128, S=32, topk=20, W=256, dtype="bf16",
               recipe="scaled"),
    W.Workload("qcal_g1_offset", B=1, T=300, L=2300, Hq=2, Hkv=2, d=128, S=64, topk=6, W=64, dtype="bf16",
               recipe="scaled", q_pos0=2000),
], ids=lambda w: w.name)
def test_select_fused_qcal(w):
    """Selection with Q-Cal fused into the score kernel (q^ = q + W_up W_down q formed in shared memory)
    against the oracle's Q-Cal + selection on the same bf16 q and weights; the unfused call on a q^ made
    the same way agrees outside near ties."""
    x = W.prefill_inputs(w, seed=9)
    # The recipe's q (std d^-1/4) packs the retrieval scores so tightly that up to half of the rows would
    # fall inside the tie band; q x 4 spreads them so that most rows are compared id by id. Rows still
    # inside the band are checked to hold a valid top-k of the oracle's fp64 scores.
    x["q"] = (x["q"].float() * 4).to(x["q"].dtype)
    g = geometry(w)
    xd = {n: t.cuda() for n, t in x.items()}
    k_sum, b_sum = H.chunk_summary(xd["k"], xd["q_land"], w.S)
    ridx, rgap = oracle.select_topk_qcal(g, np64(x["q"]), np64(x["w_down"]), np64(x["w_up"]), np64(k_sum),
                                         np64(b_sum))
    idx, gap = H.select_topk_qcal(xd["q"], xd["w_down"], xd["w_up"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S,
                                  topk=w.topk, window=w.W, q_pos0=w.q_pos0, with_gap=True)
    qhat = oracle.qcal(np64(x["q"]), np64(x["w_down"]), np64(x["w_up"]))
    near = check_idx(idx, ridx, rgap, scores=retrieval_group_scores(g, qhat, np64(k_sum), np64(b_sum)))
    assert near.mean() < 0.25
    finite = np.isfinite(rgap)
    assert_close(gap.cpu().numpy()[finite], rgap[finite], dict(atol=2e-3, rtol=2e-3), "gap")


def test_select_fused_qcal_scores_feed_the_attention():
    """Q-Cal without q^ in memory: the fused selection's scores drive hils_attn_fwd_shat, against the oracle's
    attention on q^ = bf16(q + W_up W_down q) (the fused kernel rounds q^ to bf16 once) and the GPU's ids."""
    w = W.Workload("qcal_shat", B=2, T=1000, L=1000, Hq=8, Hkv=2, d=128, S=64, topk=4, W=128, dtype="bf16",
                   recipe="scaled")
    x = W.prefill_inputs(w, seed=23)
    g = geometry(w)
    xd = {n: t.cuda() for n, t in x.items()}
    k_sum, b_sum = H.chunk_summary(xd["k"], xd["q_land"], w.S)
    ks, bs = np64(k_sum), np64(b_sum)
    idx, _, shat = H.select_topk_qcal(xd["q"], xd["w_down"], xd["w_up"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S,
                                      topk=w.topk, window=w.W, with_shat=True)
    qhat = oracle.qcal(np64(x["q"]), np64(x["w_down"]), np64(x["w_up"]))
    qhat_b = np64(torch.from_numpy(qhat).to(torch.bfloat16))
    ridx, rgap = oracle.select_topk_qcal(g, np64(x["q"]), np64(x["w_down"]), np64(x["w_up"]), ks, bs)
    check_idx(idx, ridx, rgap, scores=retrieval_group_scores(g, qhat, ks, bs))
    check_shat(shat, idx, g, qhat_b, ks, bs, tol=dict(atol=2e-3, rtol=2e-3))
    out, lse = H.attn_fwd_shat(xd["q"], xd["k"], xd["v"], idx, shat, S=w.S, window=w.W)
    H.check()
    ro, rl = oracle.attn_fwd(g, np64(x["q"]), np64(x["k"]), np64(x["v"]), qhat_b, ks, bs, idx.cpu().numpy())
    assert_close(out, ro, TOL["bf16"], "out")
    assert_close(lse, rl, TOL["bf16"], "lse")


def test_select_fused_qcal_full_size_sampled():
    """The prefill workload (B4 T8192 Hq16 Hkv4 d128 S64 k16 W512) with fused Q-Cal: ids of sampled 128-row
    blocks against the oracle on the GPU's summaries."""
    w = W.PREFILL_BF16
    x = W.prefill_inputs(w, seed=0, device="cuda")
    k_sum, b_sum = H.chunk_summary(x["k"], x["q_land"], w.S)
    idx = H.select_topk_qcal(x["q"], x["w_down"], x["w_up"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk,
                             window=w.W)
    torch.cuda.synchronize()
    wd, wu = np64(x["w_down"]), np64(x["w_up"])
    for b, grp in ((1, 0), (2, 3)):
        hs = slice(grp * w.G, (grp + 1) * w.G)
        for r0 in (640, 8192 - 128):
            gr = Geometry(B=1, T=128, L=w.L, Hq=w.G, Hkv=1, d=w.d, S=w.S, topk=w.topk, W=w.W, q_pos0=r0)
            rows = slice(r0, r0 + 128)
            qr = np64(x["q"][b:b + 1, hs, rows])
            ks, bs = np64(k_sum[b:b + 1, hs]), np64(b_sum[b:b + 1, hs])
            ridx, rgap = oracle.select_topk_qcal(gr, qr, wd, wu, ks, bs)
            check_idx(idx[b:b + 1, grp:grp + 1, rows], ridx, rgap, f"idx b{b} g{grp} r{r0}",
                      scores=retrieval_group_scores(gr, oracle.qcal(qr, wd, wu), ks, bs))
