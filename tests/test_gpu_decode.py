"""GPU parity of the single-token decode path against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from oracle import Geometry
from chunk_wise_hierarchical_summary_b200 import workloads as W
from tests.parity import TOL, TIE_BAND, assert_close, check_idx, np64, retrieval_group_scores

pytestmark = pytest.mark.gpu

H = None


@pytest.fixture(scope="module", autouse=True)
def hils(cuda_device):
    global H
    import chunk_wise_hierarchical_summary_b200.hils as h

    H = h
    return h


def check_group_rows(w, x, out, lse, idx, groups):
    """Oracle evaluation of the M = w.T query rows of the listed (b, group) pairs from the raw cache (the
    oracle's own summaries). Ids are bit-exact outside the tie band; a row inside it must hold a valid
    top-k of the oracle's group scores within the band. out and lse are compared element by element with
    the oracle's attention on the GPU's ids (the oracle's own ids wherever the two are compared), so no
    group goes unchecked. Near ties are common on these caches (the k-th and (k+1)-th best of thousands of
    random candidates' scores often lie within 1e-3), so the guard that enough ids are still compared one
    by one fails only when more than three quarters of the query rows (and more than one) are near ties.
    Returns the number of near-tie rows."""
    tol = TOL[w.dtype]
    M = w.T
    near_rows = 0
    for b, grp in groups:
        hs = slice(grp * w.G, (grp + 1) * w.G)
        g1 = Geometry(B=1, T=M, L=w.L, Hq=w.G, Hkv=1, d=w.d, S=w.S, topk=w.topk, W=w.W, q_pos0=w.L - M)
        kk = np64(x["k_cache"][b:b + 1, grp:grp + 1])
        vv = np64(x["v_cache"][b:b + 1, grp:grp + 1])
        rk, rb = oracle.chunk_summary(g1, kk, np64(x["q_land"][b:b + 1, hs]))
        qh = np64(x["q_hat"][b:b + 1, hs])
        ridx, rgap = oracle.select_topk(g1, qh, rk, rb)
        got = idx[b, grp].reshape(1, 1, M, w.topk)
        near = check_idx(got, ridx, rgap, f"decode idx b{b} g{grp}", scores=retrieval_group_scores(g1, qh, rk, rb))
        near_rows += int(near.sum())
        used = got.cpu().numpy()
        ro, rl = oracle.attn_fwd(g1, np64(x["q"][b:b + 1, hs]), kk, vv, qh, rk, rb, used)
        assert_close(out[b:b + 1, hs], ro, tol, f"decode out b{b} g{grp}")
        assert_close(lse[b:b + 1, hs].reshape(1, w.G, M), rl, tol, f"decode lse b{b} g{grp}")
    rows = len(groups) * M
    assert near_rows <= max(1, 3 * rows // 4), f"{near_rows} of {rows} query rows are near ties"
    return near_rows


@pytest.mark.parametrize("w", [
    W.Workload("dec_small_ragged", B=2, T=1, L=4133, Hq=8, Hkv=2, d=128, S=64, topk=8, W=256, dtype="bf16",
               recipe="needle", q_pos0=4132, needles=4),
    W.Workload("dec_fp32_d64", B=1, T=1, L=2000, Hq=4, Hkv=4, d=64, S=16, topk=12, W=50, dtype="fp32",
               recipe="needle", q_pos0=1999, needles=3),
    W.Workload("dec_short_no_candidates", B=1, T=1, L=300, Hq=4, Hkv=1, d=128, S=64, topk=4, W=512, dtype="bf16",
               recipe="needle", q_pos0=299, needles=0),
    W.Workload("dec_topk_over_cands", B=1, T=1, L=900, Hq=4, Hkv=2, d=128, S=64, topk=32, W=512, dtype="bf16",
               recipe="needle", q_pos0=899, needles=2),
    W.Workload("dec_g8_ragged", B=2, T=1, L=5000, Hq=16, Hkv=2, d=128, S=64, topk=12, W=300, dtype="bf16",
               recipe="needle", q_pos0=4999, needles=5),
    W.Workload("dec_g1", B=1, T=1, L=3000, Hq=3, Hkv=3, d=128, S=64, topk=8, W=200, dtype="bf16",
               recipe="needle", q_pos0=2999, needles=3),
    # the selection kernels' boundary: 2048 candidates (the short-list kernel, every warp full, G = 8) and
    # 2049 (the bounded survivor kernel with its parallel ranking, G = 4 and G = 8)
    W.Workload("dec_short_list_full_g8", B=1, T=1, L=131584, Hq=8, Hkv=1, d=128, S=64, topk=32, W=512,
               dtype="bf16", recipe="needle", q_pos0=131583, needles=4),
    W.Workload("dec_long_list_first_g4", B=1, T=1, L=131648, Hq=4, Hkv=1, d=128, S=64, topk=32, W=512,
               dtype="bf16", recipe="needle", q_pos0=131647, needles=4),
    W.Workload("dec_long_list_first_g8", B=1, T=1, L=131648, Hq=8, Hkv=1, d=128, S=64, topk=16, W=512,
               dtype="bf16", recipe="needle", q_pos0=131647, needles=4),
    # one KV group over a 1M-token cache (16385 candidates): the list is split over several selection CTAs
    W.Workload("dec_long_one_group", B=1, T=1, L=1049176, Hq=4, Hkv=1, d=128, S=64, topk=8, W=512, dtype="bf16",
               recipe="needle", q_pos0=1049175, needles=4),
], ids=lambda w: w.name)
def test_decode_shapes(w):
    x = W.decode_inputs(w, seed=1, device="cpu")
    xd = {n: t.cuda() for n, t in x.items()}
    k_sum, b_sum = H.chunk_summary(xd["k_cache"], xd["q_land"], w.S)
    out, lse, idx = H.decode(xd["q"], xd["q_hat"], xd["k_cache"], xd["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk,
                             window=w.W, return_idx=True)
    check_group_rows(w, x, out, lse, idx, [(b, g) for b in range(w.B) for g in range(w.Hkv)])


def test_decode_equals_prefill_last_row():
    """A decode step equals the last row of a prefill over the same cache (same kernels' semantics)."""
    w = W.Workload("dec_vs_prefill", B=1, T=1, L=1500, Hq=4, Hkv=2, d=128, S=64, topk=6, W=128, dtype="fp32",
                   recipe="needle", q_pos0=1499, needles=3)
    x = {n: t.cuda() for n, t in W.decode_inputs(w, seed=2, device="cpu").items()}
    k_sum, b_sum = H.chunk_summary(x["k_cache"], x["q_land"], w.S)
    out, lse, idx = H.decode(x["q"], x["q_hat"], x["k_cache"], x["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk,
                             window=w.W, return_idx=True)
    pidx, gap = H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                              q_pos0=w.L - 1, with_gap=True)
    assert torch.equal(pidx[:, :, 0], idx) or bool((gap < TIE_BAND).any())
    pout, plse = H.attn_fwd(x["q"], x["k_cache"], x["v_cache"], x["q_hat"], k_sum, b_sum, pidx, S=w.S, window=w.W,
                            q_pos0=w.L - 1)
    assert_close(out, np64(pout), dict(atol=1e-5, rtol=1e-5), "out")
    assert_close(lse, np64(plse[..., 0]), dict(atol=1e-5, rtol=1e-5), "lse")


def test_decode_full_size_sampled():
    """The decode workload at full size (B8 L524288 Hq32 Hkv8 d128 S64 k32 W512, 16 needles/sequence),
    checked against the oracle on three (b, group) pairs; needles must all be retrieved."""
    w = W.DECODE_BF16
    x = W.decode_inputs(w, seed=0, device="cuda")
    k_sum, b_sum = H.chunk_summary(x["k_cache"], x["q_land"], w.S)
    out, lse, idx = H.decode(x["q"], x["q_hat"], x["k_cache"], x["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk,
                             window=w.W, return_idx=True)
    torch.cuda.synchronize()
    check_group_rows(w, x, out, lse, idx, [(0, 0), (3, 5), (7, 7)])
    for b in range(w.B):
        got = set(idx[b, 0].tolist())
        assert set(x["needle_chunks"][b].tolist()) <= got


@pytest.mark.parametrize("L", list(W.DECODE_SWEEP_L))
def test_decode_sweep_sampled(L):
    """Context-length sweep (B1, same heads/S/k/W; every length the benchmark times, 32K to 4M tokens):
    six KV groups per length against the oracle."""
    w = W.decode_sweep(L)
    x = W.decode_inputs(w, seed=5, device="cuda")
    k_sum, b_sum = H.chunk_summary(x["k_cache"], x["q_land"], w.S)
    out, lse, idx = H.decode(x["q"], x["q_hat"], x["k_cache"], x["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk,
                             window=w.W, return_idx=True)
    torch.cuda.synchronize()
    check_group_rows(w, x, out, lse, idx, [(0, g) for g in (0, 1, 3, 4, 6, 7)])


def test_decode_select_periodic_scores():
    """Scores boosted on every 32nd candidate: one lane of every warp of the single-CTA selection holds
    all the winners, so the candidates at or below the per-thread bound (about 200 here) overflow the
    survivor buffer and the out-of-line running-top-32 path decides. Ids must still equal the oracle's
    selection on the same summaries, and the attention must match the oracle's with those ids."""
    w = W.Workload("dec_periodic", B=1, T=1, L=400000, Hq=4, Hkv=1, d=128, S=64, topk=32, W=512, dtype="bf16",
                   recipe="needle", q_pos0=399999, needles=0)
    x = W.decode_inputs(w, seed=5, device="cpu")
    g = torch.Generator().manual_seed(11)
    k_sum = (torch.randn((1, w.Hq, w.Nc, w.d), generator=g) * 0.5).to(torch.bfloat16)  # spread: no near ties
    b_sum = torch.zeros((1, w.Hq, w.Nc), dtype=torch.float32)
    b_sum[:, :, ::32] = 8.0
    xd = {n: t.cuda() for n, t in x.items()}
    out, lse, idx = H.decode(xd["q"], xd["q_hat"], xd["k_cache"], xd["v_cache"], k_sum.cuda(), b_sum.cuda(), S=w.S,
                             topk=w.topk, window=w.W, return_idx=True)
    g1 = Geometry(B=1, T=1, L=w.L, Hq=w.G, Hkv=1, d=w.d, S=w.S, topk=w.topk, W=w.W, q_pos0=w.L - 1)
    rk, rb = np64(k_sum), np64(b_sum)
    qh = np64(x["q_hat"])
    ridx, rgap = oracle.select_topk(g1, qh, rk, rb)
    assert (np.asarray(ridx).reshape(-1) % 32 == 0).all()  # the boosted candidates win
    near = check_idx(idx[:, :, None], ridx, rgap, "periodic idx")
    assert not near.any()
    ro, rl = oracle.attn_fwd(g1, np64(x["q"]), np64(x["k_cache"]), np64(x["v_cache"]), qh, rk, rb, ridx)
    assert_close(out, ro, TOL["bf16"], "periodic out")
    assert_close(lse, rl[..., 0], TOL["bf16"], "periodic lse")


@pytest.mark.parametrize("w", [
    # positions 4093..4096 with W 256: the window's left edge crosses a chunk boundary inside the block,
    # so the queries have 59, 59, 60 and 60 candidates
    W.Workload("dec_m4_straddle", B=2, T=4, L=4097, Hq=8, Hkv=2, d=128, S=64, topk=8, W=256, dtype="bf16",
               recipe="needle", q_pos0=4093, needles=4),
    W.Workload("dec_m8_g8", B=1, T=8, L=5000, Hq=16, Hkv=2, d=128, S=64, topk=12, W=300, dtype="bf16",
               recipe="needle", q_pos0=4992, needles=5),
    W.Workload("dec_m2_g1", B=3, T=2, L=3000, Hq=4, Hkv=4, d=128, S=64, topk=8, W=200, dtype="bf16",
               recipe="needle", q_pos0=2998, needles=3),
    # topk >= every query's candidates: the last two queries select chunk 10, which lies in the first two
    # queries' windows (a union tile that is a window tile for some rows and a selected chunk for others)
    W.Workload("dec_m4_window_and_selected", B=1, T=4, L=961, Hq=8, Hkv=2, d=128, S=64, topk=16, W=256,
               dtype="bf16", recipe="needle", q_pos0=957, needles=2),
    W.Workload("dec_m8_g4", B=2, T=8, L=7000, Hq=8, Hkv=2, d=128, S=64, topk=16, W=200, dtype="bf16",
               recipe="needle", q_pos0=6992, needles=5),
], ids=lambda w: w.name)
def test_multi_token_decode(w):
    """M query tokens at the end of the cache in one decode call: per query its own candidates, top-k
    and window, equal to the oracle's prefill-form evaluation of the same M rows."""
    x = W.decode_inputs(w, seed=3, device="cpu")
    xd = {n: t.cuda() for n, t in x.items()}
    k_sum, b_sum = H.chunk_summary(xd["k_cache"], xd["q_land"], w.S)
    out, lse, idx = H.decode(xd["q"], xd["q_hat"], xd["k_cache"], xd["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk,
                             window=w.W, return_idx=True)
    assert tuple(out.shape) == (w.B, w.Hq, w.T, w.d) and tuple(lse.shape) == (w.B, w.Hq, w.T)
    assert tuple(idx.shape) == (w.B, w.Hkv, w.T, w.topk)
    check_group_rows(w, x, out, lse, idx, [(b, g) for b in range(w.B) for g in range(w.Hkv)])


def test_multi_token_decode_full_size_sampled():
    """Multi-token decode at the decode workload's size (B8 L524288 Hq32 Hkv8 d128 S64 k32 W512, M = 4 query
    tokens per sequence) on three (b, group) pairs against the oracle."""
    w = W.DECODE_BF16.with_(name="decode_m4", T=4, q_pos0=W.DECODE_BF16.L - 4)
    x = W.decode_inputs(w, seed=11, device="cuda")
    k_sum, b_sum = H.chunk_summary(x["k_cache"], x["q_land"], w.S)
    out, lse, idx = H.decode(x["q"], x["q_hat"], x["k_cache"], x["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk,
                             window=w.W, return_idx=True)
    torch.cuda.synchronize()
    check_group_rows(w, x, out, lse, idx, [(0, 0), (5, 3), (7, 7)])


def test_multi_token_decode_rows_match_single_token_at_last_position():
    """The last of M queries sees exactly what a single-token step at L-1 sees (same cache, same row)."""
    w = W.Workload("dec_m4_vs_m1", B=2, T=4, L=6000, Hq=8, Hkv=2, d=128, S=64, topk=16, W=512, dtype="bf16",
                   recipe="needle", q_pos0=5996, needles=6)
    x = {n: t.cuda() for n, t in W.decode_inputs(w, seed=9, device="cpu").items()}
    k_sum, b_sum = H.chunk_summary(x["k_cache"], x["q_land"], w.S)
    out4, lse4, idx4 = H.decode(x["q"], x["q_hat"], x["k_cache"], x["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk,
                                window=w.W, return_idx=True)
    q1, qh1 = x["q"][:, :, 3:].contiguous(), x["q_hat"][:, :, 3:].contiguous()
    out1, lse1, idx1 = H.decode(q1, qh1, x["k_cache"], x["v_cache"], k_sum, b_sum, S=w.S, topk=w.topk, window=w.W,
                                return_idx=True)
    # the two paths score with different kernels (fp32 sums in different orders): same ids, outputs
    # within a couple of bf16 steps
    assert torch.equal(idx4[:, :, 3], idx1)
    assert torch.allclose(out4[:, :, 3:].float(), out1.float(), atol=1e-2, rtol=0)
    assert torch.allclose(lse4[:, :, 3], lse1, atol=1e-3, rtol=0)
