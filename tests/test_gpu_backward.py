"""GPU parity of the backward (training) path against the oracle's analytic gradients."""
import numpy as np
import pytest
import torch

import oracle
from oracle import Geometry
from chunk_wise_hierarchical_summary_b200 import workloads as W
from tests.parity import TOL, assert_close, check_idx, geometry, np64, retrieval_group_scores, splice

pytestmark = pytest.mark.gpu

H = None
NAMES = ("dq", "dk", "dv", "dq_hat", "dq_land")


@pytest.fixture(scope="module", autouse=True)
def hils(cuda_device):
    global H
    import chunk_wise_hierarchical_summary_b200.hils as h

    H = h
    return h


def run_bwd(w, seed=0):
    x = W.prefill_inputs(w, seed=seed, device="cpu", with_dout=True)
    g = geometry(w)
    xs = {n: np64(t) for n, t in x.items()}
    ref = oracle.forward(g, xs["q"], xs["k"], xs["v"], xs["q_hat"], xs["q_land"])
    xd = {n: t.cuda() for n, t in x.items()}
    k_sum, b_sum = H.chunk_summary(xd["k"], xd["q_land"], w.S)
    idx, gap = H.select_topk(xd["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                             with_gap=True)
    near = check_idx(idx, ref["idx"], ref["gap"],
                     scores=retrieval_group_scores(g, xs["q_hat"], ref["k_sum"], ref["b_sum"]))
    used = splice(idx, ref["idx"], near)
    out, lse = H.attn_fwd(xd["q"], xd["k"], xd["v"], xd["q_hat"], k_sum, b_sum, used, S=w.S, window=w.W)
    grads = H.attn_bwd(xd["q"], xd["k"], xd["v"], xd["q_hat"], xd["q_land"], k_sum, b_sum, used, out, lse,
                       xd["dout"], S=w.S, window=w.W)
    rgrads = oracle.attn_bwd(g, xs["q"], xs["k"], xs["v"], xs["q_hat"], xs["q_land"], np64(used), xs["dout"])
    tol = TOL[w.dtype]
    for name, a, r in zip(NAMES, grads, rgrads):
        assert_close(a, r, tol, name)


@pytest.mark.parametrize("w", [
    W.Workload("bwd_fp32_c1geom_gqa", B=1, T=512, L=512, Hq=4, Hkv=2, d=64, S=32, topk=4, W=64, dtype="fp32",
               recipe="tiny"),
    W.Workload("bwd_bf16_ragged", B=2, T=700, L=700, Hq=8, Hkv=2, d=128, S=64, topk=3, W=96, dtype="bf16",
               recipe="scaled"),
    W.Workload("bwd_fp32_d128_S16", B=1, T=333, L=333, Hq=2, Hkv=1, d=128, S=16, topk=5, W=20, dtype="fp32",
               recipe="tiny"),
    W.Workload("bwd_bf16_g2_nc15", B=1, T=1000, L=1000, Hq=4, Hkv=2, d=128, S=64, topk=4, W=128, dtype="bf16",
               recipe="scaled"),
    W.Workload("bwd_bf16_g1", B=1, T=900, L=900, Hq=2, Hkv=2, d=128, S=64, topk=5, W=200, dtype="bf16",
               recipe="scaled"),
], ids=lambda w: w.name)
def test_backward_shapes(w):
    run_bwd(w)


def test_backward_training_geometry_one_group():
    """The training workload's per-group geometry (Hq/Hkv = 4, d128, S64, k16, W512) at T = 2048 and one
    KV group, every gradient element against the oracle (which runs one thread per group)."""
    w = W.TRAIN_BF16.with_(B=1, T=2048, L=2048, Hq=4, Hkv=1)
    run_bwd(w, seed=0)


@pytest.mark.slow
def test_backward_training_workload_full_size_sampled():
    """The training workload at full size (B2 T8192 Hq16 Hkv4 d128 S64 k16 W512; Nc = 128 chunks, the most the
    tensor-core backward takes), run whole on the GPU. One (b, KV group) slice, whose gradients depend on
    nothing outside it, is compared element by element with the oracle's analytic gradients: dq, dq_hat of
    the group's heads, dk, dv of its KV head and dq_land of its heads' landmark queries. Near-tie rows of the
    slice get the oracle's ids, fed to the GPU forward and backward."""
    w = W.TRAIN_BF16
    x = W.prefill_inputs(w, seed=0, device="cuda", with_dout=True)
    k_sum, b_sum = H.chunk_summary(x["k"], x["q_land"], w.S)
    idx, gap = H.select_topk(x["q_hat"], k_sum, b_sum, Hkv=w.Hkv, L=w.L, S=w.S, topk=w.topk, window=w.W,
                             with_gap=True)
    b, grp = 1, 2
    hs = slice(grp * w.G, (grp + 1) * w.G)
    g1 = Geometry(B=1, T=w.T, L=w.L, Hq=w.G, Hkv=1, d=w.d, S=w.S, topk=w.topk, W=w.W)
    xs = {n: np64(x[n][b:b + 1, hs]) for n in ("q", "q_hat", "q_land", "dout")}
    xs.update({n: np64(x[n][b:b + 1, grp:grp + 1]) for n in ("k", "v")})
    ref = oracle.forward(g1, xs["q"], xs["k"], xs["v"], xs["q_hat"], xs["q_land"])
    near = check_idx(idx[b:b + 1, grp:grp + 1], ref["idx"], ref["gap"], f"idx b{b} g{grp}",
                     scores=retrieval_group_scores(g1, xs["q_hat"], ref["k_sum"], ref["b_sum"]))
    used = idx.clone()
    used[b:b + 1, grp:grp + 1] = splice(idx[b:b + 1, grp:grp + 1], ref["idx"], near)
    out, lse = H.attn_fwd(x["q"], x["k"], x["v"], x["q_hat"], k_sum, b_sum, used, S=w.S, window=w.W)
    grads = H.attn_bwd(x["q"], x["k"], x["v"], x["q_hat"], x["q_land"], k_sum, b_sum, used, out, lse, x["dout"],
                       S=w.S, window=w.W)
    torch.cuda.synchronize()
    tol = TOL[w.dtype]
    ref_used = np64(used[b:b + 1, grp:grp + 1])
    ro, rl = oracle.attn_fwd(g1, xs["q"], xs["k"], xs["v"], xs["q_hat"], ref["k_sum"], ref["b_sum"], ref_used)
    assert_close(out[b:b + 1, hs], ro, tol, "out")
    assert_close(lse[b:b + 1, hs], rl, tol, "lse")
    rgrads = oracle.attn_bwd(g1, xs["q"], xs["k"], xs["v"], xs["q_hat"], xs["q_land"], ref_used, xs["dout"])
    sl = {"dq": (b, hs), "dq_hat": (b, hs), "dq_land": (b, hs), "dk": (b, grp), "dv": (b, grp)}
    for name, a, r in zip(NAMES, grads, rgrads):
        bb, hh = sl[name]
        sub = a[bb:bb + 1, hh] if isinstance(hh, slice) else a[bb:bb + 1, hh:hh + 1]
        assert_close(sub, r, tol, name)
