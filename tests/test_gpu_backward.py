"""GPU parity of the backward (training) path against the oracle's analytic gradients."""
import numpy as np
import pytest
import torch

import oracle
from oracle import Geometry
from chunk_wise_hierarchical_summary_b200 import workloads as W
from tests.parity import TOL, assert_close, check_idx, geometry, np64, splice

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
    near = check_idx(idx, ref["idx"], ref["gap"])
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
