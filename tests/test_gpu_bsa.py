"""GPU parity of the naive BSA selection (exact chunk masses + group top-k) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from oracle import Geometry
from chunk_wise_hierarchical_summary_b200 import workloads as W
from tests.parity import TOL, assert_close, check_idx, geometry, mass_group_scores, np64

pytestmark = pytest.mark.gpu

H = None
# masses are fp32 LSEs of the same bf16/fp32 inputs on both sides (no rounding of the inputs in between)
MASS_TOL = dict(atol=1e-4, rtol=1e-4)


@pytest.fixture(scope="module", autouse=True)
def hils(cuda_device):
    global H
    import chunk_wise_hierarchical_summary_b200.hils as h

    H = h
    return h


def run_case(w: W.Workload, seed=0):
    x = W.prefill_inputs(w, seed=seed, device="cpu")
    g = geometry(w)
    ridx, rgap, rmass = oracle.bsa_select_topk(g, np64(x["q"]), np64(x["k"]))
    idx, gap, mass = H.bsa_select_topk(x["q"].cuda(), x["k"].cuda(), S=w.S, topk=w.topk, window=w.W,
                                       q_pos0=w.q_pos0, with_gap=True)
    have = ~np.isnan(rmass)
    assert_close(mass.cpu().numpy()[have], rmass[have], MASS_TOL, "mass")
    near = check_idx(idx, ridx, rgap, scores=mass_group_scores(g, rmass))
    finite = np.isfinite(rgap)
    assert_close(gap.cpu().numpy()[finite], rgap[finite], dict(atol=1e-3, rtol=1e-3), "gap")
    assert np.all(np.isinf(gap.cpu().numpy()[~finite]))
    return near


@pytest.mark.parametrize("w", [
    W.TINY_FP32,
    # tensor-core masses: several query tiles, a ragged tail, each GQA width the kernel takes
    W.Workload("bsa_bf16_g4", B=2, T=1000, L=1000, Hq=8, Hkv=2, d=128, S=64, topk=4, W=128, dtype="bf16",
               recipe="tiny"),
    W.Workload("bsa_bf16_g1", B=1, T=700, L=700, Hq=2, Hkv=2, d=128, S=64, topk=5, W=64, dtype="bf16",
               recipe="tiny"),
    W.Workload("bsa_bf16_g2", B=1, T=600, L=600, Hq=4, Hkv=2, d=128, S=64, topk=3, W=200, dtype="bf16",
               recipe="tiny"),
    W.Workload("bsa_bf16_g8", B=1, T=520, L=520, Hq=8, Hkv=1, d=128, S=64, topk=2, W=64, dtype="bf16",
               recipe="tiny"),
    # rows at the end of a longer cache (chunked prefill / decode form)
    W.Workload("bsa_bf16_offset", B=1, T=150, L=2100, Hq=4, Hkv=1, d=128, S=64, topk=8, W=256, dtype="bf16",
               recipe="tiny", q_pos0=1950),
    # CUDA-core masses: d 64, fp32, S 16, topk 32 (the largest the selection takes), > 32 candidates
    W.Workload("bsa_fp32_d64", B=1, T=900, L=900, Hq=4, Hkv=2, d=64, S=16, topk=32, W=32, dtype="fp32",
               recipe="tiny"),
    W.Workload("bsa_bf16_S32", B=1, T=400, L=400, Hq=4, Hkv=4, d=128, S=32, topk=3, W=40, dtype="bf16",
               recipe="tiny"),
    W.Workload("bsa_single_row", B=1, T=1, L=1, Hq=4, Hkv=2, d=128, S=64, topk=3, W=64, dtype="bf16",
               recipe="tiny"),
], ids=lambda w: w.name)
def test_bsa_shapes(w):
    near = run_case(w)
    assert near.mean() < 0.25  # most rows are compared id by id; the others hold a valid top-k


def test_bsa_equals_hils_selection_on_chunk_constant_keys():
    """Chunk-constant keys make the landmark summary exact (Prop. 3.1): the GPU's HiLS selection with
    q^ = q and its naive BSA selection agree (both checked against the oracle first)."""
    w = W.Workload("const", B=1, T=640, L=640, Hq=8, Hkv=2, d=128, S=64, topk=3, W=128, dtype="bf16",
                   recipe="tiny")
    x = W.prefill_inputs(w, seed=5)
    kc = x["k"].reshape(1, 2, 10, 64, 128)[:, :, :, :1].expand(1, 2, 10, 64, 128).reshape(1, 2, 640, 128)
    q, k = x["q"].cuda(), kc.contiguous().cuda()
    g = geometry(w)
    ridx, rgap, _ = oracle.bsa_select_topk(g, np64(x["q"]), np64(kc))
    idx_b, _, _ = H.bsa_select_topk(q, k, S=64, topk=3, window=128)
    near = check_idx(idx_b, ridx, rgap)
    k_sum, b_sum = H.chunk_summary(k, x["q_land"].cuda(), 64)
    idx_h = H.select_topk(q, k_sum, b_sum, Hkv=2, L=640, S=64, topk=3, window=128)
    far = ~near
    assert np.array_equal(idx_h.cpu().numpy()[far], idx_b.cpu().numpy()[far])


def test_bsa_full_size_sampled():
    """The prefill workload's shape (B4 T8192 Hq16 Hkv4 d128 S64 k16 W512) with unit-variance q and k: masses
    and ids of sampled 64-row blocks against the oracle."""
    w = W.Workload("bsa_full", B=4, T=8192, L=8192, Hq=16, Hkv=4, d=128, S=64, topk=16, W=512, dtype="bf16",
                   recipe="tiny")
    x = W.prefill_inputs(w, seed=1, device="cuda")
    idx, gap, mass = H.bsa_select_topk(x["q"], x["k"], S=64, topk=16, window=512, with_gap=True)
    torch.cuda.synchronize()
    for b, grp in ((0, 1), (3, 2)):
        hs = slice(grp * w.G, (grp + 1) * w.G)
        kk = np64(x["k"][b:b + 1, grp:grp + 1])
        for r0 in (512, 4096, w.T - 64):
            gr = Geometry(B=1, T=64, L=w.L, Hq=w.G, Hkv=1, d=w.d, S=w.S, topk=w.topk, W=w.W, q_pos0=r0)
            rows = slice(r0, r0 + 64)
            ridx, rgap, rmass = oracle.bsa_select_topk(gr, np64(x["q"][b:b + 1, hs, rows]), kk)
            have = ~np.isnan(rmass)
            assert_close(mass[b:b + 1, hs, rows].cpu().numpy()[have], rmass[have], MASS_TOL, "mass")
            check_idx(idx[b:b + 1, grp:grp + 1, rows], ridx, rgap, f"idx b{b} g{grp} r{r0}",
                      scores=mass_group_scores(gr, rmass))


def test_bsa_rejects_what_it_does_not_take():
    q = torch.zeros((1, 2, 4, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 2, 4, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError, match="topk"):
        H.bsa_select_topk(q, k, S=1, topk=33, window=1)
