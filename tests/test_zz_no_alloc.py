"""hils_decode_noalloc: the decode entry point that allocates nothing (its scratch is a static device
array). It serves callers that cannot hand the library a workspace, such as a serving engine whose
memory planner owns the device, or a foreign-language binding with no device allocator.

Called through the C ABI with raw pointers, it must give the same result as hils_decode (within the
tolerance the other tests use) on two calls in a row, the second with different inputs and sizes so
leftovers of the first call in the shared static array cannot leak into it. Runs alone or after the
other tests; collected last so that a run stopping at the first failure has run everything else."""
import ctypes

import numpy as np
import pytest
import torch

from chunk_wise_hierarchical_summary_b200 import workloads as W
from tests.parity import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H(cuda_device):
    import chunk_wise_hierarchical_summary_b200.hils as h

    return h


def vp(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def reference_and_noalloc(H, w, seed):
    x = {n: t.cuda() for n, t in W.decode_inputs(w, seed=seed, device="cpu").items()}
    k_sum, b_sum = H.chunk_summary(x["k_cache"], x["q_land"], w.S)
    ref_out, ref_lse, ref_idx = H.decode(x["q"], x["q_hat"], x["k_cache"], x["v_cache"], k_sum, b_sum, S=w.S,
                                         topk=w.topk, window=w.W, return_idx=True)
    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    idx = torch.full_like(ref_idx, -7)
    p = H.make_params(w.B, 1, w.L, w.Hq, w.Hkv, w.d, w.S, w.topk, w.W, w.L - 1, 0.0, x["q"].dtype)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = H.lib.hils_decode_noalloc(ctypes.byref(p), vp(x["q"]), vp(x["q_hat"]), vp(x["k_cache"]), vp(x["v_cache"]),
                                   vp(k_sum), vp(b_sum), vp(out), vp(lse), vp(idx), stream)
    assert st == 0, H.lib.hils_last_error()
    assert H.lib.hils_check(stream) == 0
    return (ref_out, ref_lse, ref_idx), (out, lse, idx)


def test_noalloc_decode_matches_decode_twice(H):
    first = W.Workload("noalloc_a", B=2, T=1, L=6000, Hq=8, Hkv=2, d=128, S=64, topk=8, W=256, dtype="bf16",
                       recipe="needle", q_pos0=5999, needles=4)
    second = W.Workload("noalloc_b", B=3, T=1, L=3333, Hq=4, Hkv=1, d=128, S=32, topk=12, W=128, dtype="bf16",
                        recipe="needle", q_pos0=3332, needles=3)
    for w, seed in ((first, 11), (second, 12)):
        (ro, rl, ri), (o, l, i) = reference_and_noalloc(H, w, seed)
        assert torch.equal(i, ri)
        np.testing.assert_allclose(o.float().cpu().numpy(), ro.float().cpu().numpy(), **TOL["bf16"])
        np.testing.assert_allclose(l.cpu().numpy(), rl.cpu().numpy(), **TOL["bf16"])


def test_noalloc_rejects_sizes_beyond_the_static_buffer(H):
    p = H.make_params(256, 1, 1 << 20, 32, 8, 128, 64, 32, 512, (1 << 20) - 1)
    assert H.workspace_size(p, H.OP_DECODE) > (32 << 20)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the call fails before any launch
    st = H.lib.hils_decode_noalloc(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, None, None)
    assert st == 2
    assert b"static buffer" in H.lib.hils_last_error()
