"""Failure detection without a GPU fault: a bounded device-side wait that runs out is recorded in a
device error word and reported by hils_check as HILS_ERR_TIMEOUT, and the context stays usable.

The library's test hook waits, with the same bounded mbarrier wait every kernel uses, on a barrier that
nothing arrives at (no copy, no tensor-core operation is in flight), with a poll limit of a few thousand."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from chunk_wise_hierarchical_summary_b200 import workloads as W
from tests.parity import TOL, assert_close, geometry, np64

pytestmark = pytest.mark.gpu

HILS_OK, HILS_ERR_INVALID_ARG, HILS_ERR_TIMEOUT = 0, 1, 5


@pytest.fixture(scope="module")
def H(cuda_device):
    import chunk_wise_hierarchical_summary_b200.hils as h

    return h


def test_expired_wait_is_reported_and_the_next_call_is_clean(H):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert H.lib.hils_check(stream) == HILS_OK
    # a control: the CTA arrives before it waits, so the wait completes and nothing is recorded
    assert H.lib.hils_test_wait_expiry(4096, 1, stream) == HILS_OK
    assert H.lib.hils_check(stream) == HILS_OK
    # nothing arrives: the wait runs out after its polls and the expiry is reported once
    assert H.lib.hils_test_wait_expiry(4096, 0, stream) == HILS_OK
    assert H.lib.hils_check(stream) == HILS_ERR_TIMEOUT
    assert b"bounded wait expired" in H.lib.hils_last_error()
    assert H.lib.hils_check(stream) == HILS_OK  # reading the error word cleared it
    # out-of-range limits are rejected before any launch
    assert H.lib.hils_test_wait_expiry(0, 0, stream) == HILS_ERR_INVALID_ARG
    assert H.lib.hils_test_wait_expiry((1 << 20) + 1, 0, stream) == HILS_ERR_INVALID_ARG
    # the context is usable: a prefill after the expiry returns HILS_OK and matches the oracle
    w = W.Workload("after_timeout", B=1, T=300, L=300, Hq=8, Hkv=2, d=128, S=64, topk=2, W=64, dtype="bf16",
                   recipe="scaled")
    x = W.prefill_inputs(w, seed=21)
    ref = oracle.forward(geometry(w), *(np64(x[n]) for n in ("q", "k", "v", "q_hat", "q_land")))
    xd = {n: t.cuda() for n, t in x.items()}
    k_sum, b_sum = H.chunk_summary(xd["k"], xd["q_land"], w.S)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    out, lse = H.attn_fwd(xd["q"], xd["k"], xd["v"], xd["q_hat"], k_sum, b_sum, idx, S=w.S, window=w.W)
    assert H.lib.hils_check(stream) == HILS_OK
    assert_close(out, ref["out"], TOL["bf16"], "out")
    assert_close(lse, ref["lse"], TOL["bf16"], "lse")
