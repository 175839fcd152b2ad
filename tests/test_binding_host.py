"""Host-side checks of the Python binding (no GPU needed). Each wrapper is driven against a stand-in for
the C library that checks every argument against the real library's ctypes signature and records the
call, so the test sees exactly what would cross the C ABI: the sizes in hils_params, and the tensors'
data pointers in the header's order. The CUDA-only rules (a leading tensor on the CPU, of the wrong
rank or not contiguous) are checked with the binding as it is."""
import contextlib
import ctypes

import pytest
import torch

import chunk_wise_hierarchical_summary_b200.hils as H

REAL = H.lib
B, HQ, HKV, T, L, D, S, K, W = 1, 4, 2, 8, 128, 64, 32, 2, 32
NC = L // S


class FakeLib:
    """Entry points that convert their arguments through the real argtypes (ctypes raises on a wrong
    count or type) and return HILS_OK; host-only calls go to the real library."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        real = getattr(REAL, name)
        if name in ("hils_workspace_size", "hils_last_error", "hils_status_string", "hils_version"):
            return real

        def call(*args):
            assert len(args) == len(real.argtypes), (name, len(args), len(real.argtypes))
            for a, t in zip(args, real.argtypes):
                t.from_param(a)
            self.calls.append((name, args))
            return H.HILS_OK

        return call


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(H, "lib", lib)
    monkeypatch.setattr(H, "_stream", lambda device: ctypes.c_void_p(None))
    monkeypatch.setattr(torch.cuda, "device", lambda device: contextlib.nullcontext())

    def lead_on_cpu(name, t, ndim):  # the binding's rules except the device type
        assert t.dim() == ndim and t.is_contiguous(), name
        return t.device, t.dtype

    monkeypatch.setattr(H, "_lead", lead_on_cpu)
    return lib


def rnd(*shape, dtype=torch.float32):
    return torch.randn(shape, dtype=torch.float32).to(dtype)


def ptrs(args):
    """Data pointers among a call's arguments (c_void_p or None), in order, without the stream."""
    out = [a.value if isinstance(a, ctypes.c_void_p) else None for a in args[1:-1]
           if a is None or isinstance(a, ctypes.c_void_p)]
    return out


def p_fields(args):
    p = args[0]._obj  # ctypes.byref keeps the structure it points at
    return {n: getattr(p, n) for n, _ in H.Params._fields_}


def dp(t):
    return None if t is None else t.data_ptr()


def test_summaries_marshal_their_tensors(fake):
    k, q_land = rnd(B, HKV, L, D), rnd(B, HQ, NC, D)
    k_sum, b_sum = H.chunk_summary(k, q_land, S)
    (name, args), = fake.calls
    assert name == "hils_chunk_summary"
    assert ptrs(args) == [dp(k), dp(q_land), dp(k_sum), dp(b_sum)]
    assert args[3:5] == (0, NC)
    f = p_fields(args)
    assert (f["B"], f["L"], f["Hq"], f["Hkv"], f["d"], f["S"], f["dtype"]) == (B, L, HQ, HKV, D, S, H.HILS_FP32)
    q_shared = rnd(HQ, D)
    k_sum2, b_sum2 = H.chunk_summary_shared_query(k, q_shared, S, c_begin=1, c_end=3)
    name, args = fake.calls[-1]
    assert name == "hils_chunk_summary_shared_query"
    assert ptrs(args) == [dp(k), dp(q_shared), dp(k_sum2), dp(b_sum2)]
    assert args[3:5] == (1, 3)


def test_selections_marshal_their_tensors(fake):
    q_hat, k_sum, b_sum = rnd(B, HQ, T, D), rnd(B, HQ, NC, D), rnd(B, HQ, NC)
    idx, gap, shat = H.select_topk(q_hat, k_sum, b_sum, Hkv=HKV, L=L, S=S, topk=K, window=W, q_pos0=L - T,
                                   with_gap=True, with_shat=True)
    name, args = fake.calls[-1]
    assert name == "hils_select_topk"
    got = ptrs(args)
    assert got[:6] == [dp(q_hat), dp(k_sum), dp(b_sum), dp(idx), dp(gap), dp(shat)]
    assert tuple(idx.shape) == (B, HKV, T, K) and tuple(shat.shape) == (B, HQ, T, K)
    f = p_fields(args)
    assert (f["T"], f["topk"], f["window"], f["q_pos0"]) == (T, K, W, L - T)
    # without the optional outputs the pointers are NULL
    idx2 = H.select_topk(q_hat, k_sum, b_sum, Hkv=HKV, L=L, S=S, topk=K, window=W, q_pos0=L - T)
    _, args = fake.calls[-1]
    assert ptrs(args)[3:6] == [dp(idx2), None, None]

    q, w_down, w_up = rnd(B, HQ, T, D), rnd(32, D), rnd(D, 32)
    idx3, _, shat3 = H.select_topk_qcal(q, w_down, w_up, k_sum, b_sum, Hkv=HKV, L=L, S=S, topk=K, window=W,
                                        q_pos0=L - T, with_shat=True)
    name, args = fake.calls[-1]
    assert name == "hils_select_topk_qcal"
    assert args[4] == 32
    assert ptrs(args) == [dp(q), dp(w_down), dp(w_up), dp(k_sum), dp(b_sum), dp(idx3), None, dp(shat3)]

    k = rnd(B, HKV, L, D)
    idx4, gap4, mass = H.bsa_select_topk(q, k, S=S, topk=K, window=W, q_pos0=L - T, with_gap=True)
    name, args = fake.calls[-1]
    assert name == "hils_bsa_select_topk"
    assert ptrs(args) == [dp(q), dp(k), dp(idx4), dp(gap4), dp(mass)]
    assert tuple(mass.shape) == (B, HQ, T, NC)


def test_attention_calls_marshal_their_tensors(fake):
    q, k, v = rnd(B, HQ, T, D), rnd(B, HKV, L, D), rnd(B, HKV, L, D)
    q_hat, k_sum, b_sum = rnd(B, HQ, T, D), rnd(B, HQ, NC, D), rnd(B, HQ, NC)
    idx = torch.zeros((B, HKV, T, K), dtype=torch.int32)
    shat = rnd(B, HQ, T, K)
    out, lse = H.attn_fwd(q, k, v, q_hat, k_sum, b_sum, idx, S=S, window=W, q_pos0=L - T)
    name, args = fake.calls[-1]
    assert name == "hils_attn_fwd"
    assert ptrs(args)[:9] == [dp(q), dp(k), dp(v), dp(q_hat), dp(k_sum), dp(b_sum), dp(idx), dp(out), dp(lse)]
    out2, lse2 = H.attn_fwd_shat(q, k, v, idx, shat, S=S, window=W, q_pos0=L - T)
    name, args = fake.calls[-1]
    assert name == "hils_attn_fwd_shat"
    assert ptrs(args) == [dp(q), dp(k), dp(v), dp(idx), dp(shat), dp(out2), dp(lse2)]
    assert tuple(out2.shape) == (B, HQ, T, D) and tuple(lse2.shape) == (B, HQ, T)

    # the backward (self-attention: T = L)
    qf, qh, q_land = rnd(B, HQ, L, D), rnd(B, HQ, L, D), rnd(B, HQ, NC, D)
    idxf = torch.zeros((B, HKV, L, K), dtype=torch.int32)
    outf, lsef, dout = rnd(B, HQ, L, D), rnd(B, HQ, L), rnd(B, HQ, L, D)
    dq, dk, dv, dq_hat, dq_land = H.attn_bwd(qf, k, v, qh, q_land, k_sum, b_sum, idxf, outf, lsef, dout, S=S,
                                             window=W)
    name, args = fake.calls[-1]
    assert name == "hils_attn_bwd"
    assert ptrs(args)[:16] == [dp(t) for t in (qf, k, v, qh, q_land, k_sum, b_sum, idxf, outf, lsef, dout, dq, dk,
                                                dv, dq_hat, dq_land)]
    assert p_fields(args)["q_pos0"] == 0


@pytest.mark.parametrize("M", [1, 4])
def test_decode_marshals_its_tensors(fake, M):
    q, q_hat = rnd(B, HQ, M, D), rnd(B, HQ, M, D)
    kc, vc, k_sum, b_sum = rnd(B, HKV, L, D), rnd(B, HKV, L, D), rnd(B, HQ, NC, D), rnd(B, HQ, NC)
    out, lse, idx = H.decode(q, q_hat, kc, vc, k_sum, b_sum, S=S, topk=K, window=W, return_idx=True)
    name, args = fake.calls[-1]
    assert name == "hils_decode"
    assert ptrs(args)[:9] == [dp(q), dp(q_hat), dp(kc), dp(vc), dp(k_sum), dp(b_sum), dp(out), dp(lse), dp(idx)]
    f = p_fields(args)
    assert (f["T"], f["q_pos0"]) == (M, L - M)
    assert tuple(lse.shape) == ((B, HQ) if M == 1 else (B, HQ, M))
    assert tuple(idx.shape) == ((B, HKV, K) if M == 1 else (B, HKV, M, K))


def test_prefill_is_summaries_selection_and_score_taking_attention(fake):
    q, k, v = rnd(B, HQ, L, D), rnd(B, HKV, L, D), rnd(B, HKV, L, D)
    q_hat, q_land = rnd(B, HQ, L, D), rnd(B, HQ, NC, D)
    out, lse, idx, k_sum, b_sum = H.prefill(q, k, v, q_hat, q_land, S=S, topk=K, window=W)
    assert [n for n, _ in fake.calls] == ["hils_chunk_summary", "hils_select_topk", "hils_attn_fwd_shat"]
    sel, att = fake.calls[1][1], fake.calls[2][1]
    shat = ptrs(sel)[5]
    assert shat is not None and ptrs(att)[4] == shat  # the selection's s^ feed the attention
    assert ptrs(att)[3] == dp(idx) and ptrs(att)[5:7] == [dp(out), dp(lse)]


def test_check_reads_the_given_device(fake):
    H.check(torch.device("cuda", 0))
    name, args = fake.calls[-1]
    assert name == "hils_check" and len(args) == 1


def test_leading_tensor_must_be_a_contiguous_cuda_tensor():
    q_hat, k_sum, b_sum = rnd(B, HQ, T, D), rnd(B, HQ, NC, D), rnd(B, HQ, NC)
    kw = dict(Hkv=HKV, L=L, S=S, topk=K, window=W, q_pos0=L - T)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        H.select_topk(q_hat, k_sum, b_sum, **kw)
    with pytest.raises(ValueError, match="dimensions"):
        H.select_topk(q_hat[0], k_sum, b_sum, **kw)
    with pytest.raises(ValueError, match="contiguous"):
        H.select_topk(q_hat.transpose(2, 3).contiguous().transpose(2, 3), k_sum, b_sum, **kw)
    with pytest.raises(TypeError, match="torch.Tensor"):
        H.select_topk(q_hat.numpy(), k_sum, b_sum, **kw)
    # every wrapper checks its leading tensor before reading sizes from it
    q, k = rnd(B, HQ, T, D), rnd(B, HKV, L, D)
    for call in (lambda: H.chunk_summary(k, rnd(B, HQ, NC, D), S),
                 lambda: H.chunk_summary_shared_query(k, rnd(HQ, D), S),
                 lambda: H.select_topk_qcal(q, rnd(32, D), rnd(D, 32), k_sum, b_sum, **kw),
                 lambda: H.bsa_select_topk(q, k, S=S, topk=K, window=W, q_pos0=L - T),
                 lambda: H.attn_fwd(q, k, k, q_hat, k_sum, b_sum, torch.zeros((B, HKV, T, K), dtype=torch.int32),
                                    S=S, window=W, q_pos0=L - T),
                 lambda: H.attn_fwd_shat(q, k, k, torch.zeros((B, HKV, T, K), dtype=torch.int32), rnd(B, HQ, T, K),
                                         S=S, window=W, q_pos0=L - T),
                 lambda: H.decode(rnd(B, HQ, 1, D), rnd(B, HQ, 1, D), k, k, k_sum, b_sum, S=S, topk=K, window=W)):
        with pytest.raises(ValueError, match="CUDA tensors only"):
            call()
