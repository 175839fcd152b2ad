"""Python binding of libhils.so (include/hils.h): torch tensors in, torch tensors out.

Argument marshalling only. Every stage of the computation runs in the library's sm_100a kernels;
this module checks tensor devices/dtypes/shapes, allocates outputs and workspace with torch, passes
raw pointers and the current CUDA stream, and raises HilsError on a non-OK status. If libhils.so is
missing it raises at import time: there is no fallback implementation.

Paper: "Hierarchical Sparse Attention Done Right: Toward Infinite Context Modeling" (arXiv 2607.02980).
Call map: chunk_summary = Eq. 8, select_topk = Eq. 7 + Sec. 3 RQ1 + Sec. 4 GQA selection,
attn_fwd = Eq. 10 (prefill), decode = one-token Eq. 7/10 over a KV cache, attn_bwd = its gradients.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhils.so")

HILS_OK = 0
STATUS = {0: "HILS_OK", 1: "HILS_ERR_INVALID_ARG", 2: "HILS_ERR_UNSUPPORTED", 3: "HILS_ERR_WORKSPACE",
          4: "HILS_ERR_CUDA", 5: "HILS_ERR_TIMEOUT"}
HILS_BF16, HILS_FP32 = 0, 1
OP_SUMMARY, OP_SELECT, OP_ATTN_FWD, OP_DECODE, OP_ATTN_BWD = 0, 1, 2, 3, 4

# Every symbol include/hils.h declares (checked by the tests against the header and the library).
EXPORTED = ("hils_workspace_size", "hils_chunk_summary", "hils_chunk_summary_shared_query", "hils_select_topk",
            "hils_select_topk_qcal", "hils_bsa_select_topk", "hils_attn_fwd", "hils_decode", "hils_attn_bwd", "hils_check", "hils_status_string", "hils_last_error",
            "hils_version", "hils_decode_noalloc", "hils_test_wait_expiry", "hils_attn_fwd_shat")


class HilsError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "T", "L", "Hq", "Hkv", "d", "S", "topk", "window", "q_pos0")] + [
        ("scale", ctypes.c_float), ("dtype", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m chunk_wise_hierarchical_summary_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Params)
    vp, st = ctypes.c_void_p, ctypes.c_int
    lib.hils_workspace_size.argtypes = [P, ctypes.c_int]
    lib.hils_workspace_size.restype = ctypes.c_size_t
    lib.hils_chunk_summary.argtypes = [P, vp, vp, ctypes.c_int32, ctypes.c_int32, vp, vp, vp]
    lib.hils_chunk_summary.restype = st
    lib.hils_chunk_summary_shared_query.argtypes = [P, vp, vp, ctypes.c_int32, ctypes.c_int32, vp, vp, vp]
    lib.hils_chunk_summary_shared_query.restype = st
    lib.hils_select_topk.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.hils_select_topk.restype = st
    lib.hils_bsa_select_topk.argtypes = [P, vp, vp, vp, vp, vp, vp]
    lib.hils_bsa_select_topk.restype = st
    lib.hils_select_topk_qcal.argtypes = [P, vp, vp, vp, ctypes.c_int32, vp, vp, vp, vp, vp, vp]
    lib.hils_select_topk_qcal.restype = st
    lib.hils_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.hils_attn_fwd_shat.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.hils_attn_fwd_shat.restype = st
    lib.hils_attn_fwd.restype = st
    lib.hils_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.hils_decode.restype = st
    lib.hils_attn_bwd.argtypes = [P] + [vp] * 17 + [ctypes.c_size_t, vp]
    lib.hils_attn_bwd.restype = st
    lib.hils_decode_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.hils_decode_noalloc.restype = st
    lib.hils_test_wait_expiry.argtypes = [ctypes.c_uint32, ctypes.c_int32, vp]
    lib.hils_test_wait_expiry.restype = st
    lib.hils_check.argtypes = [vp]
    lib.hils_check.restype = st
    lib.hils_status_string.argtypes = [st]
    lib.hils_status_string.restype = ctypes.c_char_p
    lib.hils_last_error.argtypes = []
    lib.hils_last_error.restype = ctypes.c_char_p
    lib.hils_version.argtypes = []
    lib.hils_version.restype = ctypes.c_char_p
    return lib


lib = _load()


def _raise(status: int) -> None:
    if status != HILS_OK:
        raise HilsError(status, lib.hils_last_error().decode())


def make_params(B, T, L, Hq, Hkv, d, S, topk, window, q_pos0=0, scale=0.0, dtype=torch.bfloat16) -> Params:
    code = {torch.bfloat16: HILS_BF16, torch.float32: HILS_FP32}.get(dtype)
    if code is None:
        raise TypeError(f"unsupported dtype {dtype} (bf16 or fp32)")
    return Params(B, T, L, Hq, Hkv, d, S, topk, window, q_pos0, float(scale), code)


def workspace_size(p: Params, op: int) -> int:
    n = lib.hils_workspace_size(ctypes.byref(p), op)
    if n == ctypes.c_size_t(-1).value:
        raise HilsError(1, lib.hils_last_error().decode())
    return int(n)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _lead(name, t, ndim):
    """Device and dtype of a call's leading tensor, the one its sizes are read from: a contiguous CUDA
    tensor with ndim dimensions. The library launches on the current CUDA device, so every call runs
    with this tensor's device current (torch.cuda.device around the C call)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dim() != ndim:
        raise ValueError(f"{name} has {t.dim()} dimensions, expected {ndim}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device.type != "cuda":
        raise ValueError(f"{name} is on {t.device}: the library takes CUDA tensors only")
    return t.device, t.dtype


def _check(name, t, dtype, shape, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _workspace(p: Params, op: int, device, workspace):
    need = workspace_size(p, op)
    if need == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if workspace.numel() < need:
        raise ValueError(f"workspace too small: {workspace.numel()} < {need}")
    return workspace, workspace.numel()


def chunk_summary(k, q_land, S: int, *, c_begin: int = 0, c_end: int | None = None, k_sum=None, b_sum=None,
                  scale: float = 0.0):
    """Eq. 8 summaries. k [B,Hkv,L,d], q_land [B,Hq,Nc,d] -> (k_sum [B,Hq,Nc,d], b_sum [B,Hq,Nc] fp32).
    With c_begin/c_end only those chunks are (re)computed into the given k_sum/b_sum."""
    dev, dt = _lead("k", k, 4)
    B, Hkv, L, d = k.shape
    Hq, Nc = q_land.shape[1], q_land.shape[2]
    _check("q_land", q_land, dt, (B, Hq, L // S, d), dev)
    if k_sum is None:
        k_sum = torch.empty((B, Hq, Nc, d), dtype=dt, device=dev)
    if b_sum is None:
        b_sum = torch.empty((B, Hq, Nc), dtype=torch.float32, device=dev)
    _check("k_sum", k_sum, dt, (B, Hq, Nc, d), dev)
    _check("b_sum", b_sum, torch.float32, (B, Hq, Nc), dev)
    _check("k", k, dt, (B, Hkv, L, d), dev)
    p = make_params(B, 1, L, Hq, Hkv, d, S, 1, 1, 0, scale, dt)
    c_end = Nc if c_end is None else c_end
    with torch.cuda.device(dev):
        _raise(lib.hils_chunk_summary(ctypes.byref(p), _ptr(k), _ptr(q_land), c_begin, c_end, _ptr(k_sum), _ptr(b_sum),
                                      _stream(dev)))
    return k_sum, b_sum


def chunk_summary_shared_query(k, q_shared, S: int, *, c_begin: int = 0, c_end: int | None = None, k_sum=None,
                               b_sum=None, scale: float = 0.0):
    """Eq. 8 summaries with one shared landmark query per head (Sec. 4): k [B,Hkv,L,d], q_shared [Hq,d]
    -> (k_sum [B,Hq,Nc,d], b_sum [B,Hq,Nc] fp32), as chunk_summary with q_land[b,h,c] = q_shared[h]."""
    dev, dt = _lead("k", k, 4)
    B, Hkv, L, d = k.shape
    Hq, Nc = q_shared.shape[0], L // S
    _check("q_shared", q_shared, dt, (Hq, d), dev)
    if k_sum is None:
        k_sum = torch.empty((B, Hq, Nc, d), dtype=dt, device=dev)
    if b_sum is None:
        b_sum = torch.empty((B, Hq, Nc), dtype=torch.float32, device=dev)
    _check("k_sum", k_sum, dt, (B, Hq, Nc, d), dev)
    _check("b_sum", b_sum, torch.float32, (B, Hq, Nc), dev)
    _check("k", k, dt, (B, Hkv, L, d), dev)
    p = make_params(B, 1, L, Hq, Hkv, d, S, 1, 1, 0, scale, dt)
    c_end = Nc if c_end is None else c_end
    with torch.cuda.device(dev):
        _raise(lib.hils_chunk_summary_shared_query(ctypes.byref(p), _ptr(k), _ptr(q_shared), c_begin, c_end,
                                                   _ptr(k_sum), _ptr(b_sum), _stream(dev)))
    return k_sum, b_sum


def _selection_outputs(B, Hq, Hkv, T, topk, dev, with_gap, with_shat, idx, gap, shat):
    if idx is None:
        idx = torch.empty((B, Hkv, T, topk), dtype=torch.int32, device=dev)
    _check("idx", idx, torch.int32, (B, Hkv, T, topk), dev)
    if with_gap and gap is None:
        gap = torch.empty((B, Hkv, T), dtype=torch.float32, device=dev)
    if gap is not None:
        _check("gap", gap, torch.float32, (B, Hkv, T), dev)
    if with_shat and shat is None:
        shat = torch.empty((B, Hq, T, topk), dtype=torch.float32, device=dev)
    if shat is not None:
        _check("shat", shat, torch.float32, (B, Hq, T, topk), dev)
    return idx, gap, shat


def _selection_result(idx, gap, shat, with_shat):
    if with_shat or shat is not None:
        return idx, gap, shat
    return (idx, gap) if gap is not None else idx


def select_topk(q_hat, k_sum, b_sum, *, Hkv: int, L: int, S: int, topk: int, window: int, q_pos0: int = 0,
                    scale: float = 0.0, with_gap: bool = False, with_shat: bool = False, idx=None, gap=None,
                    shat=None):
    """GQA-shared top-k (Eq. 7, Sec. 3 RQ1, Sec. 4). q_hat [B,Hq,T,d], k_sum [B,Hq,Nc,d], b_sum [B,Hq,Nc]
    -> idx [B,Hkv,T,topk] int32 (ascending ids, -1 padded); with with_gap also gap [B,Hkv,T] fp32 and with
    with_shat (idx, gap or None, shat [B,Hq,T,topk] fp32: each head's s^ of the selected ids)."""
    dev, dt = _lead("q_hat", q_hat, 4)
    B, Hq, T, d = q_hat.shape
    Nc = L // S
    _check("k_sum", k_sum, dt, (B, Hq, Nc, d), dev)
    _check("b_sum", b_sum, torch.float32, (B, Hq, Nc), dev)
    idx, gap, shat = _selection_outputs(B, Hq, Hkv, T, topk, dev, with_gap, with_shat, idx, gap, shat)
    p = make_params(B, T, L, Hq, Hkv, d, S, topk, window, q_pos0, scale, dt)
    ws, nws = _workspace(p, OP_SELECT, dev, None)
    with torch.cuda.device(dev):
        _raise(lib.hils_select_topk(ctypes.byref(p), _ptr(q_hat), _ptr(k_sum), _ptr(b_sum), _ptr(idx), _ptr(gap),
                                    _ptr(shat), _ptr(ws), nws, _stream(dev)))
    return _selection_result(idx, gap, shat, with_shat)


def select_topk_qcal(q, w_down, w_up, k_sum, b_sum, *, Hkv: int, L: int, S: int, topk: int, window: int,
                     q_pos0: int = 0, scale: float = 0.0, with_gap: bool = False, with_shat: bool = False, idx=None,
                     gap=None, shat=None):
    """select_topk with Q-Cal fused (Sec. 4): q [B,Hq,T,d], w_down [r,d], w_up [d,r] (r = 32) ->
    idx [B,Hkv,T,topk] int32 (and gap, shat as select_topk), selected on q^ = q + W_up (W_down q)."""
    dev, dt = _lead("q", q, 4)
    B, Hq, T, d = q.shape
    r = w_down.shape[0]
    _check("w_down", w_down, dt, (r, d), dev)
    _check("w_up", w_up, dt, (d, r), dev)
    Nc = L // S
    _check("k_sum", k_sum, dt, (B, Hq, Nc, d), dev)
    _check("b_sum", b_sum, torch.float32, (B, Hq, Nc), dev)
    idx, gap, shat = _selection_outputs(B, Hq, Hkv, T, topk, dev, with_gap, with_shat, idx, gap, shat)
    p = make_params(B, T, L, Hq, Hkv, d, S, topk, window, q_pos0, scale, dt)
    with torch.cuda.device(dev):
        _raise(lib.hils_select_topk_qcal(ctypes.byref(p), _ptr(q), _ptr(w_down), _ptr(w_up), r, _ptr(k_sum),
                                         _ptr(b_sum), _ptr(idx), _ptr(gap), _ptr(shat), _stream(dev)))
    return _selection_result(idx, gap, shat, with_shat)


def bsa_select_topk(q, k, *, S: int, topk: int, window: int, q_pos0: int = 0, scale: float = 0.0,
                    with_gap: bool = False, idx=None, gap=None, mass=None):
    """Naive BSA selection (Sec. 2): exact chunk log-masses and the GQA top-k on them. q [B,Hq,T,d],
    k [B,Hkv,L,d] -> (idx [B,Hkv,T,topk] int32, gap [B,Hkv,T] fp32 or None, mass [B,Hq,T,Nc] fp32; entries
    of mass at c >= n_i are not written)."""
    dev, dt = _lead("q", q, 4)
    B, Hq, T, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    Nc = L // S
    _check("k", k, dt, (B, Hkv, L, d), dev)
    if idx is None:
        idx = torch.empty((B, Hkv, T, topk), dtype=torch.int32, device=dev)
    _check("idx", idx, torch.int32, (B, Hkv, T, topk), dev)
    if with_gap and gap is None:
        gap = torch.empty((B, Hkv, T), dtype=torch.float32, device=dev)
    if gap is not None:
        _check("gap", gap, torch.float32, (B, Hkv, T), dev)
    if mass is None:
        mass = torch.empty((B, Hq, T, Nc), dtype=torch.float32, device=dev)
    _check("mass", mass, torch.float32, (B, Hq, T, Nc), dev)
    p = make_params(B, T, L, Hq, Hkv, d, S, topk, window, q_pos0, scale, dt)
    with torch.cuda.device(dev):
        _raise(lib.hils_bsa_select_topk(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(idx), _ptr(gap), _ptr(mass),
                                        _stream(dev)))
    return idx, gap, mass


def attn_fwd(q, k, v, q_hat, k_sum, b_sum, idx, *, S: int, window: int, q_pos0: int = 0, scale: float = 0.0,
             out=None, lse=None, workspace=None):
    """Eq. 10 prefill. q, q_hat [B,Hq,T,d]; k, v [B,Hkv,L,d]; idx [B,Hkv,T,topk] -> out [B,Hq,T,d], lse [B,Hq,T]."""
    dev, dt = _lead("q", q, 4)
    B, Hq, T, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    topk = idx.shape[-1]
    Nc = L // S
    for name, t, shape in (("k", k, (B, Hkv, L, d)), ("v", v, (B, Hkv, L, d)), ("q_hat", q_hat, (B, Hq, T, d)),
                           ("k_sum", k_sum, (B, Hq, Nc, d))):
        _check(name, t, dt, shape, dev)
    _check("b_sum", b_sum, torch.float32, (B, Hq, Nc), dev)
    _check("idx", idx, torch.int32, (B, Hkv, T, topk), dev)
    if out is None:
        out = torch.empty((B, Hq, T, d), dtype=dt, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
    _check("out", out, dt, (B, Hq, T, d), dev)
    _check("lse", lse, torch.float32, (B, Hq, T), dev)
    p = make_params(B, T, L, Hq, Hkv, d, S, topk, window, q_pos0, scale, dt)
    ws, nws = _workspace(p, OP_ATTN_FWD, dev, workspace)
    with torch.cuda.device(dev):
        _raise(lib.hils_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_hat), _ptr(k_sum), _ptr(b_sum),
                                 _ptr(idx), _ptr(out), _ptr(lse), _ptr(ws), nws, _stream(dev)))
    return out, lse


def attn_fwd_shat(q, k, v, idx, shat, *, S: int, window: int, q_pos0: int = 0, scale: float = 0.0, out=None,
                  lse=None):
    """Eq. 10 prefill from the selection's ids and retrieval scores (select_topk with_shat). q [B,Hq,T,d];
    k, v [B,Hkv,L,d]; idx [B,Hkv,T,topk] canonical; shat [B,Hq,T,topk] -> out [B,Hq,T,d], lse [B,Hq,T]."""
    dev, dt = _lead("q", q, 4)
    B, Hq, T, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    topk = idx.shape[-1]
    for name, t, shape in (("k", k, (B, Hkv, L, d)), ("v", v, (B, Hkv, L, d))):
        _check(name, t, dt, shape, dev)
    _check("idx", idx, torch.int32, (B, Hkv, T, topk), dev)
    _check("shat", shat, torch.float32, (B, Hq, T, topk), dev)
    if out is None:
        out = torch.empty((B, Hq, T, d), dtype=dt, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
    _check("out", out, dt, (B, Hq, T, d), dev)
    _check("lse", lse, torch.float32, (B, Hq, T), dev)
    p = make_params(B, T, L, Hq, Hkv, d, S, topk, window, q_pos0, scale, dt)
    with torch.cuda.device(dev):
        _raise(lib.hils_attn_fwd_shat(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(shat), _ptr(out),
                                      _ptr(lse), _stream(dev)))
    return out, lse


def decode(q, q_hat, k_cache, v_cache, k_sum, b_sum, *, S: int, topk: int, window: int, scale: float = 0.0,
           out=None, lse=None, idx_out=None, return_idx: bool = False, workspace=None):
    """One decode step for the last M = q.shape[2] positions of the cache (M = 1: position L-1).
    q, q_hat [B,Hq,M,d]; caches [B,Hkv,L,d]; k_sum [B,Hq,Nc,d]; b_sum [B,Hq,Nc] -> out [B,Hq,M,d],
    lse [B,Hq] for M = 1 else [B,Hq,M] (and idx [B,Hkv,topk] for M = 1 else [B,Hkv,M,topk] with
    return_idx)."""
    dev, dt = _lead("q", q, 4)
    B, Hq, M, d = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    Nc = L // S
    _check("q", q, dt, (B, Hq, M, d), dev)
    _check("q_hat", q_hat, dt, (B, Hq, M, d), dev)
    _check("k_cache", k_cache, dt, (B, Hkv, L, d), dev)
    _check("v_cache", v_cache, dt, (B, Hkv, L, d), dev)
    _check("k_sum", k_sum, dt, (B, Hq, Nc, d), dev)
    _check("b_sum", b_sum, torch.float32, (B, Hq, Nc), dev)
    lse_shape = (B, Hq) if M == 1 else (B, Hq, M)
    idx_shape = (B, Hkv, topk) if M == 1 else (B, Hkv, M, topk)
    if out is None:
        out = torch.empty((B, Hq, M, d), dtype=dt, device=dev)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=dev)
    _check("out", out, dt, (B, Hq, M, d), dev)
    _check("lse", lse, torch.float32, lse_shape, dev)
    if return_idx and idx_out is None:
        idx_out = torch.empty(idx_shape, dtype=torch.int32, device=dev)
    if idx_out is not None:
        _check("idx_out", idx_out, torch.int32, idx_shape, dev)
    p = make_params(B, M, L, Hq, Hkv, d, S, topk, window, L - M, scale, dt)
    ws, nws = _workspace(p, OP_DECODE, dev, workspace)
    with torch.cuda.device(dev):
        _raise(lib.hils_decode(ctypes.byref(p), _ptr(q), _ptr(q_hat), _ptr(k_cache), _ptr(v_cache), _ptr(k_sum),
                               _ptr(b_sum), _ptr(out), _ptr(lse), _ptr(idx_out), _ptr(ws), nws, _stream(dev)))
    return (out, lse, idx_out) if idx_out is not None else (out, lse)


def attn_bwd(q, k, v, q_hat, q_land, k_sum, b_sum, idx, out, lse, dout, *, S: int, window: int, scale: float = 0.0,
             workspace=None):
    """Gradients of sum(dout * out) with idx fixed -> (dq, dk, dv, dq_hat, dq_land)."""
    dev, dt = _lead("q", q, 4)
    B, Hq, T, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    topk = idx.shape[-1]
    Nc = L // S
    for name, t, shape in (("k", k, (B, Hkv, L, d)), ("v", v, (B, Hkv, L, d)), ("q_hat", q_hat, (B, Hq, T, d)),
                           ("q_land", q_land, (B, Hq, Nc, d)), ("k_sum", k_sum, (B, Hq, Nc, d)),
                           ("out", out, (B, Hq, T, d)), ("dout", dout, (B, Hq, T, d))):
        _check(name, t, dt, shape, dev)
    _check("b_sum", b_sum, torch.float32, (B, Hq, Nc), dev)
    _check("lse", lse, torch.float32, (B, Hq, T), dev)
    _check("idx", idx, torch.int32, (B, Hkv, T, topk), dev)
    dq, dq_hat = torch.empty_like(q), torch.empty_like(q_hat)
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    dq_land = torch.empty_like(q_land)
    p = make_params(B, T, L, Hq, Hkv, d, S, topk, window, 0, scale, dt)
    ws, nws = _workspace(p, OP_ATTN_BWD, dev, workspace)
    with torch.cuda.device(dev):
        _raise(lib.hils_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_hat), _ptr(q_land), _ptr(k_sum),
                                 _ptr(b_sum), _ptr(idx), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                 _ptr(dq_hat), _ptr(dq_land), _ptr(ws), nws, _stream(dev)))
    return dq, dk, dv, dq_hat, dq_land


def check(device=None) -> None:
    """Synchronise the current stream and raise on a CUDA or device-side error."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):  # the error words read are those of the current device
        _raise(lib.hils_check(_stream(dev)))


def prefill(q, k, v, q_hat, q_land, *, S: int, topk: int, window: int, scale: float = 0.0):
    """The whole prefill hot path: summaries, selection (with each selected chunk's s^) and attention on
    those scores; shapes the score-taking attention does not cover use hils_attn_fwd. Returns
    (out, lse, idx, k_sum, b_sum)."""
    B, Hq, T, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    k_sum, b_sum = chunk_summary(k, q_land, S, scale=scale)
    idx, _, shat = select_topk(q_hat, k_sum, b_sum, Hkv=Hkv, L=L, S=S, topk=topk, window=window, q_pos0=L - T,
                               scale=scale, with_shat=True)
    try:
        out, lse = attn_fwd_shat(q, k, v, idx, shat, S=S, window=window, q_pos0=L - T, scale=scale)
    except HilsError as e:
        if e.status != 2:  # HILS_ERR_UNSUPPORTED: fall through to the general attention
            raise
        out, lse = attn_fwd(q, k, v, q_hat, k_sum, b_sum, idx, S=S, window=window, q_pos0=L - T, scale=scale)
    return out, lse, idx, k_sum, b_sum
