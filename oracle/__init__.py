"""fp64 CPU oracle for the HiLS-Attention hot path (numpy in, numpy out).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the benchmark's
CPU-baseline leg. The product path (the CUDA library and its Python binding) never imports it.

Every function converts its inputs to contiguous fp64 (int32 for idx) and calls the plain C
statement in hils_oracle.c, which cites the paper section / equation each step follows:
  chunk_summary  Eq. 8 (Prop. 3.1)            select_topk  Sec. 3 RQ1 + Sec. 4 GQA selection
  chunk_summary_shared_query  Eq. 8 with one landmark query per head (Sec. 4)
  bsa_select_topk  naive BSA (Sec. 2): exact chunk masses, same group top-k
  qcal, select_topk_qcal  Sec. 4 Q-Cal (q^ = q + W_up W_down q), then select_topk
  attn_fwd       Eq. 10, chunked form          eq10_tokenwise  Eq. 10, token by token
  attn_bwd       gradients of the above with the selection held fixed
  decode         select_topk + attn_fwd for one query at position L-1
Parity pins live in tests/test_oracle_pins.py and tests/test_oracle_grad.py.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import numpy as np

from . import build as _build


class _Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "T", "L", "Hq", "Hkv", "d", "S", "topk", "W", "q_pos0")] + [
        ("scale", ctypes.c_double)
    ]


@dataclass
class Geometry:
    """Problem sizes: B batch, T query rows, L KV length, Hq/Hkv heads, d head dim, S chunk size,
    topk selected chunks, W window, q_pos0 absolute position of query row 0, scale (<=0: 1/sqrt(d))."""

    B: int
    T: int
    L: int
    Hq: int
    Hkv: int
    d: int
    S: int
    topk: int
    W: int
    q_pos0: int = 0
    scale: float = 0.0

    @property
    def Nc(self) -> int:
        return self.L // self.S

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def tau(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(self.d)

    def check(self) -> None:
        assert self.B >= 1 and self.T >= 1 and self.L >= 1 and self.d >= 1 and self.S >= 1
        assert self.Hq % self.Hkv == 0, "Hq must be a multiple of Hkv"
        assert self.q_pos0 >= 0 and self.q_pos0 + self.T <= self.L, "query rows must lie inside the KV range"
        assert self.topk >= 1 and self.W >= 1

    def _c(self) -> _Params:
        self.check()
        return _Params(self.B, self.T, self.L, self.Hq, self.Hkv, self.d, self.S, self.topk, self.W, self.q_pos0,
                       float(self.scale))


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        P = ctypes.POINTER(_Params)
        D = ctypes.POINTER(ctypes.c_double)
        I = ctypes.POINTER(ctypes.c_int)
        lib.orc_set_threads.argtypes = [ctypes.c_int]
        lib.orc_max_threads.restype = ctypes.c_int
        lib.orc_window.argtypes = [P, I, I]
        lib.orc_chunk_summary.argtypes = [P, D, D, ctypes.c_int, ctypes.c_int, D, D]
        lib.orc_select_topk.argtypes = [P, D, D, D, I, D]
        lib.orc_bsa_select_topk.argtypes = [P, D, D, I, D, D]
        lib.orc_attn_fwd.argtypes = [P, D, D, D, D, D, D, I, D, D]
        lib.orc_eq10_tokenwise.argtypes = [P, D, D, D, D, D, D, I, D, D]
        lib.orc_attn_bwd.argtypes = [P, D, D, D, D, D, I, D, D, D, D, D, D]
        _lib = lib
    return _lib


def _f64(x, shape) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    assert a.shape == tuple(shape), f"expected shape {tuple(shape)}, got {a.shape}"
    return a


def _i32(x, shape) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.int32))
    assert a.shape == tuple(shape), f"expected shape {tuple(shape)}, got {a.shape}"
    return a


def _pd(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _pi(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def max_threads() -> int:
    return int(_load().orc_max_threads())


def window(g: Geometry):
    """Aligned window left edge and candidate-chunk count for each query row (Sec. 2)."""
    left = np.zeros(g.T, np.int32)
    n = np.zeros(g.T, np.int32)
    _load().orc_window(ctypes.byref(g._c()), _pi(left), _pi(n))
    return left, n


def chunk_summary(g: Geometry, k, q_land, c_begin: int = 0, c_end: int | None = None):
    """Eq. 8: landmark summaries. Returns (k_sum [B,Hq,Nc,d], b_sum [B,Hq,Nc]); chunks outside
    [c_begin, c_end) are left at zero."""
    c_end = g.Nc if c_end is None else c_end
    k = _f64(k, (g.B, g.Hkv, g.L, g.d))
    ql = _f64(q_land, (g.B, g.Hq, g.Nc, g.d))
    ks = np.zeros((g.B, g.Hq, g.Nc, g.d))
    bs = np.zeros((g.B, g.Hq, g.Nc))
    _load().orc_chunk_summary(ctypes.byref(g._c()), _pd(k), _pd(ql), int(c_begin), int(c_end), _pd(ks), _pd(bs))
    return ks, bs


def chunk_summary_shared_query(g: Geometry, k, q_shared, c_begin: int = 0, c_end: int | None = None):
    """Eq. 8 with the shared landmark query of Sec. 4 (one learned query per head instead of one per
    chunk): the summary of chunk c of sequence b under head h uses q_shared[h] as its landmark query."""
    qs = _f64(q_shared, (g.Hq, g.d))
    q_land = np.broadcast_to(qs[None, :, None, :], (g.B, g.Hq, g.Nc, g.d))
    return chunk_summary(g, k, q_land, c_begin, c_end)


def select_topk(g: Geometry, q_hat, k_sum, b_sum):
    """Sec. 3 RQ1 + Sec. 4 GQA: shared top-k chunk ids [B,Hkv,T,topk] (ascending, -1 padded) and the
    k-th minus (k+1)-th group-score gap [B,Hkv,T] (+inf when every candidate is kept)."""
    qh = _f64(q_hat, (g.B, g.Hq, g.T, g.d))
    ks = _f64(k_sum, (g.B, g.Hq, g.Nc, g.d))
    bs = _f64(b_sum, (g.B, g.Hq, g.Nc))
    idx = np.zeros((g.B, g.Hkv, g.T, g.topk), np.int32)
    gap = np.zeros((g.B, g.Hkv, g.T))
    _load().orc_select_topk(ctypes.byref(g._c()), _pd(qh), _pd(ks), _pd(bs), _pi(idx), _pd(gap))
    return idx, gap


def qcal(q, w_down, w_up):
    """Sec. 4 Q-Cal with the token's own query as h: q^ = q + W_up (W_down q), applied to every row
    (last axis) of q; w_down [r, d], w_up [d, r]."""
    q = np.asarray(q, dtype=np.float64)
    return q + (q @ np.asarray(w_down, dtype=np.float64).T) @ np.asarray(w_up, dtype=np.float64).T


def select_topk_qcal(g: Geometry, q, w_down, w_up, k_sum, b_sum):
    """select_topk on the calibrated query q^ = qcal(q, w_down, w_up)."""
    return select_topk(g, qcal(_f64(q, (g.B, g.Hq, g.T, g.d)), w_down, w_up), k_sum, b_sum)


def bsa_select_topk(g: Geometry, q, k):
    """Naive BSA (Sec. 2): exact log chunk masses M [B,Hq,T,Nc] (LSE over the chunk's token logits, for
    the row's candidates; NaN elsewhere) and the group top-k on them (same rule as select_topk), with
    its gap. Returns (idx, gap, mass)."""
    qq = _f64(q, (g.B, g.Hq, g.T, g.d))
    kk = _f64(k, (g.B, g.Hkv, g.L, g.d))
    idx = np.zeros((g.B, g.Hkv, g.T, g.topk), np.int32)
    gap = np.zeros((g.B, g.Hkv, g.T))
    mass = np.full((g.B, g.Hq, g.T, g.Nc), np.nan)
    _load().orc_bsa_select_topk(ctypes.byref(g._c()), _pd(qq), _pd(kk), _pi(idx), _pd(gap), _pd(mass))
    return idx, gap, mass


def attn_fwd(g: Geometry, q, k, v, q_hat, k_sum, b_sum, idx):
    """Eq. 10 (chunked form): out [B,Hq,T,d] and lse = log Z^ [B,Hq,T]."""
    q = _f64(q, (g.B, g.Hq, g.T, g.d))
    qh = _f64(q_hat, (g.B, g.Hq, g.T, g.d))
    k = _f64(k, (g.B, g.Hkv, g.L, g.d))
    v = _f64(v, (g.B, g.Hkv, g.L, g.d))
    ks = _f64(k_sum, (g.B, g.Hq, g.Nc, g.d))
    bs = _f64(b_sum, (g.B, g.Hq, g.Nc))
    ix = _i32(idx, (g.B, g.Hkv, g.T, g.topk))
    out = np.zeros((g.B, g.Hq, g.T, g.d))
    lse = np.zeros((g.B, g.Hq, g.T))
    _load().orc_attn_fwd(ctypes.byref(g._c()), _pd(q), _pd(k), _pd(v), _pd(qh), _pd(ks), _pd(bs), _pi(ix),
                         _pd(out), _pd(lse))
    return out, lse


def eq10_tokenwise(g: Geometry, q, k, v, q_hat, k_sum, b_sum, idx):
    """Eq. 10 weight by weight: (out [B,Hq,T,d], sum of weights [B,Hq,T]). No max subtraction."""
    q = _f64(q, (g.B, g.Hq, g.T, g.d))
    qh = _f64(q_hat, (g.B, g.Hq, g.T, g.d))
    k = _f64(k, (g.B, g.Hkv, g.L, g.d))
    v = _f64(v, (g.B, g.Hkv, g.L, g.d))
    ks = _f64(k_sum, (g.B, g.Hq, g.Nc, g.d))
    bs = _f64(b_sum, (g.B, g.Hq, g.Nc))
    ix = _i32(idx, (g.B, g.Hkv, g.T, g.topk))
    out = np.zeros((g.B, g.Hq, g.T, g.d))
    ws = np.zeros((g.B, g.Hq, g.T))
    _load().orc_eq10_tokenwise(ctypes.byref(g._c()), _pd(q), _pd(k), _pd(v), _pd(qh), _pd(ks), _pd(bs), _pi(ix),
                               _pd(out), _pd(ws))
    return out, ws


def attn_bwd(g: Geometry, q, k, v, q_hat, q_land, idx, dout):
    """Gradients of sum(dout * out) with idx fixed: (dq, dk, dv, dq_hat, dq_land)."""
    q = _f64(q, (g.B, g.Hq, g.T, g.d))
    qh = _f64(q_hat, (g.B, g.Hq, g.T, g.d))
    k = _f64(k, (g.B, g.Hkv, g.L, g.d))
    v = _f64(v, (g.B, g.Hkv, g.L, g.d))
    ql = _f64(q_land, (g.B, g.Hq, g.Nc, g.d))
    ix = _i32(idx, (g.B, g.Hkv, g.T, g.topk))
    do = _f64(dout, (g.B, g.Hq, g.T, g.d))
    dq = np.zeros_like(q)
    dqh = np.zeros_like(qh)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dql = np.zeros_like(ql)
    _load().orc_attn_bwd(ctypes.byref(g._c()), _pd(q), _pd(k), _pd(v), _pd(qh), _pd(ql), _pi(ix), _pd(do),
                         _pd(dq), _pd(dk), _pd(dv), _pd(dqh), _pd(dql))
    return dq, dk, dv, dqh, dql


def forward(g: Geometry, q, k, v, q_hat, q_land):
    """The whole prefill path: summaries, selection, attention. Returns a dict of every stage's output."""
    k_sum, b_sum = chunk_summary(g, k, q_land)
    idx, gap = select_topk(g, q_hat, k_sum, b_sum)
    out, lse = attn_fwd(g, q, k, v, q_hat, k_sum, b_sum, idx)
    return {"k_sum": k_sum, "b_sum": b_sum, "idx": idx, "gap": gap, "out": out, "lse": lse}


def decode(g: Geometry, q, q_hat, k_cache, v_cache, k_sum, b_sum):
    """One decode step: the query (T=1) sits at position L-1 of the cache. Returns (out, lse, idx, gap)."""
    assert g.T == 1 and g.q_pos0 == g.L - 1, "decode is one query row at the last cache position"
    idx, gap = select_topk(g, q_hat, k_sum, b_sum)
    out, lse = attn_fwd(g, q, k_cache, v_cache, q_hat, k_sum, b_sum, idx)
    return out, lse, idx, gap
