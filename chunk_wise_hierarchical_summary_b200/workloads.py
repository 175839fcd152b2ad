"""Seeded synthetic inputs for the HiLS-Attention hot path.

This module holds workload definitions and random-number recipes only: none of the method's
arithmetic (summaries, scores, selection, attention) lives here. Both the CUDA path's tests and
benchmark and the fp64 oracle's checks draw their inputs from it, so the two see the same bytes.

Recipes (paper: "Hierarchical Sparse Attention Done Right: Toward Infinite Context Modeling"):
  tiny      q, k, v, q' (one landmark query per chunk) and q^ all i.i.d. N(0,1), drawn in that order.
  scaled    q, k, v ~ N(0,1) * d**-0.25 (so q.k/sqrt(d) has std 1/sqrt(d)); q' ~ N(0,1);
            q^ = q + W_up (W_down q) with W_down [32,d], W_up [d,32] i.i.d. N(0, 1/128), one pair
            shared by every head (the Sec. 4 low-rank query calibration with h_i := q_i).
  local     as scaled, but each head's q is a first-order autoregressive sequence along the positions,
            q_i = rho q_(i-1) + sqrt(1 - rho^2) e_i (e_i i.i.d. N(0,1), rho = 0.995), so adjacent queries
            are correlated and select overlapping chunks, the regime Sec. 4's query packing assumes.
  needle    decode cache: q, q' ~ N(0,1), q^ from q as above, K/V ~ N(0,1); 16 distinct candidate
            chunks per sequence hold "needle" keys 0.8*sqrt(d)*q^_h0/|q^_h0| + N(0, 0.2^2), h0 the
            first query head of each KV group.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    L: int
    Hq: int
    Hkv: int
    d: int
    S: int
    topk: int
    W: int
    dtype: str  # "fp32" or "bf16"
    recipe: str  # "tiny", "scaled", "local" or "needle"
    q_pos0: int = 0
    needles: int = 0
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def Nc(self) -> int:
        return self.L // self.S

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads the method is measured on.
TINY_FP32 = Workload("tiny_fp32_B1_T512_H2_d64_S32_k4_W64", B=1, T=512, L=512, Hq=2, Hkv=2, d=64, S=32, topk=4,
                     W=64, dtype="fp32", recipe="tiny")
PREFILL_BF16 = Workload("prefill_bf16_B4_T8192_Hq16_Hkv4_d128_S64_k16_W512", B=4, T=8192, L=8192, Hq=16, Hkv=4,
                        d=128, S=64, topk=16, W=512, dtype="bf16", recipe="scaled")
DECODE_BF16 = Workload("decode_bf16_B8_L524288_Hq32_Hkv8_d128_S64_k32_W512", B=8, T=1, L=524288, Hq=32, Hkv=8,
                       d=128, S=64, topk=32, W=512, dtype="bf16", recipe="needle", q_pos0=524287, needles=16)
DECODE_SWEEP_L = (32768, 131072, 524288, 1048576, 2097152, 4194304)
# The prefill shape with position-correlated queries (recipe "local"), for the attention's packing.
PREFILL_LOCAL_BF16 = Workload("prefill_local_bf16_B4_T8192_Hq16_Hkv4_d128_S64_k16_W512", B=4, T=8192, L=8192, Hq=16,
                              Hkv=4, d=128, S=64, topk=16, W=512, dtype="bf16", recipe="local")
TRAIN_BF16 = Workload("train_bf16_B2_T8192_Hq16_Hkv4_d128_S64_k16_W512", B=2, T=8192, L=8192, Hq=16, Hkv=4, d=128,
                      S=64, topk=16, W=512, dtype="bf16", recipe="scaled")


def decode_sweep(L: int) -> Workload:
    return DECODE_BF16.with_(name=f"decode_bf16_B1_L{L}_Hq32_Hkv8_d128_S64_k32_W512", B=1, L=L, q_pos0=L - 1)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device) -> torch.Tensor:
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32)


def _ar1_positions(e: torch.Tensor, rho: float) -> torch.Tensor:
    """x_i = rho x_(i-1) + sqrt(1 - rho^2) e_i along dim 2 (x_0 = e_0), as
    x_i = rho^i sum_(j<=i) rho^-j c_j e_j in float64 (c_0 = 1, c_j = sqrt(1 - rho^2))."""
    T = e.shape[2]
    j = torch.arange(T, device=e.device, dtype=torch.float64)
    c = torch.full((T,), math.sqrt(1.0 - rho * rho), device=e.device, dtype=torch.float64)
    c[0] = 1.0
    wgt = (rho ** -j) * c
    x = torch.cumsum(e.to(torch.float64) * wgt[None, None, :, None], dim=2) * (rho ** j)[None, None, :, None]
    return x.to(torch.float32)


def _qcal(q: torch.Tensor, d: int, g, device):
    """q^ = q + W_up (W_down q), rank 32, weights N(0, 1/128) (input recipe, upstream of the path).
    Returns (q^, W_down [32, d], W_up [d, 32])."""
    w_down = _randn((32, d), g, device) * math.sqrt(1.0 / 128.0)
    w_up = _randn((d, 32), g, device) * math.sqrt(1.0 / 128.0)
    return q + (q @ w_down.t()) @ w_up.t(), w_down, w_up


def prefill_inputs(w: Workload, seed: int = 0, device="cpu", with_dout: bool = False) -> dict:
    """q, q_hat [B,Hq,T,d]; k, v [B,Hkv,L,d]; q_land [B,Hq,Nc,d]; optional dout [B,Hq,T,d]; with the
    "scaled" and "local" recipes also the Q-Cal weights that made q_hat, w_down [32,d] and w_up [d,32]."""
    g = _gen(seed, device)
    B, T, L, Hq, Hkv, d, Nc = w.B, w.T, w.L, w.Hq, w.Hkv, w.d, w.Nc
    if w.recipe == "tiny":
        q = _randn((B, Hq, T, d), g, device)
        k = _randn((B, Hkv, L, d), g, device)
        v = _randn((B, Hkv, L, d), g, device)
        q_land = _randn((B, Hq, Nc, d), g, device)
        q_hat = _randn((B, Hq, T, d), g, device)
    elif w.recipe in ("scaled", "local"):
        s = d ** -0.25
        q = _randn((B, Hq, T, d), g, device)
        if w.recipe == "local":
            q = _ar1_positions(q, 0.995)
        q = q * s
        k = _randn((B, Hkv, L, d), g, device) * s
        v = _randn((B, Hkv, L, d), g, device) * s
        q_land = _randn((B, Hq, Nc, d), g, device)
        q_hat, w_down, w_up = _qcal(q, d, g, device)
    else:
        raise ValueError(f"prefill recipe {w.recipe!r}")
    out = {"q": q, "k": k, "v": v, "q_land": q_land, "q_hat": q_hat}
    if w.recipe in ("scaled", "local"):
        out.update(w_down=w_down, w_up=w_up)
    if with_dout:
        out["dout"] = _randn((B, Hq, T, d), g, device)
    return {name: t.to(w.torch_dtype).contiguous() for name, t in out.items()}


def decode_inputs(w: Workload, seed: int = 0, device="cpu") -> dict:
    """Needle-in-a-haystack decode cache for the last M = w.T positions (M = 1: plain decode; M > 1:
    multi-token decode). q, q_hat [B,Hq,M,d]; k_cache, v_cache [B,Hkv,L,d]; q_land [B,Hq,Nc,d];
    needle_chunks [B,needles] (int64, the planted chunk ids, candidates of the last query; the needle
    keys follow the first query token's q^).
    The cache is filled one sequence at a time so that only one fp32 slice is live at once."""
    assert 1 <= w.T and w.q_pos0 == w.L - w.T
    g = _gen(seed, device)
    B, L, Hq, Hkv, d, S, G = w.B, w.L, w.Hq, w.Hkv, w.d, w.S, w.G
    dt = w.torch_dtype
    q = _randn((B, Hq, w.T, d), g, device)
    q_land = _randn((B, Hq, w.Nc, d), g, device)
    q_hat, _, _ = _qcal(q, d, g, device)
    left = max(0, L - 1 - w.W + 1) // S * S
    n_cand = left // S
    n_needle = min(w.needles, n_cand)
    k = torch.empty((B, Hkv, L, d), dtype=dt, device=device)
    v = torch.empty((B, Hkv, L, d), dtype=dt, device=device)
    q0 = q_hat[:, ::G, 0, :]  # [B, Hkv, d]: the first query head of each group
    direction = q0 / q0.norm(dim=-1, keepdim=True)
    chunks = []
    for b in range(B):
        kb = _randn((Hkv, L, d), g, device)
        chosen = torch.randperm(n_cand, generator=g, device=device)[:n_needle]
        for c in chosen.tolist():
            noise = _randn((Hkv, S, d), g, device) * 0.2
            kb[:, c * S:(c + 1) * S, :] = 0.8 * math.sqrt(d) * direction[b][:, None, :] + noise
        k[b].copy_(kb)
        del kb
        v[b].copy_(_randn((Hkv, L, d), g, device))
        chunks.append(chosen)
    return {"q": q.to(dt).contiguous(), "q_hat": q_hat.to(dt).contiguous(), "k_cache": k, "v_cache": v,
            "q_land": q_land.to(dt).contiguous(), "needle_chunks": torch.stack(chunks)}
