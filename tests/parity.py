"""Shared helpers for the GPU-vs-oracle parity tests (imported by tests only)."""
import numpy as np
import torch

import oracle
from oracle import Geometry
from chunk_wise_hierarchical_summary_b200 import workloads as W

# Tolerances of the method's spec: |x - y| <= atol + rtol * |y|.
TOL = {"bf16": dict(atol=2e-2, rtol=1e-2), "fp32": dict(atol=1e-4, rtol=1e-4)}
# b_sum is fp32 arithmetic on exactly representable inputs in both modes.
BSUM_TOL = dict(atol=1e-4, rtol=1e-4)
# Rows whose k-th and (k+1)-th group scores differ by less than this are near ties: the oracle's
# selection is fed to the GPU attention instead of comparing ids.
TIE_BAND = 1e-3


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy() if t.is_floating_point() else t.detach().cpu().numpy()


def geometry(w: W.Workload, **kw) -> Geometry:
    g = dict(B=w.B, T=w.T, L=w.L, Hq=w.Hq, Hkv=w.Hkv, d=w.d, S=w.S, topk=w.topk, W=w.W, q_pos0=w.q_pos0)
    g.update(kw)
    return Geometry(**g)


def assert_close(gpu, ref, tol, what):
    a = np64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    np.testing.assert_allclose(a, ref, err_msg=what, **tol)


def check_idx(gpu_idx: torch.Tensor, ref_idx: np.ndarray, ref_gap: np.ndarray, what="idx"):
    """Bit-exact ids on every row outside the near-tie band; returns the near-tie row mask."""
    g = gpu_idx.cpu().numpy()
    near = ref_gap < TIE_BAND
    bad = (g != ref_idx).any(-1) & ~near
    if bad.any():
        where = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} rows differ outside the tie band, e.g. {where.tolist()}; "
                             f"gpu {g[tuple(where[0])]} oracle {ref_idx[tuple(where[0])]} gap "
                             f"{ref_gap[tuple(where[0])]}")
    return near


def splice(gpu_idx: torch.Tensor, ref_idx: np.ndarray, near: np.ndarray) -> torch.Tensor:
    out = gpu_idx.clone()
    if near.any():
        fixed = np.where(near[..., None], ref_idx, gpu_idx.cpu().numpy())
        out.copy_(torch.from_numpy(fixed.astype(np.int32)))
    return out
