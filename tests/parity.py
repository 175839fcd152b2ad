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
# Rows whose k-th and (k+1)-th group scores differ by less than this are near ties: their ids are not
# compared one by one; the GPU's selection must instead be a valid top-k within this band (or the
# oracle's selection is fed to the GPU attention).
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


def group_scores(head_scores: np.ndarray, n: int) -> np.ndarray:
    """Group score of each of the n candidates of one row (Sec. 4 GQA rule, the oracle's reading):
    head_scores [G, >= n] per-head chunk scores; per head log-softmax over the candidates, max over heads."""
    s = np.asarray(head_scores, dtype=np.float64)[:, :n]
    m = s.max(1, keepdims=True)
    lse = m + np.log(np.exp(s - m).sum(1, keepdims=True))
    return (s - lse).max(0)


def retrieval_group_scores(g: Geometry, q_hat, k_sum, b_sum):
    """Function (b, kv_group, row) -> group scores of the row's candidates, from fp64 retrieval scores
    s^ = tau q^.k' + b' (Eq. 7) of the given summaries. q_hat [B,Hq,T,d], k_sum [B,Hq,Nc,d], b_sum [B,Hq,Nc]."""
    _, n = oracle.window(g)
    tau = g.tau()

    def f(b, grp, i):
        hs = slice(grp * g.G, (grp + 1) * g.G)
        nn = int(n[i])
        s = tau * np.einsum("hd,hcd->hc", q_hat[b, hs, i], k_sum[b, hs, :nn]) + b_sum[b, hs, :nn]
        return group_scores(s, nn)

    return f


def check_shat(shat: torch.Tensor, idx: torch.Tensor, g: Geometry, q_hat, k_sum, b_sum, what="shat",
               tol=dict(atol=1e-4, rtol=1e-4)):
    """Per-head retrieval scores of the selected ids (Eq. 7, fp64 on the given q^ and summaries): slot t of
    row (b, h, i) holds s^ of chunk idx[b, h/G, i, t], -inf where the id is -1."""
    sh, ix = np64(shat), idx.cpu().numpy()
    tau = g.tau()
    B, Hq, T, K = sh.shape
    hq = np.arange(Hq)
    if k_sum.shape[2] == 0:  # no chunk at all: every slot is -1 and scores -inf
        assert (ix == -1).all() and np.isneginf(sh).all(), f"{what}: slots without a chunk"
        return
    for b in range(B):
        ids = ix[b][hq // g.G]                       # [Hq, T, K]
        safe = np.where(ids >= 0, ids, 0)
        kk = k_sum[b][hq[:, None, None], safe]       # [Hq, T, K, d]
        ref = tau * np.einsum("htd,htkd->htk", q_hat[b], kk) + b_sum[b][hq[:, None, None], safe]
        ref = np.where(ids >= 0, ref, -np.inf)
        assert np.array_equal(np.isinf(sh[b]), np.isinf(ref)), f"{what}: -inf slots differ (b {b})"
        fin = np.isfinite(ref)
        np.testing.assert_allclose(sh[b][fin], ref[fin], err_msg=f"{what} (b {b})", **tol)


def mass_group_scores(g: Geometry, mass):
    """Function (b, kv_group, row) -> group scores from exact chunk masses [B,Hq,T,Nc] (naive BSA, Sec. 2)."""
    _, n = oracle.window(g)

    def f(b, grp, i):
        hs = slice(grp * g.G, (grp + 1) * g.G)
        return group_scores(mass[b, hs, i], int(n[i]))

    return f


def assert_valid_selection(row: np.ndarray, scores: np.ndarray, topk: int, what: str):
    """A GPU id row is a valid top-k of `scores` within the tie band: the min(topk, n) leading entries are
    distinct ascending candidates, the rest -1, and no selected candidate scores more than TIE_BAND below
    the k-th best score (so no left-out candidate beats a selected one by more than the band)."""
    n = len(scores)
    m = min(topk, n)
    ids = np.asarray(row[:m])
    assert (np.asarray(row[m:]) == -1).all(), f"{what}: padding is not -1: {row}"
    if m == 0:
        return
    assert ids.min() >= 0 and ids.max() < n, f"{what}: ids outside [0, {n}): {row}"
    assert (np.diff(ids) > 0).all(), f"{what}: ids not strictly ascending: {row}"
    kth = np.sort(scores)[::-1][m - 1]
    worst = scores[ids].min()
    assert worst >= kth - TIE_BAND, f"{what}: selected score {worst} below the k-th best {kth} by more than the band"


def check_idx(gpu_idx: torch.Tensor, ref_idx: np.ndarray, ref_gap: np.ndarray, what="idx", scores=None):
    """Bit-exact ids on every row outside the near-tie band; returns the near-tie row mask.
    With `scores` (a function (b, kv_group, row) -> group scores of that row's candidates, indexed like
    gpu_idx), every near-tie row is also checked to be a valid top-k within the band."""
    g = gpu_idx.cpu().numpy()
    near = ref_gap < TIE_BAND
    bad = (g != ref_idx).any(-1) & ~near
    if bad.any():
        where = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} rows differ outside the tie band, e.g. {where.tolist()}; "
                             f"gpu {g[tuple(where[0])]} oracle {ref_idx[tuple(where[0])]} gap "
                             f"{ref_gap[tuple(where[0])]}")
    if scores is not None:
        topk = g.shape[-1]
        for b, grp, i in np.argwhere(near):
            at = (int(b), int(grp), int(i))
            assert_valid_selection(g[b, grp, i], scores(*at), topk, f"{what} near-tie row {at}")
    return near


def splice(gpu_idx: torch.Tensor, ref_idx: np.ndarray, near: np.ndarray) -> torch.Tensor:
    out = gpu_idx.clone()
    if near.any():
        fixed = np.where(near[..., None], ref_idx, gpu_idx.cpu().numpy())
        out.copy_(torch.from_numpy(fixed.astype(np.int32)))
    return out
