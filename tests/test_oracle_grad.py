"""Pin the oracle's analytic backward against central finite differences in fp64 (no GPU).

The selection idx is held fixed (the hard top-k is not differentiable), so the loss
sum(dout * out) is a smooth function of q, k, v, q^ and the landmark queries q'.
"""
import numpy as np
import pytest

import oracle
from oracle import Geometry


def loss(g, x, idx, dout):
    ks, bs = oracle.chunk_summary(g, x["k"], x["q_land"])
    out, _ = oracle.attn_fwd(g, x["q"], x["k"], x["v"], x["q_hat"], ks, bs, idx)
    return float(np.sum(out * dout))


def make(g, seed, scale=0.6):
    r = np.random.default_rng(seed)
    x = dict(
        q=r.standard_normal((g.B, g.Hq, g.T, g.d)) * scale,
        k=r.standard_normal((g.B, g.Hkv, g.L, g.d)) * scale,
        v=r.standard_normal((g.B, g.Hkv, g.L, g.d)),
        q_hat=r.standard_normal((g.B, g.Hq, g.T, g.d)) * scale,
        q_land=r.standard_normal((g.B, g.Hq, g.Nc, g.d)) * scale,
    )
    ks, bs = oracle.chunk_summary(g, x["k"], x["q_land"])
    idx, _ = oracle.select_topk(g, x["q_hat"], ks, bs)
    dout = r.standard_normal((g.B, g.Hq, g.T, g.d))
    return x, idx, dout


NAMES = ("q", "k", "v", "q_hat", "q_land")


def test_grad_entrywise_tiny():
    """Every entry of every gradient against central differences (GQA, several chunks, a ragged tail)."""
    g = Geometry(B=1, T=30, L=30, Hq=4, Hkv=2, d=4, S=4, topk=2, W=5)
    x, idx, dout = make(g, 1)
    grads = dict(zip(NAMES, oracle.attn_bwd(g, x["q"], x["k"], x["v"], x["q_hat"], x["q_land"], idx, dout)))
    eps = 1e-5
    for name in NAMES:
        a = x[name]
        fd = np.zeros_like(a)
        it = np.nditer(a, flags=["multi_index"])
        for _ in it:
            mi = it.multi_index
            old = a[mi]
            a[mi] = old + eps
            lp = loss(g, x, idx, dout)
            a[mi] = old - eps
            lm = loss(g, x, idx, dout)
            a[mi] = old
            fd[mi] = (lp - lm) / (2 * eps)
        err = np.abs(fd - grads[name]).max() / max(1e-3, np.abs(fd).max())
        assert err < 1e-7, (name, err)
        assert np.abs(grads[name]).max() > 0, name  # every path is live at this geometry


@pytest.mark.parametrize("seed", [2, 3])
def test_grad_directional_c1_geometry(seed):
    """Directional derivatives at T = 512 with the tiny config's chunking (S = 32, W = 64, k = 4) plus GQA
    (Hq = 4, Hkv = 2), d = 64: <grad, u> against (L(x + eps u) - L(x - eps u)) / (2 eps) for a random u."""
    g = Geometry(B=1, T=512, L=512, Hq=4, Hkv=2, d=64, S=32, topk=4, W=64)
    x, idx, dout = make(g, seed, scale=0.5)
    grads = dict(zip(NAMES, oracle.attn_bwd(g, x["q"], x["k"], x["v"], x["q_hat"], x["q_land"], idx, dout)))
    r = np.random.default_rng(seed + 100)
    eps = 1e-5
    for name in NAMES:
        u = r.standard_normal(x[name].shape)
        base = x[name].copy()
        x[name] = base + eps * u
        lp = loss(g, x, idx, dout)
        x[name] = base - eps * u
        lm = loss(g, x, idx, dout)
        x[name] = base
        fd = (lp - lm) / (2 * eps)
        an = float(np.sum(grads[name] * u))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)
