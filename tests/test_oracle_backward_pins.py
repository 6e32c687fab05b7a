"""Pins of the oracle's prefill backward (CPU).

The backward differentiates the forward with its skip decisions held fixed,
i.e. softmax attention restricted to the kept blocks.  Pinned by facts that
do not come from the oracle's own formulas:
  * central finite differences of an independent numpy forward (a masked
    softmax written in this file), for dense masks and for random kept /
    skipped block patterns, causal and not, with grouped heads;
  * the restricted forward equals the oracle's blockwise forward
    (``oracle.prefill``: its O and lse with the decisions it took), which is
    what makes that forward's gradient the restricted one;
  * grouped heads: dK and dV of a KV head are the sums of the per-head
    gradients of the same problem with the KV heads repeated.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import planted_gap


def _masked_attention(q, k, v, keep, scale):
    """One head, float64: O and lse of softmax(scale q k^T) over `keep`."""
    s = scale * (q @ k.T)
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    den = p.sum(axis=1, keepdims=True)
    return (p @ v) / den, (m + np.log(den))[:, 0]


def _keep(mask_h, Lq, Lkv, Br, Bc, causal):
    keep = np.zeros((Lq, Lkv), bool)
    for r in range(Lq):
        for c in range(Lkv):
            vis = (not causal) or c <= r + (Lkv - Lq)
            keep[r, c] = vis and mask_h[r // Br, c // Bc] == 1
    return keep


def _forward(q, k, v, mask, scale, causal, Br, Bc):
    B, Hq, Lq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.zeros(q.shape)
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        for h in range(Hq):
            keep = _keep(mask[b, h], Lq, Lkv, Br, Bc, causal)
            o[b, h], lse[b, h] = _masked_attention(q[b, h], k[b, h // G],
                                                   v[b, h // G], keep, scale)
    return o, lse


def _random_mask(rng, B, Hq, nq, nk, causal, p_skip):
    mask = np.where(rng.random((B, Hq, nq, nk)) < p_skip, 2, 1).astype(np.uint8)
    for i in range(nq):
        mask[:, :, i, i if causal else 0] = 1  # every row keeps a visible key
    return mask


@pytest.mark.parametrize("causal,p_skip,Hq,Hkv", [
    (True, 0.0, 2, 2), (True, 0.5, 4, 2), (False, 0.5, 2, 1),
    (False, 0.0, 4, 4), (True, 0.7, 4, 1)])
def test_backward_equals_finite_differences(causal, p_skip, Hq, Hkv):
    rng = np.random.default_rng(11 + int(10 * p_skip) + Hq)
    B, L, d, Br = 1, 96, 16, 32
    n = L // Br
    q = rng.standard_normal((B, Hq, L, d))
    k = rng.standard_normal((B, Hkv, L, d))
    v = rng.standard_normal((B, Hkv, L, d))
    w = rng.standard_normal((B, Hq, L, d))  # dO: the loss is sum(O * w)
    scale = 1.0 / math.sqrt(d)
    mask = _random_mask(rng, B, Hq, n, n, causal, p_skip)
    o, lse = _forward(q, k, v, mask, scale, causal, Br, Br)
    dq, dk, dv = oracle.prefill_backward(q, k, v, o, lse, w, mask, scale,
                                         causal, Br, Br)
    eps = 1e-5

    def loss(qq, kk, vv):
        oo, _ = _forward(qq, kk, vv, mask, scale, causal, Br, Br)
        return float((oo * w).sum())

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            idx = tuple(rng.integers(0, s) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd,
                                                                  g[idx])


@pytest.mark.parametrize("lnl,causal", [(-3.0, True), (-2.0, False),
                                        (-math.inf, True)])
def test_restricted_forward_equals_blockwise_forward(lnl, causal):
    Br = 64
    x = planted_gap(1, 4, 2, 320, 320, 64, block=Br, gap=8.0, heavy_frac=0.1,
                    window=64, seed=950)
    scale = 0.125
    res = oracle.prefill(x.q, x.k, x.v, scale, causal, lnl, Br, Br)
    nq = nk = 5
    mask = res["mask"].reshape(1, 4, nq, nk)
    if lnl > -math.inf:
        assert (mask == 2).any()
    o, lse = oracle.restricted_forward(x.q, x.k, x.v, mask, scale, causal, Br,
                                       Br)
    np.testing.assert_allclose(o.reshape(-1, Br, 64)[:, :, :],
                               res["o"][:, :Br], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1, Br), res["lse"][:, :Br],
                               rtol=1e-12, atol=1e-12)


def test_grouped_heads_sum_over_group():
    rng = np.random.default_rng(5)
    B, Hq, Hkv, L, d, Br = 1, 4, 2, 64, 16, 32
    q = rng.standard_normal((B, Hq, L, d))
    k = rng.standard_normal((B, Hkv, L, d))
    v = rng.standard_normal((B, Hkv, L, d))
    w = rng.standard_normal((B, Hq, L, d))
    mask = _random_mask(rng, B, Hq, 2, 2, True, 0.5)
    o, lse = _forward(q, k, v, mask, 0.25, True, Br, Br)
    dq, dk, dv = oracle.prefill_backward(q, k, v, o, lse, w, mask, 0.25, True,
                                         Br, Br)
    kr, vr = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    dq2, dk2, dv2 = oracle.prefill_backward(q, kr, vr, o, lse, w, mask, 0.25,
                                            True, Br, Br)
    np.testing.assert_allclose(dq, dq2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dk, dk2.reshape(B, Hkv, 2, L, d).sum(axis=2),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dv, dv2.reshape(B, Hkv, 2, L, d).sum(axis=2),
                               rtol=1e-12, atol=1e-12)
