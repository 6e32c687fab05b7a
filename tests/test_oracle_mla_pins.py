"""Pins of the oracle's MLA decode (CPU).

MLA decode with d_v = d_qk is plain decode with one KV head whose K and V
are the cache rows, so it must reproduce the C decode oracle (an
independent implementation: C loops there, numpy block products here) in
outputs, split partials, decisions and margins; the dense limit must be
float64 softmax attention over the whole cache with V = the latent part;
and with d_v < d_qk the decisions cannot depend on d_v (they use the full
score only).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle.mla import mla_decode
from synth import planted_gap


def _mla_inputs(B, H, L, dqk, seed):
    x = planted_gap(B, H, 1, 1, L, dqk, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=seed)
    return x.q, x.k[:, 0].contiguous()  # cache [B, L, d_qk]


@pytest.mark.parametrize("B,H,L,S,lnl", [(2, 8, 700, 3, -3.0),
                                         (1, 16, 512, 1, -2.0),
                                         (2, 4, 1000, 4, -math.inf)])
def test_mla_with_full_value_equals_decode(B, H, L, S, lnl):
    d = 64
    q, c = _mla_inputs(B, H, L, d, seed=960 + H)
    scale = 1.0 / math.sqrt(d)
    a = mla_decode(q, c, d, scale, lnl, 64, S)
    kv = c[:, None]  # one KV head: K = V = the cache rows
    r = oracle.decode(q, kv, kv, scale, lnl, 64, S)
    np.testing.assert_allclose(a["o"], r["o"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(a["lse"], r["lse"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(a["o_part"], r["o_part"], rtol=1e-11, atol=1e-13)
    np.testing.assert_array_equal(a["mask"], r["mask"][:, 0])
    fin = np.isfinite(r["margin"][:, 0])
    np.testing.assert_allclose(a["margin"][fin], r["margin"][:, 0][fin],
                               rtol=1e-9, atol=1e-9)
    assert (a["visited"], a["skipped"]) == (r["visited"], r["skipped"])


def test_mla_dense_limit_equals_softmax():
    B, H, L, dqk, dv = 2, 8, 640, 96, 64
    q, c = _mla_inputs(B, H, L, dqk, seed=970)
    scale = 0.1
    a = mla_decode(q, c, dv, scale, -math.inf, 64, 3)
    qd, cd = q.double().numpy(), c.double().numpy()
    for b in range(B):
        s = scale * (qd[b] @ cd[b].T)
        mx = s.max(axis=1, keepdims=True)
        p = np.exp(s - mx)
        o = (p @ cd[b][:, :dv]) / p.sum(axis=1, keepdims=True)
        np.testing.assert_allclose(a["o"][b], o, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(a["lse"][b], (mx + np.log(p.sum(1, keepdims=True)))[:, 0],
                                   rtol=1e-12, atol=1e-12)
    assert a["skipped"] == 0


def test_mla_decisions_do_not_depend_on_value_width():
    q, c = _mla_inputs(2, 8, 900, 96, seed=980)
    a = mla_decode(q, c, 64, 0.1, -2.5, 64, 2)
    b = mla_decode(q, c, 32, 0.1, -2.5, 64, 2)
    np.testing.assert_array_equal(a["mask"], b["mask"])
    np.testing.assert_allclose(a["lse"], b["lse"], rtol=1e-12)
    np.testing.assert_allclose(a["o"][..., :32], b["o"], rtol=1e-12, atol=1e-13)
    assert a["skipped"] > 0
