"""Pins of the oracle's decode with tiles of fewer query heads than a KV
head has (CPU): MQA (Hkv = 1) and GQA ratios above the decode tile's 8
rows, where the G query heads of a KV head are cut into G / T consecutive
tiles of T heads, each with its own skip vote.

The tiling has a plain definition (tile u of KV head h holds query heads
h*G + u*T .. h*G + (u+1)*T - 1 and reads KV head h), so it is pinned by
facts that do not come from the oracle's head repetition:
  * each tile's result is the plain decode of its T heads alone against
    its KV head (sliced inputs, the already-pinned decode), bit for bit;
  * dense limit: at ln(lambda) = -inf the result is float64 softmax
    attention (numpy);
  * T = G is the default decode exactly; the batched decision rule and the
    paged cache follow the same slicing identity.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import paginate, planted_gap
from tests import _brute as bf

Bc = 64


def _inputs(B, Hq, Hkv, L, d, seed):
    return planted_gap(B, Hq, Hkv, 1, L, d, decode=True, block=Bc, gap=8.0,
                       heavy_frac=0.05, seed=seed)


def _per_tile(fn, x, Hkv, G, T):
    """Runs fn(q_tile, k_head, v_head) for every tile: {(h, u): result}."""
    out = {}
    for h in range(Hkv):
        for u in range(G // T):
            h0 = h * G + u * T
            out[(h, u)] = fn(x.q[:, h0:h0 + T].contiguous(),
                             x.k[:, h:h + 1].contiguous(),
                             x.v[:, h:h + 1].contiguous())
    return out


@pytest.mark.parametrize("Hq,Hkv,T,L,S,lnl", [
    (32, 1, 8, 700, 3, -3.0),     # MQA, 4 tiles
    (16, 1, 8, 1000, 1, -2.0),
    (32, 2, 8, 640, 2, -4.0),     # G = 16: 2 tiles per KV head
    (8, 1, 2, 500, 2, -1.0),      # tiles of 2 heads
    (8, 2, 1, 300, 1, -2.5),      # a tile per head
])
def test_tiles_equal_sliced_decode(Hq, Hkv, T, L, S, lnl):
    B, d, G = 2, 64, Hq // Hkv
    x = _inputs(B, Hq, Hkv, L, d, seed=900 + Hq + T)
    scale = 1.0 / math.sqrt(d)
    res = oracle.decode(x.q, x.k, x.v, scale, lnl, Bc, S, tile_heads=T)
    parts = _per_tile(lambda q, k, v: oracle.decode(q, k, v, scale, lnl, Bc, S),
                      x, Hkv, G, T)
    nt = G // T
    assert res["mask"].shape == (B, Hkv * nt, -(-L // Bc))
    vis = skp = 0
    for (h, u), r in parts.items():
        h0 = h * G + u * T
        np.testing.assert_array_equal(res["o"][:, h0:h0 + T], r["o"])
        np.testing.assert_array_equal(res["lse"][:, h0:h0 + T], r["lse"])
        np.testing.assert_array_equal(res["o_part"][:, h0:h0 + T], r["o_part"])
        np.testing.assert_array_equal(res["mask"][:, h * nt + u], r["mask"][:, 0])
        np.testing.assert_array_equal(res["margin"][:, h * nt + u],
                                      r["margin"][:, 0])
        vis += r["visited"]
        skp += r["skipped"]
    assert (res["visited"], res["skipped"]) == (vis, skp)
    assert skp > 0


def test_tiles_dense_limit_equals_softmax():
    B, Hq, Hkv, L, d = 2, 32, 1, 777, 64
    x = _inputs(B, Hq, Hkv, L, d, seed=931)
    scale = 1.0 / math.sqrt(d)
    res = oracle.decode(x.q, x.k, x.v, scale, -math.inf, Bc, 4, tile_heads=8)
    o_ref, lse_ref = bf.dense_decode(*(bf.bf16_to_f64(t) for t in (x.q, x.k, x.v)),
                                     scale)
    np.testing.assert_allclose(res["o"], o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lse_ref, rtol=1e-12, atol=1e-12)
    assert res["skipped"] == 0 and res["visited"] == B * 4 * (-(-L // Bc))


def test_tile_of_whole_group_is_default():
    x = _inputs(2, 16, 2, 600, 64, seed=932)
    a = oracle.decode(x.q, x.k, x.v, 0.125, -3.0, Bc, 2, tile_heads=8)
    b = oracle.decode(x.q, x.k, x.v, 0.125, -3.0, Bc, 2)
    for key in ("o", "lse", "mask", "margin"):
        np.testing.assert_array_equal(a[key], b[key])


def test_tiles_batched_rule_equal_sliced():
    B, Hq, Hkv, L, d, S, lnl = 2, 16, 1, 900, 64, 2, -3.0
    x = _inputs(B, Hq, Hkv, L, d, seed=933)
    res = oracle.decode_batched(x.q, x.k, x.v, 0.125, lnl, Bc, S, 2,
                                tile_heads=8)
    parts = _per_tile(lambda q, k, v: oracle.decode_batched(q, k, v, 0.125, lnl,
                                                            Bc, S, 2),
                      x, Hkv, 16, 8)
    for (h, u), r in parts.items():
        np.testing.assert_array_equal(res["o"][:, 8 * u:8 * u + 8], r["o"])
        np.testing.assert_array_equal(res["mask"][:, u], r["mask"][:, 0])


def test_tiles_paged_equal_sliced():
    lens = [70, 300, 129]
    B, Hq, Hkv, d = len(lens), 16, 1, 64
    x = _inputs(B, Hq, Hkv, max(lens), d, seed=934)
    pk = paginate(x.k, x.v, lens, 16, seed=6, spare_pages=2,
                  poison=(3.0, 300.0))
    res = oracle.decode_paged(x.q, pk.k_pages, pk.v_pages, pk.block_table,
                              pk.seq_lens, 0.125, -2.5, 2, tile_heads=8)
    for u in range(2):
        r = oracle.decode_paged(x.q[:, 8 * u:8 * u + 8].contiguous(), pk.k_pages,
                                pk.v_pages, pk.block_table, pk.seq_lens, 0.125,
                                -2.5, 2)
        np.testing.assert_array_equal(res["o"][:, 8 * u:8 * u + 8], r["o"])
        np.testing.assert_array_equal(res["mask"][:, u], r["mask"][:, 0])


def test_tile_heads_must_divide_group():
    x = _inputs(1, 12, 1, 128, 64, seed=935)
    with pytest.raises(ValueError):
        oracle.decode(x.q, x.k, x.v, 0.125, -3.0, Bc, 1, tile_heads=8)
