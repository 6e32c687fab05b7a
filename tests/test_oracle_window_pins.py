"""Pins of the oracle's sliding-window forms (CPU).

The window is the attention variant in which query r attends only to the W
keys ending at its (bottom-right aligned) diagonal; decode attends to the
last W keys of the cache.  Each oracle function is checked against an
independent restatement: a whole-matrix numpy softmax under the window mask
(dense limit), the closed-form skip mask computed from the windowed block
maxima, plain causal attention when the window covers everything, and the
split partition of the visible blocks for decode.
"""
import math

import numpy as np
import pytest

import oracle
from synth import planted_gap
from tests import _brute as bf


@pytest.mark.parametrize("L,Lq,W,Br,Bc", [
    (300, 300, 64, 32, 32), (300, 300, 100, 64, 32), (512, 512, 200, 64, 64),
    (400, 250, 90, 32, 64), (256, 256, 1, 32, 32), (256, 256, 256, 64, 64)])
def test_window_dense_limit_equals_masked_softmax(L, Lq, W, Br, Bc):
    x = planted_gap(1, 4, 2, Lq, L, 32, block=32, gap=8.0, heavy_frac=0.1,
                    seed=700 + W)
    scale = 1.0 / math.sqrt(32)
    res = oracle.prefill(x.q, x.k, x.v, scale, True, -math.inf, Br, Bc,
                         window=W)
    qd, kd, vd = (bf.bf16_to_f64(t) for t in (x.q, x.k, x.v))
    vis = bf.window_visible(Lq, L, W)
    assert vis.any(axis=1).all()  # every query sees at least itself
    for u, (b, h, i) in enumerate(res["units"]):
        o_ref, lse_ref = bf.dense_masked(qd[b, h], kd[b, h // 2], vd[b, h // 2],
                                         scale, vis)
        r0, r1 = i * Br, min((i + 1) * Br, Lq)
        np.testing.assert_allclose(res["o"][u, :r1 - r0], o_ref[r0:r1],
                                   rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["lse"][u, :r1 - r0], lse_ref[r0:r1],
                                   rtol=1e-12, atol=1e-12)
    assert res["skipped"] == 0


def test_window_covering_everything_is_plain_causal():
    x = planted_gap(1, 4, 2, 384, 384, 64, block=64, gap=8.0, heavy_frac=0.1,
                    seed=711)
    a = oracle.prefill(x.q, x.k, x.v, 0.125, True, -4.0, 64, 64, window=384)
    b = oracle.prefill(x.q, x.k, x.v, 0.125, True, -4.0, 64, 64)
    for key in ("o", "lse", "mask"):
        np.testing.assert_array_equal(a[key], b[key])
    assert a["visited"] == b["visited"] and a["skipped"] == b["skipped"]


@pytest.mark.parametrize("ln_lambda", [-8.0, -4.0, -2.0])
@pytest.mark.parametrize("W", [96, 200])
def test_window_mask_equals_closed_form(ln_lambda, W):
    L, Br, Bc = 640, 64, 64
    x = planted_gap(1, 4, 2, L, L, 64, block=64, gap=8.0, heavy_frac=0.08,
                    window=128, seed=720)
    scale = 0.125
    res = oracle.prefill(x.q, x.k, x.v, scale, True, ln_lambda, Br, Bc,
                         window=W)
    qd, kd = bf.bf16_to_f64(x.q), bf.bf16_to_f64(x.k)
    vis = bf.window_visible(L, L, W)
    skipped = 0
    not_visited = 0
    for u, (b, h, i) in enumerate(res["units"]):
        s = np.where(vis, scale * (qd[b, h] @ kd[b, h // 2].T), -np.inf)
        mt = bf.block_row_max(s[i * Br:(i + 1) * Br], Bc)
        dec, D = bf.closed_form_decisions(mt, ln_lambda)
        close = np.abs(D - ln_lambda) < 1e-9
        assert np.array_equal(res["mask"][u][~close], dec[~close])
        skipped += int((res["mask"][u] == oracle.SKIPPED).sum())
        not_visited += int((dec == 0).sum())
    assert skipped == res["skipped"]
    assert not_visited > 0  # blocks left of every row's window exist


def test_prefill_window_rejected_without_causal():
    x = planted_gap(1, 2, 2, 128, 128, 32, block=32, seed=730)
    with pytest.raises(ValueError):
        oracle.prefill(x.q, x.k, x.v, 0.2, False, -4.0, 32, 32, window=64)
    with pytest.raises(ValueError):
        oracle.prefill(x.q, x.k, x.v, 0.2, True, -4.0, 32, 32, window=-1)


@pytest.mark.parametrize("Lkv,W,S", [(1000, 300, 1), (1000, 300, 3),
                                     (1000, 64, 2), (777, 500, 4),
                                     (1000, 5000, 3)])
def test_decode_window_dense_limit_and_splits(Lkv, W, S):
    x = planted_gap(2, 8, 2, 1, Lkv, 64, decode=True, block=64, gap=8.0,
                    heavy_frac=0.1, seed=740 + S)
    scale = 0.125
    Bc = 64
    res = oracle.decode(x.q, x.k, x.v, scale, -math.inf, Bc, S, window=W)
    qd, kd, vd = (bf.bf16_to_f64(t) for t in (x.q, x.k, x.v))
    lo = max(0, Lkv - W)
    o_ref, lse_ref = bf.dense_decode(qd, kd[:, :, lo:], vd[:, :, lo:], scale)
    np.testing.assert_allclose(res["o"], o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lse_ref, rtol=1e-12, atol=1e-12)
    nk = -(-Lkv // Bc)
    jlo = lo // Bc
    assert (res["mask"][:, :, :jlo] == oracle.NOT_VISITED).all()
    assert (res["mask"][:, :, jlo:] == oracle.KEPT).all()
    assert res["visited"] == 2 * 2 * (nk - jlo)
    # each split's partial is the dense result over its own key range
    for sp in range(S):
        j0 = jlo + oracle.split_begin(nk - jlo, S, sp)
        j1 = jlo + oracle.split_begin(nk - jlo, S, sp + 1)
        c0, c1 = max(j0 * Bc, lo), min(j1 * Bc, Lkv)
        if c1 <= c0:
            assert np.isneginf(res["lse_part"][:, :, sp]).all()
            continue
        op, lp = bf.dense_decode(qd, kd[:, :, c0:c1], vd[:, :, c0:c1], scale)
        np.testing.assert_allclose(res["o_part"][:, :, sp], op, rtol=1e-10,
                                   atol=1e-12)
        np.testing.assert_allclose(res["lse_part"][:, :, sp], lp, rtol=1e-12)


@pytest.mark.parametrize("ln_lambda", [-6.0, -2.0])
def test_decode_window_mask_closed_form(ln_lambda):
    Lkv, W, S, Bc = 1500, 700, 3, 64
    x = planted_gap(2, 8, 2, 1, Lkv, 64, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=750)
    scale = 0.125
    res = oracle.decode(x.q, x.k, x.v, scale, ln_lambda, Bc, S, window=W)
    qd, kd = bf.bf16_to_f64(x.q), bf.bf16_to_f64(x.k)
    lo = Lkv - W
    nk, jlo = -(-Lkv // Bc), (Lkv - W) // Bc
    for b in range(2):
        for h in range(2):
            s = scale * (qd[b, h * 4:(h + 1) * 4] @ kd[b, h].T)
            s[:, :lo] = -np.inf
            mt = bf.block_row_max(s, Bc)
            for sp in range(S):
                j0 = jlo + oracle.split_begin(nk - jlo, S, sp)
                j1 = jlo + oracle.split_begin(nk - jlo, S, sp + 1)
                dec, D = bf.closed_form_decisions(mt[:, j0:j1], ln_lambda)
                close = np.abs(D - ln_lambda) < 1e-9
                got = res["mask"][b, h, j0:j1]
                assert np.array_equal(got[~close], dec[~close])
    assert res["skipped"] > 0


def test_decode_window_covering_everything_is_plain_decode():
    x = planted_gap(2, 8, 2, 1, 640, 64, decode=True, block=64, seed=760)
    a = oracle.decode(x.q, x.k, x.v, 0.125, -3.0, 64, 3, window=640)
    b = oracle.decode(x.q, x.k, x.v, 0.125, -3.0, 64, 3)
    for key in ("o", "lse", "mask", "o_part", "lse_part"):
        np.testing.assert_array_equal(a[key], b[key])
