"""Pins of the oracle's batched-decision decode (CPU).

The batched rule judges every block of a batch of k consecutive blocks
against the max over all earlier blocks and the whole batch.  Checked
against: the sequential oracle (k = 1 identical), the dense softmax
(ln lambda = -inf), a closed form computed from the block maxima alone,
the superset property (k > 1 skips every block the sequential rule skips),
and the bound on what a skipped block can contribute.
"""
import math

import numpy as np
import pytest

import oracle
from synth import planted_gap
from tests import _brute as bf


def _x(seed, B=2, Hq=8, Hkv=2, L=1500):
    return planted_gap(B, Hq, Hkv, 1, L, 64, decode=True, block=64, gap=8.0,
                       heavy_frac=0.05, seed=seed)


@pytest.mark.parametrize("S", [1, 3])
@pytest.mark.parametrize("ln_lambda", [-8.0, -3.0, 0.0])
def test_batch_one_is_sequential(S, ln_lambda):
    x = _x(800)
    a = oracle.decode_batched(x.q, x.k, x.v, 0.125, ln_lambda, 64, S, 1)
    b = oracle.decode(x.q, x.k, x.v, 0.125, ln_lambda, 64, S)
    for key in ("o", "lse", "mask", "o_part", "lse_part"):
        np.testing.assert_array_equal(a[key], b[key])
    assert (a["visited"], a["skipped"]) == (b["visited"], b["skipped"])


@pytest.mark.parametrize("k", [2, 3, 8])
def test_dense_limit(k):
    x = _x(801, L=1000)
    res = oracle.decode_batched(x.q, x.k, x.v, 0.125, -math.inf, 64, 3, k)
    o_ref, lse_ref = bf.dense_decode(bf.bf16_to_f64(x.q), bf.bf16_to_f64(x.k),
                                     bf.bf16_to_f64(x.v), 0.125)
    np.testing.assert_allclose(res["o"], o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lse_ref, rtol=1e-12, atol=1e-12)
    assert res["skipped"] == 0


def _closed_form_batched(mt, ln_lambda, k):
    """mt [R, n] block maxima of one split.  Decisions of the batched rule
    from the maxima alone: block j of batch [b0, b1) is skipped iff
    max_r(mt[r, j] - max(prefix max before b0, max over the batch)) <
    ln_lambda."""
    R, n = mt.shape
    dec = np.ones(n, np.uint8)
    D = np.zeros(n)
    prev = np.full(R, -np.inf)
    for b0 in range(0, n, k):
        b1 = min(b0 + k, n)
        Mb = np.maximum(prev, mt[:, b0:b1].max(axis=1))
        for j in range(b0, b1):
            D[j] = (mt[:, j] - Mb).max()
            dec[j] = 2 if D[j] < ln_lambda else 1
        prev = Mb
    return dec, D


@pytest.mark.parametrize("k", [2, 4])
@pytest.mark.parametrize("S", [1, 2])
@pytest.mark.parametrize("ln_lambda", [-6.0, -3.0, -1.0])
def test_mask_closed_form_and_superset(k, S, ln_lambda):
    L, Bc = 1500, 64
    x = _x(802, L=L)
    res = oracle.decode_batched(x.q, x.k, x.v, 0.125, ln_lambda, Bc, S, k)
    seq = oracle.decode(x.q, x.k, x.v, 0.125, ln_lambda, Bc, S)
    qd, kd = bf.bf16_to_f64(x.q), bf.bf16_to_f64(x.k)
    nk = -(-L // Bc)
    for b in range(2):
        for h in range(2):
            s = 0.125 * (qd[b, h * 4:(h + 1) * 4] @ kd[b, h].T)
            mt = bf.block_row_max(s, Bc)
            for sp in range(S):
                j0 = oracle.split_begin(nk, S, sp)
                j1 = oracle.split_begin(nk, S, sp + 1)
                dec, D = _closed_form_batched(mt[:, j0:j1], ln_lambda, k)
                close = np.abs(D - ln_lambda) < 1e-9
                got = res["mask"][b, h, j0:j1]
                assert np.array_equal(got[~close], dec[~close])
    # every block the sequential rule skips is skipped by the batched rule
    assert ((seq["mask"] == 2) <= (res["mask"] == 2)).all()
    assert res["skipped"] >= seq["skipped"]


def test_batched_skips_more_and_stays_bounded():
    L, Bc, S, k, lnl = 2000, 64, 2, 4, -4.0
    x = _x(803, L=L)
    res = oracle.decode_batched(x.q, x.k, x.v, 0.125, lnl, Bc, S, k)
    seq = oracle.decode(x.q, x.k, x.v, 0.125, lnl, Bc, S)
    assert res["skipped"] > seq["skipped"]  # the look-ahead finds more
    # each skipped block's weights are below lambda relative to the split's
    # final max: exp(s - m_final) < lambda for every entry of the block
    qd, kd = bf.bf16_to_f64(x.q), bf.bf16_to_f64(x.k)
    nk = -(-L // Bc)
    for b in range(2):
        for h in range(2):
            s = 0.125 * (qd[b, h * 4:(h + 1) * 4] @ kd[b, h].T)
            for sp in range(S):
                j0 = oracle.split_begin(nk, S, sp)
                j1 = oracle.split_begin(nk, S, sp + 1)
                c1 = min(j1 * Bc, L)
                m_final = s[:, j0 * Bc:c1].max(axis=1, keepdims=True)
                for j in range(j0, j1):
                    if res["mask"][b, h, j] == 2:
                        blk = s[:, j * Bc:min((j + 1) * Bc, L)]
                        assert (np.exp(blk - m_final) < math.exp(lnl)).all()
    # and the output error stays within the sequential rule's kind of bound
    dense = oracle.decode(x.q, x.k, x.v, 0.125, -math.inf, Bc, S)
    assert np.abs(res["o"] - dense["o"]).max() < 0.1
