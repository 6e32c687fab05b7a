"""Pins of the CPU oracle against facts that do not come from the oracle.

The pages print no worked numeric example, so the oracle is pinned by:
  * the dense limit: ln(lambda) = -inf skips nothing, so the result is plain
    softmax attention (float64 whole-matrix numpy, causal bottom-right,
    GQA, ragged tiles, Lq != Lkv);
  * closed forms on hand-sized inputs (single key, uniform scores, a
    two-block case computed by hand from the criterion);
  * an independent closed-form skip mask (prefix max of block maxima);
  * the skipped-mass bound implied by the criterion (every skipped score is
    more than |ln lambda| below its row's final max) and the resulting
    output-error bound;
  * monotonicity: the skip set at a smaller lambda is a subset of the skip
    set at a larger one;
  * split-KV + log-sum-exp merge equals the unsplit dense result.
Together these catch a dropped rescale factor, a flipped criterion, a wrong
causal offset, a transposed operand or a wrong GQA mapping.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import planted_gap
from tests import _brute as bf



def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


DENSE_CASES = [
    # B, Hq, Hkv, Lq, Lkv, d, causal, Br, Bc
    (1, 1, 1, 64, 64, 16, True, 16, 16),
    (1, 2, 2, 100, 100, 16, True, 32, 16),      # ragged tiles and blocks
    (2, 4, 2, 37, 91, 64, True, 16, 32),        # GQA, Lq < Lkv causal
    (1, 4, 1, 50, 130, 16, False, 32, 64),      # MQA, non-causal, ragged
    (1, 2, 1, 256, 256, 64, True, 64, 64),
    (1, 2, 2, 80, 80, 16, True, 64, 16),        # Br != Bc
]


@pytest.mark.parametrize("case", DENSE_CASES)
def test_dense_limit_equals_softmax(case):
    B, Hq, Hkv, Lq, Lkv, d, causal, Br, Bc = case
    q = _rand_bf16((B, Hq, Lq, d), 1, 1.5)
    k = _rand_bf16((B, Hkv, Lkv, d), 2, 1.5)
    v = _rand_bf16((B, Hkv, Lkv, d), 3)
    scale = 1.0 / math.sqrt(d)
    res = oracle.prefill(q, k, v, scale, causal, -math.inf, Br, Bc)
    o_ref, lse_ref = bf.dense_prefill(bf.bf16_to_f64(q), bf.bf16_to_f64(k),
                                      bf.bf16_to_f64(v), scale, causal)
    nq = -(-Lq // Br)
    for u, (b, h, i) in enumerate(res["units"]):
        r0, r1 = i * Br, min((i + 1) * Br, Lq)
        np.testing.assert_allclose(res["o"][u, :r1 - r0], o_ref[b, h, r0:r1],
                                   rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["lse"][u, :r1 - r0],
                                   lse_ref[b, h, r0:r1], rtol=1e-12, atol=1e-12)
    assert res["skipped"] == 0
    # visited pairs: every block with some visible key
    vis = bf.causal_visible(Lq, Lkv) if causal else np.ones((Lq, Lkv), bool)
    nk = -(-Lkv // Bc)
    expect = 0
    for i in range(nq):
        rows = vis[i * Br:min((i + 1) * Br, Lq)]
        for j in range(nk):
            if rows[:, j * Bc:(j + 1) * Bc].any():
                expect += 1
    assert res["visited"] == expect * B * Hq


def test_single_key_and_uniform_scores():
    # one key: the output is that key's value row, lse is its score
    q = _rand_bf16((1, 1, 1, 16), 5)
    k = _rand_bf16((1, 1, 1, 16), 6)
    v = _rand_bf16((1, 1, 1, 16), 7)
    res = oracle.prefill(q, k, v, 0.25, True, -3.0, 16, 16)
    np.testing.assert_array_equal(res["o"][0, 0], bf.bf16_to_f64(v)[0, 0, 0])
    s = 0.25 * float(bf.bf16_to_f64(q)[0, 0, 0] @ bf.bf16_to_f64(k)[0, 0, 0])
    assert res["lse"][0, 0] == pytest.approx(s, abs=1e-12)
    # zero query: uniform attention over the visible keys (non-causal)
    q0 = torch.zeros(1, 1, 3, 16, dtype=torch.bfloat16)
    k = _rand_bf16((1, 1, 40, 16), 8)
    v = _rand_bf16((1, 1, 40, 16), 9)
    res = oracle.prefill(q0, k, v, 0.25, False, -1.0, 16, 8)
    vm = bf.bf16_to_f64(v)[0, 0].mean(axis=0)
    for r in range(3):
        np.testing.assert_allclose(res["o"][0, r], vm, rtol=1e-12, atol=1e-13)
        assert res["lse"][0, r] == pytest.approx(math.log(40), abs=1e-12)
    # equal scores everywhere: no block is ever below the running max
    assert res["skipped"] == 0


def test_two_block_hand_case():
    """d=1, one query q=1, keys k=[2, 0] in blocks of one key, scale 1.
    Block 0 is the first visited block (never skipped).  Block 1 has
    m~ - m = 0 - 2 = -2: skipped iff -2 < ln(lambda)."""
    q = torch.tensor([[[[1.0]]]], dtype=torch.bfloat16)
    k = torch.tensor([[[[2.0], [0.0]]]], dtype=torch.bfloat16)
    v = torch.tensor([[[[3.0], [-5.0]]]], dtype=torch.bfloat16)
    # ln(lambda) = -1: -2 < -1, block 1 skipped -> o = v0, lse = 2
    r = oracle.prefill(q, k, v, 1.0, False, -1.0, 1, 1)
    assert r["mask"][0].tolist() == [oracle.KEPT, oracle.SKIPPED]
    assert r["o"][0, 0, 0] == 3.0 and r["lse"][0, 0] == pytest.approx(2.0)
    assert r["margin"][0, 1] == pytest.approx(-1.0)
    # ln(lambda) = -2: not strictly below -> kept; exact softmax of [2, 0]
    r = oracle.prefill(q, k, v, 1.0, False, -2.0, 1, 1)
    assert r["mask"][0].tolist() == [oracle.KEPT, oracle.KEPT]
    w = math.exp(2.0) / (math.exp(2.0) + 1.0)
    assert r["o"][0, 0, 0] == pytest.approx(3.0 * w - 5.0 * (1 - w), abs=1e-12)
    assert r["lse"][0, 0] == pytest.approx(math.log(math.exp(2) + 1), abs=1e-12)
    # reversed order: keys [0, 2]; block 1 raises the max, always kept, and
    # the first block's contribution is rescaled by exp(0 - 2)
    k2 = torch.tensor([[[[0.0], [2.0]]]], dtype=torch.bfloat16)
    v2 = torch.tensor([[[[-5.0], [3.0]]]], dtype=torch.bfloat16)
    r = oracle.prefill(q, k2, v2, 1.0, False, -0.5, 1, 1)
    assert r["mask"][0].tolist() == [oracle.KEPT, oracle.KEPT]
    assert r["o"][0, 0, 0] == pytest.approx(3.0 * w - 5.0 * (1 - w), abs=1e-12)


def _planted_small(seed, L=512, d=64, Hq=4, Hkv=2, window=None, block=64):
    x = planted_gap(1, Hq, Hkv, L, L, d, block=block, gap=8.0,
                    heavy_frac=0.05, window=window, seed=seed)
    return x.q, x.k, x.v


@pytest.mark.parametrize("ln_lambda", [-12.0, -6.0, -3.0, -1.0, 0.0])
@pytest.mark.parametrize("Br,Bc", [(64, 64), (32, 64), (64, 32)])
def test_mask_equals_closed_form(ln_lambda, Br, Bc):
    q, k, v = _planted_small(11, window=128)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d)
    res = oracle.prefill(q, k, v, scale, True, ln_lambda, Br, Bc)
    qd, kd = bf.bf16_to_f64(q), bf.bf16_to_f64(k)
    G = q.shape[1] // k.shape[1]
    skipped = 0
    for u, (b, h, i) in enumerate(res["units"]):
        s = bf.prefill_scores(qd, kd, scale, True, b, h, G)
        rows = s[i * Br:(i + 1) * Br]
        mt = bf.block_row_max(rows, Bc)
        dec, D = bf.closed_form_decisions(mt, ln_lambda)
        # exact equality except where the criterion is within rounding
        close = np.abs(D - ln_lambda) < 1e-9
        assert np.array_equal(res["mask"][u][~close], dec[~close])
        vis = dec > 0
        np.testing.assert_allclose(res["margin"][u][vis],
                                   D[vis] - ln_lambda, rtol=1e-9, atol=1e-9)
        skipped += int((res["mask"][u] == oracle.SKIPPED).sum())
    assert skipped == res["skipped"]
    if ln_lambda >= -6.0:
        assert res["skipped"] > 0  # the planted structure does produce skips


def test_skipped_mass_bound_and_error_bound():
    q, k, v = _planted_small(12, L=768, d=64, window=256)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d)
    Br = Bc = 64
    qd, kd, vd = bf.bf16_to_f64(q), bf.bf16_to_f64(k), bf.bf16_to_f64(v)
    G = q.shape[1] // k.shape[1]
    o_dense, _ = bf.dense_prefill(qd, kd, vd, scale, True)
    vmax = np.abs(vd).max()
    total_skipped = 0
    for ln_lambda in (-8.0, -4.0, -2.0):
        lam = math.exp(ln_lambda)
        res = oracle.prefill(q, k, v, scale, True, ln_lambda, Br, Bc)
        total_skipped += res["skipped"]
        for u, (b, h, i) in enumerate(res["units"]):
            s = bf.prefill_scores(qd, kd, scale, True, b, h, G)
            rows = s[i * Br:(i + 1) * Br]
            m_final = rows.max(axis=1, keepdims=True)
            p = np.exp(rows - m_final)          # dense weights, max 1 per row
            l_star = p.sum(axis=1)
            skipped_cols = np.zeros(rows.shape[1], bool)
            for j in np.nonzero(res["mask"][u] == oracle.SKIPPED)[0]:
                skipped_cols[j * Bc:(j + 1) * Bc] = True
                # every skipped weight is below lambda (relative to the max)
                assert np.all(p[:, j * Bc:(j + 1) * Bc] < lam)
            mass = p[:, skipped_cols].sum(axis=1)
            err = np.abs(res["o"][u, :rows.shape[0]]
                         - o_dense[b, h, i * Br:(i + 1) * Br]).max(axis=1)
            assert np.all(err <= 2 * vmax * mass / l_star + 1e-12)
            # a row's own maximum is never in a skipped block
            assert np.all(mass / l_star < 1.0)
    assert total_skipped > 0


def test_mask_monotone_in_lambda():
    q, k, v = _planted_small(13, L=640, window=128)
    scale = 1.0 / math.sqrt(q.shape[-1])
    prev = None
    prev_frac = -1.0
    for ln_lambda in (-math.inf, -14.0, -9.0, -6.0, -4.5, -3.0, -2.0, -1.0,
                      -0.5, 0.0):
        res = oracle.prefill(q, k, v, scale, True, ln_lambda, 64, 64)
        sk = res["mask"] == oracle.SKIPPED
        if prev is not None:
            assert np.all(sk[prev]), "a block skipped at smaller lambda is kept"
        frac = oracle.sparsity(res)
        assert frac >= prev_frac
        prev, prev_frac = sk, frac
    assert prev_frac > 0.3


@pytest.mark.parametrize("S", [1, 2, 3, 7])
def test_decode_split_merge_equals_dense(S):
    x = planted_gap(2, 8, 2, 1, 300, 64, decode=True, block=32, seed=21,
                    heavy_frac=0.1)
    scale = 1.0 / 8.0
    res = oracle.decode(x.q, x.k, x.v, scale, -math.inf, 32, S)
    o_ref, lse_ref = bf.dense_decode(bf.bf16_to_f64(x.q), bf.bf16_to_f64(x.k),
                                     bf.bf16_to_f64(x.v), scale)
    np.testing.assert_allclose(res["o"], o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lse_ref, rtol=1e-12, atol=1e-12)
    assert res["skipped"] == 0 and res["visited"] == 2 * 2 * 10


@pytest.mark.parametrize("S", [1, 4])
@pytest.mark.parametrize("ln_lambda", [-8.0, -3.0, 0.0])
def test_decode_mask_closed_form_per_split(S, ln_lambda):
    x = planted_gap(2, 8, 2, 1, 1000, 64, decode=True, block=64, seed=22,
                    heavy_frac=0.05)
    scale = 1.0 / 8.0
    Bc = 64
    res = oracle.decode(x.q, x.k, x.v, scale, ln_lambda, Bc, S)
    qd, kd = bf.bf16_to_f64(x.q), bf.bf16_to_f64(x.k)
    G = 4
    nk = -(-1000 // Bc)
    for b in range(2):
        for h in range(2):
            s = scale * (qd[b, h * G:(h + 1) * G] @ kd[b, h].T)  # [G, Lkv]
            mt = bf.block_row_max(s, Bc)
            for sp in range(S):
                j0 = oracle.split_begin(nk, S, sp)
                j1 = oracle.split_begin(nk, S, sp + 1)
                dec, D = bf.closed_form_decisions(mt[:, j0:j1], ln_lambda)
                close = np.abs(D - ln_lambda) < 1e-9
                got = res["mask"][b, h, j0:j1]
                assert np.array_equal(got[~close], dec[~close])
    # merged result against the merge of the per-split partials
    n = 2 * 8
    o, lse = oracle.combine(res["o_part"].reshape(n, S, -1),
                            res["lse_part"].reshape(n, S))
    np.testing.assert_allclose(o.reshape(res["o"].shape), res["o"], atol=0)


def test_combine_closed_form():
    rng = np.random.default_rng(3)
    op = rng.standard_normal((5, 3, 8))
    lp = rng.standard_normal((5, 3)) * 4
    lp[1, 2] = -np.inf  # an empty split contributes nothing
    o, lse = oracle.combine(op, lp)
    w = np.exp(lp - lp.max(axis=1, keepdims=True))
    ref_lse = np.log(w.sum(axis=1)) + lp.max(axis=1)
    ref_o = (w[..., None] * op).sum(axis=1) / w.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-13)
    np.testing.assert_allclose(o, ref_o, rtol=1e-12, atol=1e-14)


def test_first_block_never_skipped_and_sink_kept():
    q, k, v = _planted_small(14, L=512, window=None)
    scale = 1.0 / math.sqrt(q.shape[-1])
    res = oracle.prefill(q, k, v, scale, True, 0.0, 64, 64)
    assert np.all(res["mask"][:, 0] == oracle.KEPT)
    assert np.all(np.isinf(res["margin"][:, 0]))


def test_lambda_fit_recovers_inverse_law():
    a = 37.0
    Ls = [4096, 16384, 65536]
    lam = [a / L for L in Ls]
    assert oracle.lambda_fit(lam, Ls) == pytest.approx(a, rel=1e-12)


def test_rejects_positive_ln_lambda():
    q = _rand_bf16((1, 1, 4, 16), 1)
    with pytest.raises(ValueError):
        oracle.prefill(q, q, q, 0.25, True, 0.5, 16, 16)
