"""Pins of the paged, variable-length decode oracle.

The page indirection has a plain definition (token t of sequence b lives in
page block_table[b][t // page_size], row t % page_size), so it is pinned by
facts that do not come from the oracle's gather:
  * dense limit: at ln(lambda) = -inf the result is float64 softmax attention
    over each sequence's own logical tokens (numpy, from the logical arrays
    the test scattered into the pool, never from the pool);
  * invariance: two different physical placements of the same logical
    caches, with different poison in every pool row no sequence owns, give
    bit-identical results -- so no unowned row and no wrong page is read;
  * the closed-form skip mask of each sequence's own blocks and splits;
  * lambda = a / L per sequence: on a batch, each sequence's result is the
    one it gets alone with ln lambda = min(0, ln a - ln L_b);
  * empty sequences and splits with no blocks.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import paginate, planted_gap
from tests import _brute as bf

Bc = 64


def _logical(B, Hq, Hkv, Lmax, d, seed):
    x = planted_gap(B, Hq, Hkv, 1, Lmax, d, decode=True, block=Bc, gap=8.0,
                    heavy_frac=0.05, seed=seed)
    return x.q, x.k, x.v


LENS = [1, 63, 64, 65, 200, 130]


@pytest.mark.parametrize("page_size", [16, 64, 128])
@pytest.mark.parametrize("S", [1, 3])
def test_paged_dense_limit_equals_softmax(page_size, S):
    B, Hq, Hkv, d = len(LENS), 4, 2, 32
    q, k, v = _logical(B, Hq, Hkv, max(LENS), d, 31)
    pk = paginate(k, v, LENS, page_size, seed=5, spare_pages=3,
                  poison=(4.0, 500.0))
    scale = 1.0 / math.sqrt(d)
    res = oracle.decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                              pk.seq_lens, scale, -math.inf, S)
    qd, kd, vd = bf.bf16_to_f64(q), bf.bf16_to_f64(k), bf.bf16_to_f64(v)
    for b, L in enumerate(LENS):
        o_ref, lse_ref = bf.dense_decode(qd[b:b + 1], kd[b:b + 1, :, :L],
                                         vd[b:b + 1, :, :L], scale)
        np.testing.assert_allclose(res["o"][b], o_ref[0], rtol=1e-10,
                                   atol=1e-12)
        np.testing.assert_allclose(res["lse"][b], lse_ref[0], rtol=1e-12,
                                   atol=1e-12)
    nk = [-(-L // Bc) for L in LENS]
    assert res["skipped"] == 0 and res["visited"] == Hkv * sum(nk)


def test_paged_placement_and_poison_invariance():
    B, Hq, Hkv, d = len(LENS), 8, 2, 64
    q, k, v = _logical(B, Hq, Hkv, max(LENS), d, 32)
    scale = 1.0 / 8.0
    runs = []
    for seed, poison, ps in [(1, (6.0, 900.0), 16), (2, (-6.0, -900.0), 16),
                             (3, (0.5, 3.0), 16)]:
        pk = paginate(k, v, LENS, ps, seed=seed, spare_pages=5, poison=poison)
        runs.append(oracle.decode_paged(q, pk.k_pages, pk.v_pages,
                                        pk.block_table, pk.seq_lens, scale,
                                        -2.0, 2))
    for r in runs[1:]:
        for key in ("o", "lse", "mask", "o_part", "lse_part"):
            assert np.array_equal(r[key], runs[0][key]), key
        assert (r["visited"], r["skipped"]) == (runs[0]["visited"],
                                                runs[0]["skipped"])
    # an interleaved pool (K and V pages of one pool, page stride 2x) holds the
    # same logical tokens
    pk = paginate(k, v, LENS, 16, seed=4, poison=(1.0, 1.0))
    P = pk.num_pages
    pool = torch.stack([pk.k_pages, pk.v_pages], dim=1).contiguous()
    flat = pool.view(-1)
    per = Hkv * 16 * d
    r = oracle.decode_paged(q, (flat, P, Hkv, 16, d), (flat[per:], P, Hkv, 16, d),
                            pk.block_table, pk.seq_lens, scale, -2.0, 2,
                            page_stride=2 * per)
    for key in ("o", "lse", "mask"):
        assert np.array_equal(r[key], runs[0][key]), key


@pytest.mark.parametrize("S", [1, 2])
@pytest.mark.parametrize("ln_lambda", [-6.0, -2.0, 0.0])
def test_paged_mask_closed_form(S, ln_lambda):
    lens = [700, 65, 1000, 128]
    B, Hq, Hkv, d = len(lens), 8, 2, 64
    q, k, v = _logical(B, Hq, Hkv, max(lens), d, 33)
    pk = paginate(k, v, lens, 32, seed=7, spare_pages=2, poison=(3.0, 50.0))
    scale = 1.0 / 8.0
    res = oracle.decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                              pk.seq_lens, scale, ln_lambda, S)
    qd, kd = bf.bf16_to_f64(q), bf.bf16_to_f64(k)
    G = Hq // Hkv
    nk_max = res["mask"].shape[2]
    vis = skp = 0
    for b, L in enumerate(lens):
        nk = -(-L // Bc)
        for h in range(Hkv):
            s = scale * (qd[b, h * G:(h + 1) * G] @ kd[b, h, :L].T)
            mt = bf.block_row_max(s, Bc)
            for sp in range(S):
                j0, j1 = (sp * nk) // S, ((sp + 1) * nk) // S
                dec, D = bf.closed_form_decisions(mt[:, j0:j1], ln_lambda)
                close = np.abs(D - ln_lambda) < 1e-9
                got = res["mask"][b, h, j0:j1]
                assert np.array_equal(got[~close], dec[~close])
                vis += j1 - j0
                skp += int(np.sum(dec == 2))
            assert np.all(res["mask"][b, h, nk:nk_max] == oracle.NOT_VISITED)
    assert res["visited"] == vis and abs(res["skipped"] - skp) <= 2
    assert res["skipped"] > 0 or ln_lambda < -5


def test_paged_per_length_threshold():
    lens = [900, 300, 64, 2000]
    B, Hq, Hkv, d = len(lens), 4, 1, 64
    q, k, v = _logical(B, Hq, Hkv, max(lens), d, 34)
    pk = paginate(k, v, lens, 64, seed=8, poison=(2.0, 40.0))
    scale = 1.0 / 8.0
    ln_a = math.log(100.0)  # lambda = 100 / L; clamps to 1 for L = 64
    res = oracle.decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                              pk.seq_lens, scale, ln_a, 2, per_length=True)
    for b, L in enumerate(lens):
        lnl = min(0.0, ln_a - math.log(L))
        one = oracle.decode(q[b:b + 1], k[b:b + 1, :, :L], v[b:b + 1, :, :L],
                            scale, lnl, Bc, 2)
        np.testing.assert_array_equal(res["o"][b], one["o"][0])
        np.testing.assert_array_equal(res["lse"][b], one["lse"][0])
        nk = -(-L // Bc)
        np.testing.assert_array_equal(res["mask"][b, :, :nk], one["mask"][0])
    # fixed threshold: the argument is ln lambda itself for every sequence
    fixed = oracle.decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                                pk.seq_lens, scale, -1.5, 2)
    one = oracle.decode(q[3:4], k[3:4, :, :2000], v[3:4, :, :2000], scale,
                        -1.5, Bc, 2)
    np.testing.assert_array_equal(fixed["o"][3], one["o"][0])


def test_paged_empty_sequence_and_empty_splits():
    lens = [0, 10, 64, 0]
    B, Hq, Hkv, d = len(lens), 2, 1, 32
    q, k, v = _logical(B, Hq, Hkv, 64, d, 35)
    pk = paginate(k, v, lens, 16, seed=9, spare_pages=1, poison=(5.0, 70.0))
    scale = 1.0 / math.sqrt(d)
    res = oracle.decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                              pk.seq_lens, scale, -1.0, 4)
    for b in (0, 3):
        assert np.all(res["o"][b] == 0.0) and np.all(np.isneginf(res["lse"][b]))
        assert np.all(res["mask"][b] == oracle.NOT_VISITED)
    # one block, four splits: three splits are empty and change nothing
    qd, kd, vd = bf.bf16_to_f64(q), bf.bf16_to_f64(k), bf.bf16_to_f64(v)
    for b in (1, 2):
        L = lens[b]
        o_ref, lse_ref = bf.dense_decode(qd[b:b + 1], kd[b:b + 1, :, :L],
                                         vd[b:b + 1, :, :L], scale)
        np.testing.assert_allclose(res["o"][b], o_ref[0], rtol=1e-10,
                                   atol=1e-12)
        assert np.sum(np.isneginf(res["lse_part"][b])) == 3 * Hq
    assert res["visited"] == 2 and res["skipped"] == 0


def test_paged_rejects_bad_tables():
    lens = [100]
    q, k, v = _logical(1, 2, 1, 128, 32, 36)
    pk = paginate(k, v, lens, 64, seed=1)
    bt = pk.block_table.clone()
    bt[0, 1] = pk.num_pages  # out of the pool
    with pytest.raises(ValueError):
        oracle.decode_paged(q, pk.k_pages, pk.v_pages, bt, pk.seq_lens, 0.2,
                            -1.0, 1)
    with pytest.raises(ValueError):  # longer than the table can hold
        oracle.decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                            torch.tensor([300], dtype=torch.int32), 0.2, -1.0,
                            1)
