"""GPU check of the decision margins the library reports
(blasst_skip_stats_t.margin): for every visited (tile, block) pair
max_r(m~_r - m_r) - ln lambda, +inf for a tile's first visited block.

Against the oracle's float64 margins: equal within 2e-3 (float32 scores of
128-term dot products), infinities in the same places; the mask is exactly
"skipped where the margin is < 0" (the sign of a float32 difference is the
sign of the comparison); the near-tie count (|margin| < 1e-3) agrees with
the oracle's up to the pairs whose margin is within the score error of
1e-3; and asking for margins changes no output bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import config_seed, paginate, planted_gap
from tests import _parity as P

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


def _compare(got_margin, got_mask, ref_margin, ref_mask, what):
    gm = np.asarray(got_margin, dtype=np.float64)
    visited = ref_mask > 0
    assert np.array_equal(got_mask > 0, visited), what
    g, r = gm[visited], np.asarray(ref_margin)[visited]
    assert np.array_equal(np.isposinf(g), np.isposinf(r)), what
    fin = np.isfinite(r)
    assert np.isfinite(g[fin]).all(), what
    if fin.any():
        err = np.abs(g[fin] - r[fin])
        assert err.max() <= TOL, (what, float(err.max()))
    # the decision is the sign of the margin
    assert np.array_equal(got_mask[visited] == 2, g < 0), what
    near_g = int((np.abs(g) < P.NEAR_TIE).sum())
    near_r = int((np.abs(r) < P.NEAR_TIE).sum())
    edge = int((np.abs(np.abs(r[fin]) - P.NEAR_TIE) < TOL).sum())
    assert abs(near_g - near_r) <= edge, (what, near_g, near_r, edge)
    return near_g


@pytest.mark.parametrize("d,T,L,lnl", [(128, 128, 1000, -3.0),
                                       (64, 64, 1024, -6.0),
                                       (128, 128, 700, -math.inf)])
def test_prefill_margins_match_oracle(blasst, d, T, L, lnl):
    m = blasst
    x = planted_gap(1, 4, 2, L, L, d, block=T, gap=8.0, heavy_frac=0.05,
                    window=256 if T == 128 else None,
                    seed=config_seed(0, 5150 + L + d), device="cuda")
    nq = nk = -(-L // T)
    st = m.Stats(mask_numel=4 * nq * nk, margin=True)
    o1, l1 = m.blasst_prefill(x.q, x.k, x.v, ln_lambda=lnl, Br=T, Bc=T,
                              stats=st)
    o2, l2 = m.blasst_prefill(x.q, x.k, x.v, ln_lambda=lnl, Br=T, Bc=T)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    ref = oracle.prefill(x.q, x.k, x.v, 1 / math.sqrt(d), True, lnl, T, T)
    got_m = st.margin.cpu().numpy().reshape(1, 4, nq, nk)
    got_k = st.mask.cpu().numpy().reshape(1, 4, nq, nk)
    gm = np.stack([got_m[b, h, i] for (b, h, i) in ref["units"]])
    gk = np.stack([got_k[b, h, i] for (b, h, i) in ref["units"]])
    near = _compare(gm, gk, ref["margin"], ref["mask"], f"prefill d{d}")
    assert near == st.near_ties()
    if lnl == -math.inf:
        assert np.isposinf(gm[gk > 0]).all()


@pytest.mark.parametrize("paged", [False, True])
def test_decode_margins_match_oracle(blasst, paged):
    m = blasst
    B, Hq, Hkv, L, S, lnl = 3, 16, 4, 3000, 3, -3.0
    x = planted_gap(B, Hq, Hkv, 1, L, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(1, 5151), device="cuda")
    nk = -(-L // 64)
    st = m.Stats(mask_numel=B * Hkv * nk, margin=True)
    if paged:
        pk = paginate(x.k, x.v, [L] * B, 16, seed=3, spare_pages=2)
        o1, _ = m.blasst_decode_paged(x.q, pk.k_pages, pk.v_pages,
                                      pk.block_table, pk.seq_lens,
                                      max_seq_len=L, ln_lambda=lnl,
                                      num_splits=S, stats=st)
    else:
        o1, _ = m.blasst_decode(x.q, x.k, x.v, ln_lambda=lnl, num_splits=S,
                                stats=st)
    o2, _ = m.blasst_decode(x.q, x.k, x.v, ln_lambda=lnl, num_splits=S)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    ref = oracle.decode(x.q, x.k, x.v, 1 / math.sqrt(128), lnl, 64, S)
    gm = st.margin.cpu().numpy().reshape(B, Hkv, nk)
    gk = st.mask.cpu().numpy().reshape(B, Hkv, nk)
    _compare(gm, gk, ref["margin"], ref["mask"], f"decode paged={paged}")
