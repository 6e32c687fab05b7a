"""GPU parity of the tensor-core decode for wide head groups
(blasst_decode_wide: all G = Hq/Hkv heads of a KV head vote as one tile)
against the oracle's decode with the whole group as the tile, through the
C ABI.

Checks outputs (max 2e-2 / mean 2e-3), lse, masks [B, Hkv, nk] bit-exact
except near-ties, counters, the statistics-only pass, G = 4 .. 128 (MQA and
GQA), ragged caches, explicit and automatic splits, argument checks, and
an MQA cache of 32K keys on sampled sequences.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import config_seed, planted_gap, planted_gap_kv_inplace
from tests import _parity as P

pytestmark = pytest.mark.gpu
BC = 64


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


def _compare(m, q, k, v, lnl, S_req, bs=None):
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    nk = -(-L // BC)
    S = S_req if S_req > 0 else m.blasst_decode_wide_splits(B, Hkv, L)
    scale = 1.0 / math.sqrt(d)
    st = m.Stats(mask_numel=B * Hkv * nk)
    o, lse = m.blasst_decode_wide(q, k, v, scale=scale, ln_lambda=lnl,
                                  num_splits=S_req, stats=st)
    torch.cuda.synchronize()
    e, where = m.blasst_check_device_error()
    assert e == 0, f"device error word set (wait {where})"
    bsel = list(range(B)) if bs is None else bs
    ref = oracle.decode(q[bsel], k[bsel], v[bsel], scale, lnl, BC, S)
    P.check_out(P.to_np(o)[bsel], ref["o"], "wide decode o")
    P.check_lse(P.to_np(lse)[bsel], ref["lse"], "wide decode lse")
    mask = st.mask.cpu().numpy().reshape(B, Hkv, nk)
    ties = P.check_mask(mask[bsel], ref["mask"], ref["margin"],
                        "wide decode mask")
    vis, skp = st.read()
    assert vis == B * Hkv * nk and skp == int((mask == 2).sum())
    if bs is None:
        if ties == 0:
            assert (vis, skp) == (ref["visited"], ref["skipped"])
        st2 = m.Stats(mask_numel=B * Hkv * nk)
        r2 = m.blasst_decode_wide(q, k, v, scale=scale, ln_lambda=lnl,
                                  num_splits=S_req, stats=st2, stats_only=True)
        assert r2 == (None, None)
        assert torch.equal(st2.mask, st.mask) and st2.read() == (vis, skp)
    return mask


WIDE_CASES = [
    # B, Hq, Hkv, Lkv, ln_lambda, num_splits (0 = automatic)
    (2, 32, 1, 3000, -3.0, 0),     # MQA, 32 heads
    (3, 16, 1, 1000, -2.0, 3),
    (2, 64, 4, 2048, -4.0, 2),     # G = 16
    (1, 128, 1, 777, -3.0, 0),     # G = 128
    (2, 32, 1, 2048, -math.inf, 4),
    (2, 16, 1, 65, -1.0, 2),       # a block of one key
    (2, 8, 2, 1500, -3.0, 3),      # G = 4 also runs (padded rows)
]


@pytest.mark.parametrize("case", WIDE_CASES)
def test_wide_decode_matches_oracle(blasst, case):
    B, Hq, Hkv, L, lnl, S = case
    x = planted_gap(B, Hq, Hkv, 1, L, 128, decode=True, block=BC, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(40, L + Hq), device="cuda")
    mask = _compare(blasst, x.q, x.k, x.v, lnl, S)
    if lnl == -math.inf:
        assert (mask == 2).sum() == 0


def test_wide_rejects_bad_arguments(blasst):
    m = blasst
    q = torch.zeros(1, 129, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 256, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BlasstError, match="UNSUPPORTED"):
        m.blasst_decode_wide(q, k, k)                       # G = 129
    q = torch.zeros(1, 8, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 256, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BlasstError, match="UNSUPPORTED"):
        m.blasst_decode_wide(q, k, k)                       # d = 64


def test_wide_mqa_32k_sampled(blasst):
    """B 8, Hq 32, Hkv 1 (MQA), 32K keys, ln lambda -2: sequences 0, 7 (a
    32-head tile skips fewer blocks than a 4-head one)."""
    m = blasst
    B, Hq, Hkv, L, d = 8, 32, 1, 32768, 128
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=BC, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(40, 3))
    mask = _compare(m, q, k, v, -2.0, 0, bs=[0, 7])
    assert (mask == 2).mean() > 0.05
