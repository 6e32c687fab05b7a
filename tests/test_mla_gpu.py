"""GPU parity of the MLA decode (blasst_mla_decode) against the oracle's
MLA decode, through the C ABI.

The H query heads of a token score one shared latent row per key (d_qk =
576) and take its first 512 columns as value.  Checks outputs (max 2e-2 /
mean 2e-3), lse, masks [B, nk] bit-exact except near-ties, counters, the
statistics-only pass, fewer heads than the tile's 128 rows (down to one,
and a warp that mixes real and padding heads), ragged caches, automatic and
explicit split counts, and argument checks.
"""
import math

import numpy as np
import pytest
import torch

from oracle.mla import mla_decode
from synth import config_seed, planted_gap
from tests import _parity as P

pytestmark = pytest.mark.gpu
DQK, DV, BC = 576, 512, 64


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


def _inputs(B, H, L, seed):
    x = planted_gap(B, H, 1, 1, L, DQK, decode=True, block=BC, gap=8.0,
                    heavy_frac=0.05, seed=seed, device="cuda")
    return x.q, x.k[:, 0].contiguous()


MLA_CASES = [
    # B, H, L, ln_lambda, num_splits (0 = automatic)
    (2, 128, 1000, -3.0, 0),
    (1, 16, 777, -2.0, 3),       # 16 heads in a 128-row tile
    (2, 64, 2048, -math.inf, 4),
    (3, 128, 65, -1.0, 2),       # two blocks, the second holds one key
    (1, 128, 4096, -4.0, 0),
    (2, 32, 1500, 0.0, 5),
    (1, 1, 300, -2.0, 0),        # one head: 127 padding rows
    (2, 100, 2000, -3.0, 0),     # a warp of real and padding heads
]


@pytest.mark.parametrize("case", MLA_CASES)
def test_mla_decode_matches_oracle(blasst, case):
    m = blasst
    B, H, L, lnl, S_req = case
    q, cache = _inputs(B, H, L, config_seed(30, L + H))
    nk = -(-L // BC)
    S = S_req if S_req > 0 else m.blasst_mla_decode_splits(B, L)
    scale = 1.0 / math.sqrt(DQK)
    st = m.Stats(mask_numel=B * nk)
    o, lse = m.blasst_mla_decode(q, cache, scale=scale, ln_lambda=lnl,
                                 num_splits=S_req, stats=st)
    torch.cuda.synchronize()
    e, where = m.blasst_check_device_error()
    assert e == 0, f"device error word set (wait {where})"
    ref = mla_decode(q, cache, DV, scale, lnl, BC, S)
    P.check_out(P.to_np(o), ref["o"], "mla o")
    P.check_lse(P.to_np(lse), ref["lse"], "mla lse")
    mask = st.mask.cpu().numpy().reshape(B, nk)
    ties = P.check_mask(mask, ref["mask"], ref["margin"], "mla mask")
    vis, skp = st.read()
    assert vis == B * nk and skp == int((mask == 2).sum())
    if ties == 0:
        assert (vis, skp) == (ref["visited"], ref["skipped"])
    if lnl == -math.inf:
        assert skp == 0
    st2 = m.Stats(mask_numel=B * nk)
    r2 = m.blasst_mla_decode(q, cache, scale=scale, ln_lambda=lnl,
                             num_splits=S_req, stats=st2, stats_only=True)
    assert r2 == (None, None)
    assert torch.equal(st2.mask, st.mask) and st2.read() == (vis, skp)


def test_mla_rejects_bad_arguments(blasst):
    m = blasst
    q = torch.zeros(1, 129, DQK, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(1, 256, DQK, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BlasstError, match="UNSUPPORTED"):
        m.blasst_mla_decode(q, c)                       # 129 heads
    q = torch.zeros(1, 8, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BlasstError, match="UNSUPPORTED"):
        m.blasst_mla_decode(q, c[..., :512].contiguous())  # d_qk 512
    q = torch.zeros(1, 8, DQK, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BlasstError, match="INVALID_ARG"):
        m.blasst_mla_decode(q, c, num_splits=5)         # 4 blocks only
