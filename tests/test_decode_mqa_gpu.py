"""GPU parity of decode with more than 8 query heads per KV head (MQA with
many heads, GQA 16:1 and 32:1) against the CPU oracle, through the C ABI.

The decode tile holds at most 8 query heads: for G = Hq/Hkv = 16, 32, 64
the heads of a KV head are cut into G/8 consecutive tiles with their own
skip decisions (the oracle's ``tile_heads=8``).  blasst_decode and
blasst_decode_window run these tiles on the tensor-core kernel (one CTA for
all tiles of a KV head); the batched rule and the paged cache run them on
the CUDA-core kernel (one CTA per tile).  Checks outputs (max 2e-2 / mean
2e-3), lse, masks [B, Hkv*G/8, nk] bit-exact except near-ties, counters,
the statistics-only pass, the sliding window, the batched decision rule,
the paged cache against both contiguous kernels, a full-size MQA sample,
and that a group that is not a power of two is refused.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import config_seed, paginate, planted_gap, planted_gap_kv_inplace
from tests import _parity as P

pytestmark = pytest.mark.gpu
Bc = 64


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


def _tiles(Hq, Hkv):
    G = Hq // Hkv
    return G // 8 if G > 8 else 1


def _compare(m, x, ln_lambda, S_req, window=0, batch=1, bs=None):
    q, k, v = x.q, x.k, x.v
    B, Hq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    T = _tiles(Hq, Hkv)
    nk = -(-Lkv // Bc)
    jlo = (Lkv - window) // Bc if 0 < window < Lkv else 0
    if S_req > 0:
        S = S_req
    elif batch == 2:  # the batched rule keeps the GQA policy
        S = m.blasst_decode_splits(B, Hkv, Lkv - jlo * Bc)
    else:
        S = m.blasst_decode_group_splits(B, Hq, Hkv, Lkv - jlo * Bc)
    scale = 1.0 / math.sqrt(d)
    stats = m.Stats(mask_numel=B * Hkv * T * nk)

    def call(st, stats_only=False):
        if batch == 2:
            return m.blasst_decode_batched(q, k, v, batch=2, scale=scale,
                                           ln_lambda=ln_lambda,
                                           num_splits=S_req, stats=st,
                                           stats_only=stats_only)
        return m.blasst_decode_window(q, k, v, window=window, scale=scale,
                                      ln_lambda=ln_lambda, num_splits=S_req,
                                      stats=st, stats_only=stats_only)

    o, lse = call(stats)
    torch.cuda.synchronize()
    st, where = m.blasst_check_device_error()
    assert st == 0, f"device error word set (wait {where})"
    bsel = list(range(B)) if bs is None else bs
    qs, ks, vs = q[bsel], k[bsel], v[bsel]
    if batch == 2:
        ref = oracle.decode_batched(qs, ks, vs, scale, ln_lambda, Bc, S, 2,
                                    tile_heads=min(8, Hq // Hkv))
    else:
        ref = oracle.decode(qs, ks, vs, scale, ln_lambda, Bc, S, window=window,
                            tile_heads=min(8, Hq // Hkv))
    P.check_out(P.to_np(o)[bsel], ref["o"], "mqa decode o")
    P.check_lse(P.to_np(lse)[bsel], ref["lse"], "mqa decode lse")
    mask = stats.mask.cpu().numpy().reshape(B, Hkv * T, nk)
    ties = P.check_mask(mask[bsel], ref["mask"], ref["margin"],
                        "mqa decode mask")
    vis, skp = stats.read()
    assert vis == B * Hkv * T * (nk - jlo)
    assert skp == int((mask == 2).sum())
    if bs is None and ties == 0:
        assert (vis, skp) == (ref["visited"], ref["skipped"])
    if bs is None:
        st2 = m.Stats(mask_numel=B * Hkv * T * nk)
        assert call(st2, stats_only=True) == (None, None)
        assert torch.equal(st2.mask, stats.mask)
        assert st2.read() == (vis, skp)
    return mask, ref


MQA_CASES = [
    # B, Hq, Hkv, Lkv, ln_lambda, num_splits (0 = automatic)
    (2, 32, 1, 3000, -3.0, 0),
    (3, 16, 1, 1000, -2.0, 3),
    (2, 64, 4, 2048, -4.0, 2),      # G = 16
    (1, 64, 1, 777, -3.0, 0),       # G = 64: 8 tiles
    (2, 32, 1, 2048, -math.inf, 4),
    (2, 16, 1, 65, -1.0, 2),
]


@pytest.mark.parametrize("case", MQA_CASES)
def test_mqa_decode_matches_oracle(blasst, case):
    B, Hq, Hkv, Lkv, ln_lambda, S = case
    x = planted_gap(B, Hq, Hkv, 1, Lkv, 128, decode=True, block=Bc, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(10, Lkv + Hq), device="cuda")
    mask, _ = _compare(blasst, x, ln_lambda, S)
    if ln_lambda == -math.inf:
        assert (mask == 2).sum() == 0


def test_mqa_window_and_batched(blasst):
    x = planted_gap(2, 32, 1, 1, 3000, 128, decode=True, block=Bc, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(10, 1), device="cuda")
    _compare(blasst, x, -3.0, 0, window=1000)
    _compare(blasst, x, -3.0, 3, batch=2)


def test_mqa_paged_equals_contiguous(blasst):
    m = blasst
    B, Hq, Hkv, L = 2, 32, 1, 1500
    x = planted_gap(B, Hq, Hkv, 1, L, 128, decode=True, block=Bc, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(10, 2), device="cuda")
    nk = -(-L // Bc)
    s1, s2 = m.Stats(mask_numel=B * 4 * nk), m.Stats(mask_numel=B * 4 * nk)
    # the CUDA-core kernel on the contiguous cache (batch 1 = sequential rule)
    o1, l1 = m.blasst_decode_batched(x.q, x.k, x.v, batch=1, ln_lambda=-3.0,
                                     num_splits=3, stats=s1)
    pk = paginate(x.k, x.v, [L] * B, 64, seed=4, spare_pages=3)
    o2, l2 = m.blasst_decode_paged(x.q, pk.k_pages, pk.v_pages,
                                   pk.block_table, pk.seq_lens,
                                   max_seq_len=L, ln_lambda=-3.0,
                                   num_splits=3, stats=s2)
    # the tensor-core kernel of blasst_decode: same tiles and decisions
    s3 = m.Stats(mask_numel=B * 4 * nk)
    o3, l3 = m.blasst_decode(x.q, x.k, x.v, ln_lambda=-3.0, num_splits=3,
                             stats=s3)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(s1.mask, s2.mask)
    ref = oracle.decode(x.q, x.k, x.v, 1 / math.sqrt(128), -3.0, Bc, 3,
                        tile_heads=8)
    P.check_mask(s3.mask.cpu().numpy().reshape(B, 4, nk), ref["mask"],
                 ref["margin"], "tensor-core tiles of 8")
    P.check_out(P.to_np(o3), P.to_np(o1), "tensor-core vs CUDA-core tiles")


def test_group_not_power_of_two_is_refused(blasst):
    m = blasst
    q = torch.zeros(1, 12, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 256, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BlasstError, match="UNSUPPORTED"):
        m.blasst_decode(q, k, k)


def test_mqa_full_size_sampled(blasst):
    """B 8, Hq 32, Hkv 1 (MQA), Lkv 32768, d 128, lambda calibrated for 50%
    (8-row tiles vote over more heads than the GQA 4:1 tiles, so less of
    the cache is skippable); sequences 0 and 7 compared with the oracle."""
    m = blasst
    B, Hq, Hkv, L, d = 8, 32, 1, 32768, 128
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=Bc, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(10, 3))
    cal = m.blasst_calibrate(0.50, mode="decode", q=q, k=k, v=v, Bc=Bc,
                             raise_on_no_converge=False)
    assert cal["achieved"] > 0.2
    x = type("X", (), {"q": q, "k": k, "v": v})
    mask, _ = _compare(m, x, cal["ln_lambda"], 0, bs=[0, 7])
    assert P.sparsity(mask) >= cal["achieved"] - 1e-9
