"""GPU parity of the batched decision rule (blasst_decode_batched, batch 2)
against the oracle's batched decode, through the C ABI.

Blocks are scored in pairs and each is judged against the max over the
earlier blocks and the whole pair.  Checks outputs (max 2e-2 / mean 2e-3),
lse, masks (bit-exact except near-ties), counters, the statistics-only
pass, GQA ratios, odd block counts (a last pair of one block), batch 1
identical to blasst_decode, the superset property against the sequential
rule, argument checks, and the full-size decode workload (batch 32, 32K
cache) at the 70% threshold on 4 sampled sequences.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import config_seed, planted_gap, planted_gap_kv_inplace
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


def _compare(m, q, k, v, ln_lambda, S_req, check_stats_only=True, bs=None):
    B, Hq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    Bc = 64
    nk = -(-Lkv // Bc)
    S = S_req if S_req > 0 else m.blasst_decode_splits(B, Hkv, Lkv, Bc)
    scale = 1.0 / math.sqrt(d)
    stats = m.Stats(mask_numel=B * Hkv * nk)
    o, lse = m.blasst_decode_batched(q, k, v, batch=2, scale=scale,
                                     ln_lambda=ln_lambda, num_splits=S_req,
                                     stats=stats)
    torch.cuda.synchronize()
    st, where = m.blasst_check_device_error()
    assert st == 0, f"device error word set (wait {where})"
    mask = stats.mask.cpu().numpy().reshape(B, Hkv, nk)
    bsel = list(range(B)) if bs is None else bs
    qs, ks, vs = q[bsel], k[bsel], v[bsel]
    ref = oracle.decode_batched(qs, ks, vs, scale, ln_lambda, Bc, S, 2)
    P.check_out(P.to_np(o)[bsel], ref["o"], "batched decode o")
    P.check_lse(P.to_np(lse)[bsel], ref["lse"], "batched decode lse")
    ties = P.check_mask(mask[bsel], ref["mask"], ref["margin"],
                        "batched decode mask")
    vis, skp = stats.read()
    assert vis == B * Hkv * nk and skp == int((mask == 2).sum())
    if bs is None and ties == 0:
        assert (vis, skp) == (ref["visited"], ref["skipped"])
    if check_stats_only:
        st2 = m.Stats(mask_numel=B * Hkv * nk)
        r2 = m.blasst_decode_batched(q, k, v, batch=2, scale=scale,
                                     ln_lambda=ln_lambda, num_splits=S_req,
                                     stats=st2, stats_only=True)
        assert r2 == (None, None)
        assert torch.equal(st2.mask, stats.mask)
        assert st2.read() == (vis, skp)
    return mask, ref


BATCHED_CASES = [
    # B, Hq, Hkv, Lkv, ln_lambda, num_splits (0 = automatic)
    (2, 8, 2, 1000, -3.0, 0),
    (3, 32, 8, 4096, -4.0, 3),
    (2, 8, 8, 777, -2.0, 2),
    (2, 16, 8, 2048, -5.0, 4),
    (2, 8, 2, 2048, -math.inf, 5),
    (1, 4, 1, 64 * 7, -1.0, 1),    # 7 blocks: the last pair has one block
    (2, 32, 8, 3000, 0.0, 7),
]


@pytest.mark.parametrize("case", BATCHED_CASES)
def test_batched_decode_matches_oracle(blasst, case):
    B, Hq, Hkv, Lkv, ln_lambda, S = case
    x = planted_gap(B, Hq, Hkv, 1, Lkv, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(9, Lkv + Hq + S),
                    device="cuda")
    mask, ref = _compare(blasst, x.q, x.k, x.v, ln_lambda, S)
    if ln_lambda == -math.inf:
        assert (mask == 2).sum() == 0


def test_batch_one_equals_decode(blasst):
    """batch = 1 is the sequential rule: the same decisions as
    blasst_decode (which runs it on the warp-MMA kernel; batch 1 runs on the
    CUDA-core kernel), so masks agree except on near-ties and outputs within
    the parity tolerance."""
    m = blasst
    x = planted_gap(2, 8, 2, 1, 1500, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(9, 1), device="cuda")
    s1, s2 = m.Stats(mask_numel=2 * 2 * 24), m.Stats(mask_numel=2 * 2 * 24)
    o1, l1 = m.blasst_decode(x.q, x.k, x.v, ln_lambda=-3.0, num_splits=3,
                             stats=s1)
    o2, l2 = m.blasst_decode_batched(x.q, x.k, x.v, batch=1, ln_lambda=-3.0,
                                     num_splits=3, stats=s2)
    torch.cuda.synchronize()
    ref = oracle.decode(x.q, x.k, x.v, 1 / math.sqrt(128), -3.0, 64, 3)
    P.check_mask(s1.mask.cpu().numpy().reshape(2, 2, 24), ref["mask"],
                 ref["margin"], "decode")
    P.check_mask(s2.mask.cpu().numpy().reshape(2, 2, 24), ref["mask"],
                 ref["margin"], "batch 1")
    P.check_out(P.to_np(o1), P.to_np(o2), "decode vs batch 1")
    P.check_lse(P.to_np(l1), P.to_np(l2), "decode vs batch 1")


def test_batched_skips_superset_of_sequential(blasst):
    m = blasst
    x = planted_gap(4, 32, 8, 1, 4096, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.03, seed=config_seed(9, 2), device="cuda")
    nk = 64
    s1, s2 = m.Stats(mask_numel=4 * 8 * nk), m.Stats(mask_numel=4 * 8 * nk)
    m.blasst_decode(x.q, x.k, x.v, ln_lambda=-5.0, num_splits=2, stats=s1)
    m.blasst_decode_batched(x.q, x.k, x.v, batch=2, ln_lambda=-5.0,
                            num_splits=2, stats=s2)
    torch.cuda.synchronize()
    seq = s1.mask.cpu().numpy() == 2
    bat = s2.mask.cpu().numpy() == 2
    # outside near-ties the batched skips contain the sequential ones
    ref_s = oracle.decode(x.q, x.k, x.v, 1 / math.sqrt(128), -5.0, 64, 2)
    near = np.abs(np.nan_to_num(ref_s["margin"].reshape(-1), nan=1.0,
                                posinf=1.0)) < P.NEAR_TIE
    assert not (seq & ~bat & ~near).any()
    assert bat.sum() > seq.sum()


def test_batched_head_dim_64_matches_oracle(blasst):
    m = blasst
    x = planted_gap(2, 8, 2, 1, 1999, 64, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(9, 64), device="cuda")
    nk = -(-1999 // 64)
    st = m.Stats(mask_numel=2 * 2 * nk)
    o, lse = m.blasst_decode_batched(x.q, x.k, x.v, batch=2, ln_lambda=-3.0,
                                     num_splits=3, stats=st)
    torch.cuda.synchronize()
    ref = oracle.decode_batched(x.q, x.k, x.v, 1 / 8.0, -3.0, 64, 3, 2)
    P.check_out(P.to_np(o), ref["o"], "batched d64 o")
    P.check_lse(P.to_np(lse), ref["lse"], "batched d64 lse")
    P.check_mask(st.mask.cpu().numpy().reshape(2, 2, nk), ref["mask"],
                 ref["margin"], "batched d64 mask")


def test_batched_rejects_bad_batch(blasst):
    m = blasst
    x = planted_gap(1, 8, 2, 1, 512, 128, decode=True, block=64,
                    seed=config_seed(9, 3), device="cuda")
    with pytest.raises(m.BlasstError, match="UNSUPPORTED"):
        m.blasst_decode_batched(x.q, x.k, x.v, batch=3)


def test_batched_full_size_sampled(blasst):
    """B 32, Hq 32, Hkv 8, Lkv 32768, d 128, lambda for 70% (sequential
    rule); sequences 0, 9, 22, 31 compared with the batched oracle."""
    m = blasst
    B, Hq, Hkv, L, d = 32, 32, 8, 32768, 128
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(1))
    cal = m.blasst_calibrate(0.70, mode="decode", q=q, k=k, v=v, Bc=64)
    mask, ref = _compare(m, q, k, v, cal["ln_lambda"], 0,
                         check_stats_only=False, bs=[0, 9, 22, 31])
    assert P.sparsity(mask) >= cal["achieved"] - 1e-9
