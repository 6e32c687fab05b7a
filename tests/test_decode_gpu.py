"""GPU parity of the BLASST decode path (split kernel + merge) against the
CPU oracle, called through the C ABI on seeded planted-gap inputs.

Checks: outputs within max 2e-2 / mean 2e-3, lse, per-block skip decisions
bit-exact except near-ties, counters consistent with the decisions, the
statistics-only pass, every supported GQA ratio, ragged cache lengths,
explicit and automatic split counts, and the full-size decode workload
(batch 32, 32K cache, GQA 4:1) with lambda calibrated to 70% sparsity,
checked on 4 sampled sequences.
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


def _run_and_compare(m, x, ln_lambda, S_req, Bc=64):
    q, k, v = x.q, x.k, x.v
    B, Hq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    nk = -(-Lkv // Bc)
    S = S_req if S_req > 0 else m.blasst_decode_group_splits(B, Hq, Hkv, Lkv, Bc)
    stats = m.Stats(mask_numel=B * Hkv * nk)
    scale = 1.0 / math.sqrt(d)
    o, lse = m.blasst_decode(q, k, v, scale=scale, ln_lambda=ln_lambda, Bc=Bc,
                             num_splits=S_req, stats=stats)
    torch.cuda.synchronize()
    st, where = m.blasst_check_device_error()
    assert st == 0, f"device error word set (wait {where})"
    ref = oracle.decode(q, k, v, scale, ln_lambda, Bc, S)
    P.check_out(P.to_np(o), ref["o"], "decode o")
    P.check_lse(P.to_np(lse), ref["lse"], "decode lse")
    mask = stats.mask.cpu().numpy().reshape(B, Hkv, nk)
    ties = P.check_mask(mask, ref["mask"], ref["margin"], "decode mask")
    vis, skp = stats.read()
    assert vis == B * Hkv * nk
    assert skp == int((mask == 2).sum())
    if ties == 0:
        assert (vis, skp) == (ref["visited"], ref["skipped"])
    # statistics-only pass: same decisions and counters, nothing written
    st2 = m.Stats(mask_numel=B * Hkv * nk)
    r2 = m.blasst_decode(q, k, v, scale=scale, ln_lambda=ln_lambda, Bc=Bc,
                         num_splits=S_req, stats=st2, stats_only=True)
    assert r2 == (None, None)
    assert torch.equal(st2.mask, stats.mask)
    assert st2.read() == (vis, skp)
    return ref, mask, ties


DECODE_CASES = [
    # B, Hq, Hkv, Lkv, ln_lambda, num_splits (0 = automatic)
    (2, 8, 2, 1000, -3.0, 0),
    (3, 32, 8, 4096, -4.0, 3),
    (2, 8, 8, 777, -2.0, 2),
    (2, 16, 8, 2048, -5.0, 4),
    (1, 64, 8, 1536, -3.0, 1),
    (2, 8, 2, 2048, -math.inf, 5),
    (1, 4, 1, 64, -1.0, 1),
    (1, 4, 1, 65, -1.0, 2),
    (2, 32, 8, 3000, 0.0, 7),
]


@pytest.mark.parametrize("case", DECODE_CASES)
def test_decode_matches_oracle(blasst, case):
    B, Hq, Hkv, Lkv, ln_lambda, S = case
    x = planted_gap(B, Hq, Hkv, 1, Lkv, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.03, seed=config_seed(1, Lkv + Hq),
                    device="cuda")
    ref, mask, ties = _run_and_compare(blasst, x, ln_lambda, S)
    if ln_lambda == -math.inf:
        assert (mask == 2).sum() == 0


D64_CASES = [
    # B, Hq, Hkv, Lkv, ln_lambda, num_splits: head dimension 64
    (2, 8, 2, 1000, -3.0, 0),
    (2, 32, 8, 3000, -2.0, 3),
    (1, 8, 1, 700, -math.inf, 2),
    (1, 2, 2, 65, -1.0, 1),
]


@pytest.mark.parametrize("case", D64_CASES)
def test_decode_head_dim_64_matches_oracle(blasst, case):
    B, Hq, Hkv, Lkv, ln_lambda, S = case
    x = planted_gap(B, Hq, Hkv, 1, Lkv, 64, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(1, 640 + Lkv + Hq),
                    device="cuda")
    ref, mask, ties = _run_and_compare(blasst, x, ln_lambda, S)
    if ln_lambda == -math.inf:
        assert (mask == 2).sum() == 0


def test_decode_rejects_bad_arguments(blasst):
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 256, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(blasst.BlasstError, match="INVALID_ARG"):
        blasst.blasst_decode(q, k, k, ln_lambda=0.5)
    with pytest.raises(blasst.BlasstError, match="INVALID_ARG"):
        blasst.blasst_decode(q, k, k, num_splits=5)  # more splits than blocks
    q96 = torch.zeros(1, 4, 96, dtype=torch.bfloat16, device="cuda")
    k96 = torch.zeros(1, 1, 256, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(blasst.BlasstError, match="UNSUPPORTED"):
        blasst.blasst_decode(q96, k96, k96)
    q3 = torch.zeros(1, 3, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(blasst.BlasstError, match="UNSUPPORTED"):
        blasst.blasst_decode(q3, k, k)  # 3:1 grouping is not built
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(blasst.BlasstError, match="WORKSPACE"):
        blasst.blasst_decode(q, k, k, workspace=ws)


def test_decode_full_size_sampled(blasst):
    """Batch 32, Hq 32 / Hkv 8, 32K cache, d 128, Bc 64, lambda calibrated
    to 70% sparsity in the benchmark's launch configuration (automatic
    splits); 4 sequences compared with the oracle."""
    m = blasst
    B, Hq, Hkv, Lkv, d = 32, 32, 8, 32768, 128
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, Lkv, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(1))
    cal = m.blasst_calibrate(0.70, mode="decode", q=q, k=k, v=v, Bc=64)
    assert abs(cal["achieved"] - 0.70) < 0.01
    nk = Lkv // 64
    S = m.blasst_decode_splits(B, Hkv, Lkv, 64)
    stats = m.Stats(mask_numel=B * Hkv * nk)
    o, lse = m.blasst_decode(q, k, v, ln_lambda=cal["ln_lambda"], stats=stats)
    torch.cuda.synchronize()
    vis, skp = stats.read()
    assert vis == B * Hkv * nk
    assert skp / vis == pytest.approx(cal["achieved"], abs=1e-12)
    mask = stats.mask.cpu().numpy().reshape(B, Hkv, nk)
    for b in (0, 9, 22, 31):
        ref = oracle.decode(q[b:b + 1], k[b:b + 1], v[b:b + 1], 1 / math.sqrt(d),
                            cal["ln_lambda"], 64, S)
        P.check_out(P.to_np(o[b:b + 1]), ref["o"], f"seq {b}")
        P.check_lse(P.to_np(lse[b:b + 1]), ref["lse"], f"seq {b}")
        P.check_mask(mask[b:b + 1], ref["mask"], ref["margin"], f"seq {b}")
