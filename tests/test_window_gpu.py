"""GPU parity of the sliding-window forms (blasst_prefill_window,
blasst_decode_window) against the CPU oracle, through the C ABI.

Prefill: query r sees the W keys ending at its diagonal; decode: the token
sees the last W keys.  Checks outputs (max 2e-2 / mean 2e-3), lse, skip
masks (bit-exact except near-ties, blocks outside the window = 0), counters,
the statistics-only pass, ragged tiles, Lq < Lkv, GQA ratios, windows
smaller than a block and covering everything (identical to the plain
call), argument checks, and a 32-head 8K prefill with a 2K window on
sampled tiles.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import config_seed, planted_gap
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


def _prefill_compare(m, x, W, ln_lambda, units=None, stats_only_check=True):
    q, k, v = x.q, x.k, x.v
    B, Hq, Lq, d = q.shape
    Lkv = k.shape[2]
    Br = 128
    nq, nk = -(-Lq // Br), -(-Lkv // Br)
    scale = 1.0 / math.sqrt(d)
    stats = m.Stats(mask_numel=B * Hq * nq * nk)
    o, lse = m.blasst_prefill_window(q, k, v, window=W, scale=scale,
                                     causal=True, ln_lambda=ln_lambda,
                                     stats=stats)
    torch.cuda.synchronize()
    st, where = m.blasst_check_device_error()
    assert st == 0, f"device error word set (wait {where})"
    ref = oracle.prefill(q, k, v, scale, True, ln_lambda, Br, Br, units=units,
                         window=W)
    mask = stats.mask.cpu().numpy().reshape(B, Hq, nq, nk)
    o_np, l_np = P.to_np(o), P.to_np(lse)
    go, ro, gl, rl, gm = [], [], [], [], []
    for u, (b, h, i) in enumerate(ref["units"]):
        r0, r1 = i * Br, min((i + 1) * Br, Lq)
        go.append(o_np[b, h, r0:r1])
        ro.append(ref["o"][u, :r1 - r0])
        gl.append(l_np[b, h, r0:r1])
        rl.append(ref["lse"][u, :r1 - r0])
        gm.append(mask[b, h, i])
    P.check_out(np.concatenate(go), np.concatenate(ro), "window prefill o")
    P.check_lse(np.concatenate(gl), np.concatenate(rl), "window prefill lse")
    ties = P.check_mask(np.stack(gm), ref["mask"], ref["margin"],
                        "window prefill mask")
    vis, skp = stats.read()
    assert vis == int((mask > 0).sum()) and skp == int((mask == 2).sum())
    if units is None and ties == 0:
        assert (vis, skp) == (ref["visited"], ref["skipped"])
    if stats_only_check:
        st2 = m.Stats(mask_numel=B * Hq * nq * nk)
        r2 = m.blasst_prefill_window(q, k, v, window=W, scale=scale,
                                     ln_lambda=ln_lambda, stats=st2,
                                     stats_only=True)
        assert r2 == (None, None)
        assert torch.equal(st2.mask, stats.mask)
        assert st2.read() == (vis, skp)
    return ref, mask


PREFILL_WINDOW_CASES = [
    # B, Hq, Hkv, Lq, Lkv, d, W, ln_lambda
    (1, 4, 2, 1024, 1024, 128, 300, -4.0),
    (1, 4, 2, 1024, 1024, 128, 300, -math.inf),
    (1, 2, 2, 700, 700, 128, 128, -3.0),      # ragged last tile
    (2, 4, 1, 500, 900, 128, 200, -3.0),      # Lq < Lkv, MQA
    (1, 4, 4, 640, 640, 64, 64, -2.0),        # d 64, window = half a block
    (1, 2, 2, 512, 512, 128, 1, -2.0),        # each query sees itself only
    (1, 8, 2, 1536, 1536, 128, 700, -5.0),
]


@pytest.mark.parametrize("case", PREFILL_WINDOW_CASES)
def test_prefill_window_matches_oracle(blasst, case):
    B, Hq, Hkv, Lq, Lkv, d, W, ln_lambda = case
    x = planted_gap(B, Hq, Hkv, Lq, Lkv, d, block=128, gap=8.0,
                    heavy_frac=0.05, window=256,
                    seed=config_seed(5, Lq + W + d), device="cuda")
    ref, mask = _prefill_compare(blasst, x, W, ln_lambda)
    if ln_lambda == -math.inf:
        assert (mask == 2).sum() == 0
    if W < Lkv // 2:
        assert (mask == 0).any()  # blocks left of the window exist


def test_prefill_window_covering_everything_equals_plain(blasst):
    m = blasst
    x = planted_gap(1, 4, 2, 1000, 1000, 128, block=128, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(5, 1), device="cuda")
    s1, s2 = m.Stats(mask_numel=4 * 8 * 8), m.Stats(mask_numel=4 * 8 * 8)
    o1, l1 = m.blasst_prefill(x.q, x.k, x.v, ln_lambda=-3.0, stats=s1)
    o2, l2 = m.blasst_prefill_window(x.q, x.k, x.v, window=1000,
                                     ln_lambda=-3.0, stats=s2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(s1.mask, s2.mask) and s1.read() == s2.read()


def test_prefill_window_rejects_bad_arguments(blasst):
    m = blasst
    q = torch.zeros(1, 2, 256, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BlasstError, match="INVALID_ARG"):
        m.blasst_prefill_window(q, q, q, window=64, causal=False)
    with pytest.raises(m.BlasstError, match="INVALID_ARG"):
        m.blasst_prefill_window(q, q, q, window=-1)
    q64 = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BlasstError, match="UNSUPPORTED"):
        m.blasst_prefill_window(q64, q64, q64, window=64, Br=64, Bc=64)


def test_prefill_window_32_heads_8k_sampled(blasst):
    """B 1, Hq 32, Hkv 8, L 8192, d 128, window 2048, ln lambda -4: 12
    sampled tiles (first, window edge, middle, last) of 3 heads."""
    x = planted_gap(1, 32, 8, 8192, 8192, 128, block=128, gap=8.0,
                    heavy_frac=0.02, window=512, seed=config_seed(5, 8192),
                    device="cuda")
    units = [(0, h, i) for h in (0, 13, 31) for i in (0, 16, 40, 63)]
    _prefill_compare(blasst, x, 2048, -4.0, units=units,
                     stats_only_check=False)


def _decode_compare(m, x, W, ln_lambda, S_req):
    q, k, v = x.q, x.k, x.v
    B, Hq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    Bc = 64
    nk = -(-Lkv // Bc)
    jlo = (Lkv - W) // Bc if 0 < W < Lkv else 0
    S = (S_req if S_req > 0
         else m.blasst_decode_group_splits(B, Hq, Hkv, Lkv - jlo * Bc))
    stats = m.Stats(mask_numel=B * Hkv * nk)
    stats.mask.fill_(7)  # blocks left of the window must be written 0
    scale = 1.0 / math.sqrt(d)
    o, lse = m.blasst_decode_window(q, k, v, window=W, scale=scale,
                                    ln_lambda=ln_lambda, num_splits=S_req,
                                    stats=stats)
    torch.cuda.synchronize()
    st, where = m.blasst_check_device_error()
    assert st == 0, f"device error word set (wait {where})"
    ref = oracle.decode(q, k, v, scale, ln_lambda, Bc, S, window=W)
    P.check_out(P.to_np(o), ref["o"], "window decode o")
    P.check_lse(P.to_np(lse), ref["lse"], "window decode lse")
    mask = stats.mask.cpu().numpy().reshape(B, Hkv, nk)
    ties = P.check_mask(mask, ref["mask"], ref["margin"], "window decode mask")
    assert (mask[:, :, :jlo] == 0).all()
    vis, skp = stats.read()
    assert vis == B * Hkv * (nk - jlo)
    assert skp == int((mask == 2).sum())
    if ties == 0:
        assert (vis, skp) == (ref["visited"], ref["skipped"])
    st2 = m.Stats(mask_numel=B * Hkv * nk)
    r2 = m.blasst_decode_window(q, k, v, window=W, scale=scale,
                                ln_lambda=ln_lambda, num_splits=S_req,
                                stats=st2, stats_only=True)
    assert r2 == (None, None)
    assert st2.read() == (vis, skp)
    return ref, mask


DECODE_WINDOW_CASES = [
    # B, Hq, Hkv, Lkv, W, ln_lambda, num_splits (0 = automatic)
    (2, 8, 2, 3000, 1000, -3.0, 0),
    (2, 8, 2, 3000, 1000, -math.inf, 3),
    (3, 32, 8, 4096, 2048, -4.0, 4),
    (2, 8, 8, 777, 50, -2.0, 1),          # window inside one block
    (1, 16, 8, 2048, 129, -1.0, 2),
    (2, 8, 1, 1500, 600, -3.0, 5),
]


@pytest.mark.parametrize("case", DECODE_WINDOW_CASES)
def test_decode_window_matches_oracle(blasst, case):
    B, Hq, Hkv, Lkv, W, ln_lambda, S = case
    x = planted_gap(B, Hq, Hkv, 1, Lkv, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(6, Lkv + W + Hq),
                    device="cuda")
    _decode_compare(blasst, x, W, ln_lambda, S)


def test_decode_window_covering_everything_equals_plain(blasst):
    m = blasst
    x = planted_gap(2, 8, 2, 1, 1000, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=config_seed(6, 1), device="cuda")
    o1, l1 = m.blasst_decode(x.q, x.k, x.v, ln_lambda=-3.0, num_splits=3)
    o2, l2 = m.blasst_decode_window(x.q, x.k, x.v, window=5000,
                                    ln_lambda=-3.0, num_splits=3)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_window_rejects_bad_arguments(blasst):
    m = blasst
    x = planted_gap(1, 8, 2, 1, 1000, 128, decode=True, block=64,
                    seed=config_seed(6, 2), device="cuda")
    with pytest.raises(m.BlasstError, match="INVALID_ARG"):
        m.blasst_decode_window(x.q, x.k, x.v, window=-5)
    # the last 300 keys lie in blocks 10..15: 7 splits cannot be formed
    with pytest.raises(m.BlasstError, match="INVALID_ARG"):
        m.blasst_decode_window(x.q, x.k, x.v, window=300, num_splits=7)
