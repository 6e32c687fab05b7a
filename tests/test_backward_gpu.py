"""GPU parity of the prefill backward (blasst_prefill_backward) against the
oracle's backward, through the C ABI.

The GPU backward takes the GPU forward's o, lse and decision bytes; the
oracle takes its own forward's (float64 o and lse, its mask).  The two masks
must agree exactly on the seeded inputs used here (the forward parity tests
cover near-ties), so both sides differentiate the same restricted attention.
Checked: dq, dk, dv within the gradient tolerance below, for dense and
skipping forwards, causal and not, GQA and MQA, ragged lengths, Lq < Lkv,
the dense backward (mask None) equal to an all-kept mask, skipped pairs
contributing nothing, argument checks, and a 4K causal sample at 70%.

Tolerance (derived from the arithmetic): both sides start from the same
bf16 q, k, v, dO.  The GPU rounds P and dS to bf16 before their MMAs and
dq, dk, dv to bf16 at the end (relative 2^-9 each, unbiased), uses a bf16
O for D and accumulates in f32.  Per element that is a relative error of
order 2^-8 of the element's terms, so: max |gpu - ref| <= 2e-2 * max|ref|
and mean |gpu - ref| <= 1e-2 * mean|ref| for each of dq, dk, dv.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import config_seed, output_gradient, planted_gap
from tests import _parity as P

pytestmark = pytest.mark.gpu
BR = 128


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


def _check_grad(g, r, name):
    g = P.to_np(g).astype(np.float64)
    err = np.abs(g - r)
    mx, mn = float(np.abs(r).max()), float(np.abs(r).mean())
    assert err.max() <= 2e-2 * max(mx, 1e-6), (name, err.max(), mx)
    assert err.mean() <= 1e-2 * max(mn, 1e-9), (name, err.mean(), mn)
    return err.max() / max(mx, 1e-6), err.mean() / max(mn, 1e-9)


def _run(m, B, Hq, Hkv, Lq, Lkv, causal, lnl, seed, heavy_frac=0.05,
         window=256):
    d = 128
    x = planted_gap(B, Hq, Hkv, Lq, Lkv, d, block=BR, gap=8.0,
                    heavy_frac=heavy_frac, window=window, seed=seed,
                    device="cuda")
    scale = 1.0 / math.sqrt(d)
    nq, nk = -(-Lq // BR), -(-Lkv // BR)
    st = m.Stats(mask_numel=B * Hq * nq * nk)
    o, lse = m.blasst_prefill(x.q, x.k, x.v, scale=scale, causal=causal,
                              ln_lambda=lnl, stats=st)
    dout = output_gradient((B, Hq, Lq, d), seed + 1, device="cuda")
    dq, dk, dv = m.blasst_prefill_backward(x.q, x.k, x.v, o, lse, dout,
                                           mask=st.mask, scale=scale,
                                           causal=causal)
    torch.cuda.synchronize()
    e, where = m.blasst_check_device_error()
    assert e == 0, f"device error word set (wait {where})"
    ref = oracle.prefill(x.q, x.k, x.v, scale, causal, lnl, BR, BR)
    mask_g = st.mask.cpu().numpy().reshape(B, Hq, nq, nk)
    mask_r = ref["mask"].reshape(B, Hq, nq, nk)
    assert np.array_equal(mask_g, mask_r), "forward masks differ (near-tie)"
    o_r = ref["o"].reshape(B, Hq, nq * BR, d)[:, :, :Lq]
    lse_r = ref["lse"].reshape(B, Hq, nq * BR)[:, :, :Lq]
    rq, rk, rv = oracle.prefill_backward(x.q, x.k, x.v, o_r, lse_r, dout,
                                         mask_r, scale, causal, BR, BR)
    res = {n: _check_grad(g, r, n) for n, g, r in
           (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv))}
    return x, st, (dq, dk, dv), res, mask_g


BWD_CASES = [
    # B, Hq, Hkv, Lq, Lkv, causal, ln_lambda
    (1, 2, 2, 512, 512, True, -math.inf),
    (1, 4, 2, 640, 640, True, -3.0),
    (2, 4, 1, 384, 384, False, -2.0),
    (1, 2, 2, 700, 700, True, -3.0),      # ragged last tile and block
    (1, 2, 1, 300, 500, True, -3.0),      # Lq < Lkv
    (1, 8, 8, 1024, 1024, True, -4.0),
]


@pytest.mark.parametrize("case", BWD_CASES)
def test_backward_matches_oracle(blasst, case):
    B, Hq, Hkv, Lq, Lkv, causal, lnl = case
    _, _, _, res, mask = _run(blasst, B, Hq, Hkv, Lq, Lkv, causal, lnl,
                              config_seed(20, Lq + Hq + int(causal)))
    if lnl > -math.inf:
        assert (mask == 2).any()
    print(case, res)


def test_dense_backward_equals_all_kept_mask(blasst):
    m = blasst
    x = planted_gap(1, 4, 2, 512, 512, 128, block=BR, gap=8.0, heavy_frac=0.05,
                    seed=config_seed(20, 1), device="cuda")
    st = m.Stats(mask_numel=4 * 4 * 4)
    o, lse = m.blasst_prefill(x.q, x.k, x.v, stats=st)  # dense: mask all 1
    dout = output_gradient((1, 4, 512, 128), 7, device="cuda")
    a = m.blasst_prefill_backward(x.q, x.k, x.v, o, lse, dout, mask=st.mask)
    b = m.blasst_prefill_backward(x.q, x.k, x.v, o, lse, dout, mask=None)
    torch.cuda.synchronize()
    for u, w in zip(a, b):
        assert torch.equal(u, w)


def test_skipped_pairs_contribute_nothing(blasst):
    """Marking kept pairs as skipped in the mask changes the gradients
    exactly as the oracle's restricted attention says."""
    m = blasst
    B, Hq, Hkv, L = 1, 2, 1, 512
    x = planted_gap(B, Hq, Hkv, L, L, 128, block=BR, gap=8.0, heavy_frac=0.05,
                    seed=config_seed(20, 2), device="cuda")
    o, lse = m.blasst_prefill(x.q, x.k, x.v)
    dout = output_gradient((B, Hq, L, 128), 8, device="cuda")
    mask = torch.ones(B, Hq, 4, 4, dtype=torch.uint8, device="cuda")
    mask[0, 0, 3, 1] = 2
    mask[0, 1, 2, 0] = 2
    dq, dk, dv = m.blasst_prefill_backward(x.q, x.k, x.v, o, lse, dout,
                                           mask=mask)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.prefill_backward(x.q, x.k, x.v, o, lse, dout,
                                         mask.cpu(), 1 / math.sqrt(128), True,
                                         BR, BR)
    for g, r, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        _check_grad(g, r, n)


def test_backward_rejects_bad_arguments(blasst):
    m = blasst
    q = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 2, 256, dtype=torch.float32, device="cuda")
    with pytest.raises(m.BlasstError, match="UNSUPPORTED"):
        m.blasst_prefill_backward(q, q, q, q, lse, q)  # d = 64
    q = torch.zeros(1, 2, 256, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 128, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BlasstError, match="INVALID_ARG"):
        m.blasst_prefill_backward(q, k, k, q, lse, q, causal=True)  # Lq > Lkv
    with pytest.raises(m.BlasstError, match="WORKSPACE"):
        m.blasst_prefill_backward(q, q, q, q, lse, q,
                                  workspace=torch.empty(16, dtype=torch.uint8,
                                                        device="cuda"))


def test_backward_4k_sampled(blasst):
    """B 1, Hq 8, Hkv 2, L 4096, causal, lambda calibrated for 70%."""
    m = blasst
    x = planted_gap(1, 8, 2, 4096, 4096, 128, block=BR, gap=8.0,
                    heavy_frac=0.02, window=512, seed=config_seed(20, 4096),
                    device="cuda")
    cal = m.blasst_calibrate(0.70, mode="prefill", q=x.q, k=x.k, v=x.v)
    _, _, _, res, mask = _run(m, 1, 8, 2, 4096, 4096, True, cal["ln_lambda"],
                              config_seed(20, 4096), heavy_frac=0.02,
                              window=512)
    assert P.sparsity(mask) > 0.6
