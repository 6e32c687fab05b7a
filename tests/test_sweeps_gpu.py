"""GPU parity and calibration checks on the two sweep workloads.

Decode length sweep: batch 148, Hq 32 / Hkv 8, d 128, Bc 64, planted gap 8
with sink + 3% heavy blocks, Lkv in {8K, 32K, 64K, 128K}; a is fitted once
at 32K for 70% sparsity (lambda = a / L, the inverse law of the BLASST
summary, section 2 "Calibracao Automatica") and applied to every length;
4 sampled sequences per length are compared with the oracle.

Prefill sparsity / calibration sweep: B 1, Hq 32 / Hkv 8, d 128, causal,
128x128 tiles, gap drawn per head from U[4, 12] nats, sink + 2% heavy +
512-token window boost, L in {4K, 16K, 64K}; for each target sparsity in
{0, 30, 50, 70, 90}% a is fitted over the three lengths in log space and
the deviation |s(a/L) - target| is reported; the 4K case is compared with
the oracle in full.

Each test appends a JSON record of what it measured to the file named by
the BLASST_SWEEP_RECORD environment variable, when it is set.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from synth import config_seed, planted_gap, planted_gap_kv_inplace
from tests import _parity as P

pytestmark = pytest.mark.gpu

def _record(obj):
    path = os.environ.get("BLASST_SWEEP_RECORD")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(obj) + "\n")


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


def _time_ms(fn, reps=5):
    fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


@pytest.fixture(scope="module")
def decode_a_at_32k(blasst):
    """a of lambda = a / L fitted at 32K for 70% sparsity (batch 148)."""
    m = blasst
    B, Hq, Hkv, L, d = 148, 32, 8, 32768, 128
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(3, L))
    cal = m.blasst_calibrate(0.70, mode="decode", q=q, k=k, v=v, Bc=64)
    del q, k, v
    torch.cuda.empty_cache()
    return cal


@pytest.mark.parametrize("L", [8192, 32768, 65536, 131072])
def test_decode_length_sweep(blasst, decode_a_at_32k, L):
    m = blasst
    B, Hq, Hkv, d = 148, 32, 8, 128
    a = decode_a_at_32k["a"]
    lnl = min(0.0, math.log(a / L))
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(3, L))
    nk = L // 64
    S = m.blasst_decode_splits(B, Hkv, L, 64)
    st = m.Stats(mask_numel=B * Hkv * nk)
    o, lse = m.blasst_decode(q, k, v, ln_lambda=lnl, stats=st)
    torch.cuda.synchronize()
    vis, skp = st.read()
    mask = st.mask.cpu().numpy().reshape(B, Hkv, nk)
    ties = 0
    for b in (0, 37, 101, 147):
        ref = oracle.decode(q[b:b + 1], k[b:b + 1], v[b:b + 1],
                            1 / math.sqrt(d), lnl, 64, S)
        P.check_out(P.to_np(o[b:b + 1]), ref["o"], f"L={L} seq {b}")
        P.check_lse(P.to_np(lse[b:b + 1]), ref["lse"], f"L={L} seq {b}")
        ties += P.check_mask(mask[b:b + 1], ref["mask"], ref["margin"],
                             f"L={L} seq {b}")
    sparse_ms = _time_ms(lambda: m.blasst_decode(q, k, v, ln_lambda=lnl))
    dense_ms = _time_ms(lambda: m.blasst_decode(q, k, v))
    kept_rows = int((mask == 1).sum()) * 64
    by = 2 * L * d * B * Hkv + 2 * d * kept_rows + 2 * B * Hq * d \
        + B * Hq * S * (d + 1) * 8 + B * Hq * (2 * d + 4)
    _record({"sweep": "decode_length", "L": L, "a": a, "ln_lambda": lnl,
             "splits": S, "sparsity": skp / vis, "near_ties": ties,
             "us": sparse_ms * 1e3, "dense_us": dense_ms * 1e3,
             "GBps": by / (sparse_ms / 1e3) / 1e9,
             "speedup_vs_dense": dense_ms / sparse_ms})
    assert vis == B * Hkv * nk
    del q, k, v, o, lse
    torch.cuda.empty_cache()


PREFILL_LENGTHS = [4096, 16384, 65536]
PREFILL_TARGETS = [0.0, 0.3, 0.5, 0.7, 0.9]


@pytest.fixture(scope="module")
def prefill_sweep_inputs():
    xs = {}
    for L in PREFILL_LENGTHS:
        xs[L] = planted_gap(1, 32, 8, L, L, 128, block=128, gap_range=(4.0, 12.0),
                            heavy_frac=0.02, window=512, seed=config_seed(4, L),
                            device="cuda")
    return xs


def test_prefill_sweep_calibration_law(blasst, prefill_sweep_inputs):
    """Fit lambda = a / L per target over the three lengths and report the
    deviation of the achieved sparsity from the target at each length."""
    m = blasst
    records = []
    for tgt in PREFILL_TARGETS:
        cals = {}
        for L, x in prefill_sweep_inputs.items():
            cals[L] = m.blasst_calibrate(tgt, mode="prefill", q=x.q, k=x.k,
                                         v=x.v, Br=128, Bc=128,
                                         raise_on_no_converge=False)
        # lengths whose calibration cannot reach the target (the first and
        # the diagonal blocks of a causal tile are rarely skippable, which
        # caps the sparsity of short sequences) are left out of the fit
        fit_L = [L for L in cals if cals[L]["status"] == 0]
        if tgt == 0.0 or not fit_L:
            a = None  # target 0: lambda -> 0 (the dense path)
        else:
            a = m.blasst_fit_a([cals[L]["lambda_"] for L in fit_L], fit_L)
        for L, x in prefill_sweep_inputs.items():
            lnl = -math.inf if a is None else min(0.0, math.log(a / L))
            st = m.Stats()
            m.blasst_prefill(x.q, x.k, x.v, ln_lambda=lnl, Br=128, Bc=128,
                             stats=st, stats_only=True)
            torch.cuda.synchronize()
            s = st.sparsity()
            fn = (lambda x=x, lnl=lnl: m.blasst_prefill(
                x.q, x.k, x.v, ln_lambda=lnl, Br=128, Bc=128))
            ms = _time_ms(fn, reps=3)
            dense_ms = _time_ms(lambda x=x: m.blasst_prefill(
                x.q, x.k, x.v, Br=128, Bc=128), reps=3)
            rec = {"sweep": "prefill_calibration", "L": L, "target": tgt,
                   "a": a, "ln_lambda": lnl, "sparsity": s,
                   "deviation": abs(s - tgt),
                   "calibrated_at_L": cals[L]["achieved"],
                   "us": ms * 1e3, "dense_us": dense_ms * 1e3,
                   "speedup_vs_dense": dense_ms / ms,
                   "dense_equiv_tflops": 4 * 32 * 128 * (L * (L + 1) / 2)
                   / (ms / 1e3) / 1e12}
            rec["calibration_status"] = cals[L]["status"]
            records.append(rec)
            _record(rec)
            # a per-length calibration that converged reaches its target
            if cals[L]["status"] == 0:
                assert cals[L]["achieved"] >= tgt - 1e-9
                assert abs(cals[L]["achieved"] - tgt) < 0.02
        if tgt == 0.0:
            assert all(r["sparsity"] == 0.0 for r in records if r["target"] == 0.0)
    devs = [r["deviation"] for r in records
            if r["target"] > 0 and r["calibration_status"] == 0]
    _record({"sweep": "prefill_calibration_summary",
             "mean_deviation": float(np.mean(devs)),
             "max_deviation": float(np.max(devs))})


@pytest.mark.parametrize("tgt", [0.3, 0.5, 0.7])
def test_prefill_sweep_4k_parity(blasst, prefill_sweep_inputs, tgt):
    """Full oracle comparison of the 4K sweep case at calibrated targets
    (90% is out of reach at 4K: every causal tile keeps its first block and
    nearly always its diagonal block, which caps the sparsity near 79%)."""
    m = blasst
    x = prefill_sweep_inputs[4096]
    cal = m.blasst_calibrate(tgt, mode="prefill", q=x.q, k=x.k, v=x.v,
                             Br=128, Bc=128)
    lnl = cal["ln_lambda"]
    nq = nk = 32
    st = m.Stats(mask_numel=32 * nq * nk)
    o, lse = m.blasst_prefill(x.q, x.k, x.v, ln_lambda=lnl, Br=128, Bc=128,
                              stats=st)
    torch.cuda.synchronize()
    ref = oracle.prefill(x.q, x.k, x.v, 1 / math.sqrt(128), True, lnl, 128, 128)
    o_np, l_np = P.to_np(o), P.to_np(lse)
    mask = st.mask.cpu().numpy().reshape(1, 32, nq, nk)
    go = np.stack([o_np[b, h, i * 128:(i + 1) * 128] for (b, h, i) in ref["units"]])
    gl = np.stack([l_np[b, h, i * 128:(i + 1) * 128] for (b, h, i) in ref["units"]])
    gm = np.stack([mask[b, h, i] for (b, h, i) in ref["units"]])
    mx, mean = P.check_out(go, ref["o"], f"4K target {tgt}")
    P.check_lse(gl, ref["lse"], f"4K target {tgt}")
    ties = P.check_mask(gm, ref["mask"], ref["margin"], f"4K target {tgt}")
    _record({"sweep": "prefill_4k_parity", "target": tgt, "ln_lambda": lnl,
             "sparsity": cal["achieved"], "max_abs_err": mx,
             "mean_abs_err": mean, "near_ties": ties})
