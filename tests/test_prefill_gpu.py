"""GPU parity of the BLASST prefill kernel (tcgen05 / TMEM / TMA) against
the CPU oracle, called through the C ABI on seeded planted-gap inputs.

Covers the tiny configuration of the kernel benchmarks (B 1, 2 heads, 1024
tokens, d 64, Br = Bc = 64, ln lambda = -6) in full, the dense path, ragged
tiles, GQA and MQA, Lq < Lkv with bottom-right causal alignment, the
non-causal case, both head dimensions with both tile sizes, the
statistics-only pass, and the full-size prefill (32 heads, 32K tokens, GQA
4:1, d 128, 128x128 tiles) at a calibrated 70% sparsity on sampled tiles.
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


def _compare(m, x, causal, Br, ln_lambda, units=None, check_stats_only=True):
    q, k, v = x.q, x.k, x.v
    B, Hq, Lq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    Bc = Br
    nq, nk = -(-Lq // Br), -(-Lkv // Bc)
    scale = 1.0 / math.sqrt(d)
    stats = m.Stats(mask_numel=B * Hq * nq * nk)
    o, lse = m.blasst_prefill(q, k, v, scale=scale, causal=causal,
                              ln_lambda=ln_lambda, Br=Br, Bc=Bc, stats=stats)
    torch.cuda.synchronize()
    st, where = m.blasst_check_device_error()
    assert st == 0, f"device error word set (wait {where})"
    ref = oracle.prefill(q, k, v, scale, causal, ln_lambda, Br, Bc, units=units)
    mask = stats.mask.cpu().numpy().reshape(B, Hq, nq, nk)
    o_np = P.to_np(o)
    l_np = P.to_np(lse)
    go, ro, gl, rl, gm = [], [], [], [], []
    for u, (b, h, i) in enumerate(ref["units"]):
        r0, r1 = i * Br, min((i + 1) * Br, Lq)
        go.append(o_np[b, h, r0:r1])
        ro.append(ref["o"][u, :r1 - r0])
        gl.append(l_np[b, h, r0:r1])
        rl.append(ref["lse"][u, :r1 - r0])
        gm.append(mask[b, h, i])
    P.check_out(np.concatenate(go), np.concatenate(ro), "prefill o")
    P.check_lse(np.concatenate(gl), np.concatenate(rl), "prefill lse")
    ties = P.check_mask(np.stack(gm), ref["mask"], ref["margin"], "prefill mask")
    vis, skp = stats.read()
    assert vis == int((mask > 0).sum()) and skp == int((mask == 2).sum())
    if units is None and ties == 0:
        assert (vis, skp) == (ref["visited"], ref["skipped"])
    if check_stats_only:
        st2 = m.Stats(mask_numel=B * Hq * nq * nk)
        r2 = m.blasst_prefill(q, k, v, scale=scale, causal=causal,
                              ln_lambda=ln_lambda, Br=Br, Bc=Bc, stats=st2,
                              stats_only=True)
        assert r2 == (None, None)
        assert torch.equal(st2.mask, stats.mask)
        assert st2.read() == (vis, skp)
    return ref, mask, ties


PREFILL_CASES = [
    # B, Hq, Hkv, Lq, Lkv, d, causal, Br(=Bc), ln_lambda, window
    (1, 2, 2, 1024, 1024, 64, True, 64, -6.0, None),     # tiny configuration
    (1, 2, 2, 1024, 1024, 64, True, 64, -math.inf, None),
    (1, 4, 2, 1000, 1000, 128, True, 128, -4.0, 256),
    (2, 4, 1, 300, 700, 128, True, 128, -3.0, 128),
    (1, 2, 2, 640, 640, 128, False, 128, -3.0, None),
    (1, 4, 4, 777, 777, 64, True, 128, -2.0, 256),
    (1, 4, 2, 700, 700, 128, True, 64, -3.0, 128),
    (1, 8, 2, 2048, 2048, 128, True, 128, -math.inf, 512),
    (1, 2, 1, 100, 100, 128, True, 128, 0.0, None),       # single ragged tile
    (1, 2, 2, 130, 4000, 64, False, 64, -2.5, None),
]


@pytest.mark.parametrize("case", PREFILL_CASES)
def test_prefill_matches_oracle(blasst, case):
    B, Hq, Hkv, Lq, Lkv, d, causal, Br, ln_lambda, window = case
    x = planted_gap(B, Hq, Hkv, Lq, Lkv, d, block=Br, gap=8.0, heavy_frac=0.03,
                    window=window, seed=config_seed(0, Lq + Hq + d),
                    device="cuda")
    ref, mask, ties = _compare(blasst, x, causal, Br, ln_lambda)
    if ln_lambda == -math.inf:
        assert (mask == 2).sum() == 0


@pytest.mark.parametrize("d,L,causal", [(128, 2048, True), (64, 1000, True),
                                         (128, 700, False)])
def test_dense_kernel_without_vote_equals_voting_kernel(blasst, d, L, causal):
    """ln lambda = -inf runs the 128x128 kernel built without the vote;
    -FLT_MAX runs the voting kernel with a threshold nothing reaches.  The
    arithmetic is the same, so the outputs agree bit for bit, and both
    match the oracle's dense result."""
    m = blasst
    x = planted_gap(1, 4, 2, L, L, d, block=128, gap=8.0, heavy_frac=0.03,
                    window=256, seed=config_seed(0, 900 + L + d),
                    device="cuda")
    nq = nk = -(-L // 128)
    st = m.Stats(mask_numel=4 * nq * nk)
    o1, l1 = m.blasst_prefill(x.q, x.k, x.v, causal=causal,
                              ln_lambda=-math.inf, stats=st)
    st2 = m.Stats(mask_numel=4 * nq * nk)
    o2, l2 = m.blasst_prefill(x.q, x.k, x.v, causal=causal,
                              ln_lambda=-3.4028234663852886e38, stats=st2)
    torch.cuda.synchronize()
    assert m.blasst_check_device_error()[0] == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(st.mask, st2.mask) and st.read() == st2.read()
    assert int((st.mask == 2).sum()) == 0
    ref = oracle.prefill(x.q, x.k, x.v, 1 / math.sqrt(d), causal, -math.inf,
                         128, 128)
    go = np.concatenate([P.to_np(o1)[b, h, i * 128:min((i + 1) * 128, L)]
                         for (b, h, i) in ref["units"]])
    ro = np.concatenate([ref["o"][u, :min(128, L - i * 128)]
                         for u, (b, h, i) in enumerate(ref["units"])])
    P.check_out(go, ro, "dense kernel without vote")


def test_prefill_rejects_bad_arguments(blasst):
    q = torch.zeros(1, 2, 128, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(blasst.BlasstError, match="INVALID_ARG"):
        blasst.blasst_prefill(q, q, q, ln_lambda=0.1)
    with pytest.raises(blasst.BlasstError, match="UNSUPPORTED"):
        blasst.blasst_prefill(q, q, q, Br=64, Bc=128)
    k_short = torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(blasst.BlasstError, match="INVALID_ARG"):
        blasst.blasst_prefill(q, k_short, k_short, causal=True)  # Lq > Lkv
    big = torch.zeros(1, 2, 128, 129, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(blasst.BlasstError, match="UNSUPPORTED"):
        blasst.blasst_prefill(big, big, big)


@pytest.mark.parametrize("which", ["s70", "dense"])
def test_prefill_full_size_sampled(blasst, which, capsys):
    """B 1, Hq 32, Hkv 8, L 32768, d 128, causal, 128x128 tiles, planted gap
    8 with sink + 2% heavy blocks + 512-token window boost, at the lambda
    calibrated to 70% sparsity and at the dense path; compared with the
    oracle on every one of the 256 tiles of heads 0 and 17 (the middle of
    the causal range included, where the long runs of skipped blocks and
    the lazy rescales happen) and on 64 random tiles of the other heads."""
    m = blasst
    L = 32768
    x = planted_gap(1, 32, 8, L, L, 128, block=128, gap=8.0, heavy_frac=0.02,
                    window=512, seed=config_seed(2), device="cuda")
    if which == "s70":
        cal = m.blasst_calibrate(0.70, mode="prefill", q=x.q, k=x.k, v=x.v,
                                 Br=128, Bc=128)
        assert abs(cal["achieved"] - 0.70) < 0.01
        lnl = cal["ln_lambda"]
    else:
        lnl = -math.inf
    rng = np.random.default_rng(17)
    others = [h for h in range(32) if h not in (0, 17)]
    units = [(0, h, i) for h in (0, 17) for i in range(256)]
    units += [(0, int(others[rng.integers(len(others))]),
               int(rng.integers(256))) for _ in range(64)]
    ref, mask, ties = _compare(m, x, True, 128, lnl, units=units,
                               check_stats_only=False)
    with capsys.disabled():  # shown in a quiet run too
        print(f"\nfull-size prefill ({which}, ln lambda {lnl}): {len(units)} "
              f"tiles, oracle sparsity {ref['skipped'] / ref['visited']:.4f}, "
              f"near-ties {ties}")
    if which == "dense":
        assert (mask == 2).sum() == 0
