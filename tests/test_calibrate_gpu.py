"""GPU parity of the calibration (``blasst_calibrate`` through the C ABI)
against the calibration oracle.

The oracle's sparsity s(ln lambda) is exact (counts of per-pair deltas from
one float64 run); the library bisects on the kernels' float32 decisions.
The two differ only where a delta lies within the near-tie width (1e-3) of
a threshold the search evaluates.  So, per sample and target:
  * visited counts are equal (they do not depend on lambda);
  * when no comparison of the oracle's search is near a tie, the library
    takes the same steps: the same ln lambda bit for bit, the same number
    of passes;
  * always: the returned ln lambda is on the oracle's step for the target
    within the near-tie width, and the skip count at it equals the
    oracle's up to the deltas within that width (exactly, when none is).
The sharded search (``sharded.calibrate_sharded``) with the library's
statistics-only decode passes takes the same steps as ``blasst_calibrate``.
"""
import math

import numpy as np
import pytest
import torch

from oracle import calibrate as C
from synth import config_seed, planted_gap
from tests import _parity as P

pytestmark = pytest.mark.gpu

W = P.NEAR_TIE


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


@pytest.fixture(scope="module")
def prefill_sample():
    x = planted_gap(1, 8, 2, 4096, 4096, 128, block=128, gap=8.0,
                    heavy_frac=0.02, window=512, seed=config_seed(2, 77),
                    device="cuda")
    delta = C.deltas_prefill(x.q, x.k, x.v, 1 / math.sqrt(128), True, 128,
                             128)
    return x, delta


@pytest.fixture(scope="module")
def decode_sample(blasst):
    # 16 sequences x 8 KV heads x 16K keys in 4 splits of 64 blocks (a
    # split's first block is never skipped and short splits cap the
    # reachable sparsity)
    x = planted_gap(16, 32, 8, 1, 16384, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.03, seed=config_seed(1, 77), device="cuda")
    S = 4
    delta = C.deltas_decode(x.q, x.k, x.v, 1 / math.sqrt(128), 64, S)
    return x, delta, S


def _check(got, delta, target, tol, L):
    trace = []
    ref = C.bisect(delta, target, tol=tol, L=L, trace=trace)
    assert got["status"] == ref["status"] == 0
    assert got["visited"] == ref["visited"] == delta.size
    x = got["ln_lambda"]
    near = int(np.count_nonzero(np.abs(delta - x) < W))
    want = C.counts_at(delta, x)[1]
    assert abs(got["skipped"] - want) <= near, (got["skipped"], want, near)
    if near == 0:
        assert got["skipped"] == want
        assert got["achieved"] == want / delta.size
    # on the oracle's step for the target, within the near-tie width
    edge = C.step_edge(delta, target)
    assert edge is not None and x > edge - W
    assert C.sparsity_at(delta, min(0.0, x + W)) >= target
    if tol > 0 and near == 0:
        assert target <= got["achieved"] <= target + tol
    robust = C.robust_decisions(delta, trace, target, W)
    if robust:
        assert x == ref["ln_lambda"], (x, ref["ln_lambda"])
        assert got["iterations"] == ref["iterations"]
        assert got["a"] == pytest.approx(ref["a"], rel=1e-12)
    print(f"target {target} tol {tol}: ln_lambda {x:.7f} (oracle "
          f"{ref['ln_lambda']:.7f}, edge {edge:.7f}) achieved "
          f"{got['achieved']:.5f} passes {got['iterations']} "
          f"near-ties {near} robust {robust}")
    return robust


@pytest.mark.parametrize("target,tol", [(0.5, 0.002), (0.7, 0.002),
                                        (0.7, 0.0), (0.3, 0.0)])
def test_calibrate_prefill_matches_oracle(blasst, prefill_sample, target, tol):
    x, delta = prefill_sample
    got = blasst.blasst_calibrate(target, mode="prefill", q=x.q, k=x.k,
                                  v=x.v, Br=128, Bc=128, tol=tol)
    _check(got, delta, target, tol, 4096)
    assert got["L"] == 4096


@pytest.mark.parametrize("target,tol", [(0.5, 0.002), (0.7, 0.002),
                                        (0.7, 0.0)])
def test_calibrate_decode_matches_oracle(blasst, decode_sample, target, tol):
    x, delta, S = decode_sample
    got = blasst.blasst_calibrate(target, mode="decode", q=x.q, k=x.k, v=x.v,
                                  Bc=64, num_splits=S, tol=tol)
    _check(got, delta, target, tol, 16384)


def test_calibrate_decode_automatic_splits(blasst, decode_sample):
    """num_splits = 0 calibrates with the split count blasst_decode_splits
    gives (the decisions depend on it)."""
    x, _, _ = decode_sample
    S = blasst.blasst_decode_splits(16, 8, 16384, 64)
    a = blasst.blasst_calibrate(0.5, mode="decode", q=x.q, k=x.k, v=x.v,
                                Bc=64, num_splits=0)
    b = blasst.blasst_calibrate(0.5, mode="decode", q=x.q, k=x.k, v=x.v,
                                Bc=64, num_splits=S)
    for key in ("ln_lambda", "achieved", "iterations", "visited", "skipped"):
        assert a[key] == b[key], key


def test_calibrate_unreachable_and_zero_targets(blasst, decode_sample):
    x, delta, S = decode_sample
    s0 = C.sparsity_at(delta, 0.0)
    assert s0 < 0.99
    got = blasst.blasst_calibrate(0.99, mode="decode", q=x.q, k=x.k, v=x.v,
                                  Bc=64, num_splits=S,
                                  raise_on_no_converge=False)
    assert got["status"] == 6 and got["ln_lambda"] == 0.0
    assert got["iterations"] == 1
    near = int(np.count_nonzero(np.abs(delta) < W))
    assert abs(got["skipped"] - C.counts_at(delta, 0.0)[1]) <= near
    got = blasst.blasst_calibrate(0.0, mode="decode", q=x.q, k=x.k, v=x.v,
                                  Bc=64, num_splits=S)
    assert got["status"] == 0 and got["ln_lambda"] == -64.0


@pytest.mark.parametrize("target", [0.5, 0.7])
def test_sharded_search_equals_library_search(blasst, decode_sample, target):
    from dynamic_block_sparse_fa_b200.sharded import (calibrate_sharded,
                                                      decode_counter)
    x, _, S = decode_sample
    lib = blasst.blasst_calibrate(target, mode="decode", q=x.q, k=x.k,
                                  v=x.v, Bc=64, num_splits=S, tol=0.002)
    sh = calibrate_sharded(decode_counter(x.q, x.k, x.v, Bc=64, num_splits=S),
                           target, L=16384, tol=0.002)
    torch.cuda.synchronize()
    for key in ("ln_lambda", "achieved", "iterations", "visited", "skipped",
                "status"):
        assert sh[key] == lib[key], key
