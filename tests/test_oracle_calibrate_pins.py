"""Pins of the calibration oracle (``oracle.calibrate``) on the CPU.

The calibration reads s(ln lambda) off one oracle run (the per-pair
delta = max_r(m~ - m), which does not depend on lambda) instead of
re-running the forward at every step of the search.  What pins it:
  * fresh runs of the C oracle at many thresholds -- just below, at and just
    above individual deltas, and on a grid -- give exactly the visited and
    skipped counts and the skip mask that counting deltas predicts (this is
    the claim that the running max does not depend on the decisions, and
    the strict '<' of the criterion);
  * s is non-decreasing in ln lambda;
  * hand cases for the step edge (k-th smallest delta) and the search's
    end points (target 0, unreachable targets);
  * the bisection lands within its bracket above the step edge, and a fresh
    oracle run there reaches the target while one at the edge does not;
  * the log-space fit of lambda = a / L against numpy's least squares and
    against an exact inverse law.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import calibrate as C
from synth import planted_gap


def _prefill_sample():
    x = planted_gap(1, 4, 2, 512, 512, 64, block=64, gap=8.0, heavy_frac=0.1,
                    window=128, seed=4242)
    return x.q, x.k, x.v


def _decode_sample():
    x = planted_gap(3, 8, 2, 1, 3000, 64, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=4343)
    return x.q, x.k, x.v


def _probe_points(delta):
    """Thresholds at, just below and just above finite negative deltas, and
    a grid over [-12, 0]."""
    fin = np.unique(delta[np.isfinite(delta) & (delta < 0)])
    pick = fin[np.linspace(0, fin.size - 1, min(12, fin.size)).astype(int)]
    pts = [float(x) for x in pick]
    pts += [float(np.nextafter(x, -np.inf)) for x in pick]
    pts += [float(np.nextafter(x, np.inf)) for x in pick]
    pts += list(np.linspace(-12.0, 0.0, 13))
    return sorted(set(p for p in pts if p <= 0.0))


def test_prefill_step_function_matches_fresh_oracle_runs():
    q, k, v = _prefill_sample()
    sc = 1 / 8.0
    r0 = oracle.prefill(q, k, v, sc, True, 0.0, 64, 64)
    delta = C.deltas_from_result(r0)
    dmat = np.where(r0["mask"] > 0, r0["margin"], np.nan)
    assert delta.size == r0["visited"] > 0
    prev = -1.0
    for x in _probe_points(delta):
        r = oracle.prefill(q, k, v, sc, True, x, 64, 64)
        assert (r["visited"], r["skipped"]) == C.counts_at(delta, x), x
        want = np.where(np.isnan(dmat), 0, np.where(dmat < x, 2, 1))
        assert np.array_equal(r["mask"], want), x
        s = C.sparsity_at(delta, x)
        assert s >= prev
        prev = s


@pytest.mark.parametrize("S", [1, 3])
def test_decode_step_function_matches_fresh_oracle_runs(S):
    q, k, v = _decode_sample()
    sc = 1 / 8.0
    delta = C.deltas_decode(q, k, v, sc, 64, S)
    r0 = oracle.decode(q, k, v, sc, 0.0, 64, S)
    assert delta.size == r0["visited"]
    for x in _probe_points(delta)[::2]:
        r = oracle.decode(q, k, v, sc, x, 64, S)
        assert (r["visited"], r["skipped"]) == C.counts_at(delta, x), x
    # -inf: the dense path skips nothing
    assert C.counts_at(delta, -math.inf) == (delta.size, 0)


def test_step_edge_hand_cases():
    d = np.array([math.inf, -1.0, -2.0, -3.0, -5.0])
    # 5 visited pairs; s(x) = #{delta < x} / 5
    assert C.step_edge(d, 0.0) == -math.inf
    assert C.step_edge(d, 0.2) == -5.0      # one skip needed
    assert C.step_edge(d, 0.5) == -2.0      # ceil(2.5) = 3 skips
    assert C.step_edge(d, 0.6) == -2.0      # exactly 3 skips
    assert C.step_edge(d, 0.8) == -1.0      # 4 skips
    assert C.step_edge(d, 0.9) is None      # the +inf pair never skips
    assert C.sparsity_at(d, -2.0) == 0.4    # strict: delta = -2 not skipped
    assert C.sparsity_at(d, -1.9999) == 0.6
    # a delta >= 0 never skips at ln lambda <= 0
    assert C.step_edge(np.array([0.0, 0.5]), 0.5) is None
    # float comparison of k / n with the target, as the search does it
    assert C.skips_needed(1000, 0.7) == 700
    assert C.skips_needed(3, 1 / 3) == 1
    assert C.skips_needed(10, 0.0) == 0


def test_bisect_end_points():
    d = np.array([math.inf, -1.0, -2.0, -3.0, -70.0])
    r = C.bisect(d, 0.0)
    assert r["status"] == 0 and r["ln_lambda"] == -64.0 and r["iterations"] == 2
    r = C.bisect(d, 0.2)  # s(-64) = 0.2 already
    assert r["ln_lambda"] == -64.0 and r["achieved"] == pytest.approx(0.2)
    r = C.bisect(d, 0.9)
    assert r["status"] == 6 and r["ln_lambda"] == 0.0 and r["iterations"] == 1
    with pytest.raises(ValueError):
        C.bisect(d, 1.0)


@pytest.mark.parametrize("target", [0.2, 0.35, 0.45, 0.5])
def test_bisect_lands_on_the_step_and_a_fresh_run_agrees(target):
    q, k, v = _prefill_sample()
    sc = 1 / 8.0
    delta = C.deltas_prefill(q, k, v, sc, True, 64, 64)
    edge = C.step_edge(delta, target)
    assert edge is not None and edge > -64
    trace = []
    r = C.bisect(delta, target, tol=0.0, L=512, trace=trace)
    assert r["status"] == 0
    # on the first step that reaches the target: within the bracket above
    # its edge, or anywhere on it when that step's sparsity equals the
    # target exactly (the search stops at the first hi with s = target)
    x = r["ln_lambda"]
    assert edge < x <= 0.0
    assert C.counts_at(delta, x) == C.counts_at(delta, np.nextafter(edge, 0))
    assert x <= edge + 2 * C.BRACKET or r["achieved"] == target
    assert r["a"] == pytest.approx(math.exp(r["ln_lambda"]) * 512)
    # every evaluation is a correct comparison: lo side < target, hi side >=
    for x, vis, skp in trace:
        assert (skp / vis >= target) == (x > edge)
    # fresh runs of the forward oracle on both sides of the edge
    rr = oracle.prefill(q, k, v, sc, True, r["ln_lambda"], 64, 64)
    assert rr["skipped"] == r["skipped"] and rr["visited"] == r["visited"]
    assert rr["skipped"] / rr["visited"] >= target
    re = oracle.prefill(q, k, v, sc, True, edge, 64, 64)
    assert re["skipped"] / re["visited"] < target
    # with a tolerance the search may stop early, but only inside it
    r2 = C.bisect(delta, target, tol=0.02)
    assert target <= r2["achieved"] <= target + 0.02 or \
        r2["ln_lambda"] - edge <= 2 * C.BRACKET
    assert r2["iterations"] <= r["iterations"]


def test_unreachable_target_agrees_with_a_fresh_run_at_zero():
    q, k, v = _prefill_sample()
    delta = C.deltas_prefill(q, k, v, 1 / 8.0, True, 64, 64)
    s0 = C.sparsity_at(delta, 0.0)
    r0 = oracle.prefill(q, k, v, 1 / 8.0, True, 0.0, 64, 64)
    assert s0 == r0["skipped"] / r0["visited"]
    target = s0 + 0.05
    assert C.step_edge(delta, target) is None
    assert C.bisect(delta, target)["status"] == 6


def test_robust_decisions():
    d = np.array([math.inf, -1.0, -2.0, -3.0, -5.0])
    tr = []
    C.bisect(d, 0.5, tol=0.5, trace=tr)   # stops after the first halving
    assert C.robust_decisions(d, tr, 0.5, 1e-3)
    tr = []
    C.bisect(d, 0.5, trace=tr)            # converges onto delta = -2
    assert not C.robust_decisions(d, tr, 0.5, 1e-3)


def test_fit_a_is_the_log_space_least_squares_fit():
    rng = np.random.default_rng(5)
    Ls = np.array([4096, 16384, 65536])
    lam = 3.0 / Ls * np.exp(rng.normal(0, 0.3, 3))
    # least squares of ln lambda = ln a - ln L over the single unknown ln a
    sol, *_ = np.linalg.lstsq(np.ones((3, 1)), np.log(lam) + np.log(Ls),
                              rcond=None)
    assert C.fit_a(list(lam), list(Ls)) == pytest.approx(math.exp(sol[0]),
                                                        rel=1e-12)
    assert C.fit_a([2.0 / 1000, 2.0 / 8000], [1000, 8000]) == \
        pytest.approx(2.0, rel=1e-12)


def test_deviation_per_length():
    d1 = np.array([math.inf, -1.0, -2.0, -3.0])
    d2 = np.array([math.inf, -0.5, -4.0, -4.5])
    a = 1000.0 * math.exp(-1.5)             # ln(a / 1000) = -1.5
    dev = C.deviation({1000: d1, 2000: d2}, a, 0.5)
    # L 1000: x = -1.5 skips {-2, -3} -> s 0.5; L 2000: x = -2.19 -> {-4, -4.5}
    assert dev[1000] == pytest.approx(0.0)
    assert dev[2000] == pytest.approx(0.0)
    dev = C.deviation({1000: d1}, a, 0.75)
    assert dev[1000] == pytest.approx(0.25)
