"""Calibration oracle: the threshold lambda = a / L for a target sparsity --
TEST INFRASTRUCTURE ONLY (same import rule as the rest of ``oracle``).

What the pages fix ("BLASST: Dynamic BLocked Attention Sparsity via Softmax
Thresholding", gist.science summary, section 2 "Calibracao Automatica";
MLSys'26 reading notes, key observation 2): the threshold scales as
lambda = a / L with the context length L, and a is fitted on calibration
data so that a chosen fraction of the blocks is skipped.  The pages give no
search procedure; the reading taken here is a bisection of ln lambda, the
plainest search for a monotone quantity.

The step function.  Let delta(t, j) = max over the rows r of tile t of
(m~_r(j) - m_r(j)) for every visited (tile, block) pair, m_r(j) the running
max before block j (+inf for the tile's first visited block).  A pair is
skipped at threshold ln lambda exactly when delta < ln lambda (strict '<',
rows with no visible key in the block do not vote).  With ln lambda <= 0 a
skip happens only where every row has m~ < m, which leaves the running max
unchanged, so the running max after block j is the max of all m~ up to j
whatever was skipped: delta does not depend on lambda.  Hence the sparsity

    s(x) = #{pairs with delta < x} / #{visited pairs}

is a non-decreasing, right-open step function of x = ln lambda, with its
steps at the delta values.  ``deltas`` reads delta from one run of the
C oracle at ln lambda = 0 (its margin there is delta itself);
``tests/test_oracle_calibrate_pins.py`` checks s(x) against fresh oracle
runs at many x, so this reading is pinned, not assumed.

The search (``bisect``): keep lo with s(lo) < target and hi with
s(hi) >= target, start from [-64, 0], halve until the bracket is narrower
than 1e-6 or s(hi) is within ``tol`` above the target, return hi.  Its
infimum over all thresholds reaching the target is ``step_edge``: the
k-th smallest delta, k = ceil(target * visited).

Several lengths (``fit_a``): a = exp(mean_L ln(lambda*_L * L)), the least
squares fit of ln lambda = ln a - ln L; ``deviation`` is |s_L(a / L) -
target| per length.
"""
from __future__ import annotations

import math

import numpy as np

from . import decode as _decode
from . import lambda_fit as fit_a  # noqa: F401  (a = exp(mean ln(lambda*L)))
from . import prefill as _prefill

LN_LAMBDA_LO = -64.0
LN_LAMBDA_HI = 0.0
BRACKET = 1e-6
MAX_ITER = 100


def deltas_from_result(res):
    """delta of every visited pair from an oracle result computed at
    ln lambda = 0 (its margin is max_r(m~ - m) - 0).  Returns a float64
    1-D array (+inf for each tile's first visited block)."""
    mask = np.asarray(res["mask"])
    margin = np.asarray(res["margin"], dtype=np.float64)
    return np.ascontiguousarray(margin[mask > 0])


def deltas_prefill(q, k, v, scale, causal, Br, Bc, units=None, window=0,
                   n_threads=0):
    """delta per visited (query tile, KV block) pair of a prefill sample."""
    r = _prefill(q, k, v, scale, causal, 0.0, Br, Bc, units=units,
                 n_threads=n_threads, window=window)
    return deltas_from_result(r)


def deltas_decode(q, k, v, scale, Bc, num_splits, n_threads=0, window=0,
                  tile_heads=None):
    """delta per visited ((sequence, KV head, split), block) pair of a
    decode sample; ``num_splits`` is the resolved split count the call
    uses (the decisions depend on it)."""
    r = _decode(q, k, v, scale, 0.0, Bc, num_splits, n_threads=n_threads,
                window=window, tile_heads=tile_heads)
    return deltas_from_result(r)


def counts_at(delta, ln_lambda):
    """(visited, skipped) at threshold ln_lambda (<= 0, or -inf)."""
    delta = np.asarray(delta)
    if ln_lambda == -math.inf:
        return int(delta.size), 0
    return int(delta.size), int(np.count_nonzero(delta < ln_lambda))


def sparsity_at(delta, ln_lambda):
    v, s = counts_at(delta, ln_lambda)
    return s / v if v else 0.0


def skips_needed(visited, target):
    """Smallest k with k / visited >= target, compared in float64 exactly
    as the search compares s with the target (so 0.7 * 1000 rounding up to
    700.0000000000001 does not ask for 701)."""
    k = max(0, math.ceil(target * visited))
    while k > 0 and (k - 1) / visited >= target:
        k -= 1
    while k <= visited and k / visited < target:
        k += 1
    return k


def step_edge(delta, target):
    """Infimum of {x <= 0 : s(x) >= target}: the k-th smallest delta with
    k = ceil(target * visited); s reaches the target for every x above it
    (up to 0) and not at it.  -inf when the target is 0 (every x works);
    None when no x <= 0 reaches the target."""
    d = np.sort(np.asarray(delta, dtype=np.float64))
    n = d.size
    if n == 0:
        return None if target > 0 else -math.inf
    kneed = skips_needed(n, target)
    if kneed <= 0:
        return -math.inf
    if kneed > n:
        return None
    edge = float(d[kneed - 1])
    # s(0) counts delta < 0: unreachable when the k-th delta is >= 0
    return edge if edge < 0.0 else None


def bisect(delta, target, tol=0.0, lo=LN_LAMBDA_LO, hi=LN_LAMBDA_HI,
           bracket=BRACKET, max_iter=MAX_ITER, L=None, trace=None):
    """Bisection of ln lambda for the smallest threshold whose sparsity
    reaches ``target``.

    Evaluates hi (0) first, then lo (-64): status 6 (no threshold reaches
    the target) when s(hi) < target, lo itself when s(lo) >= target.  Then
    halves [lo, hi] while the bracket is wider than ``bracket``, s(hi) is
    more than ``tol`` above the target and fewer than ``max_iter``
    evaluations were made.  ``trace`` (a list) receives every evaluated
    (ln lambda, visited, skipped).  Returns a dict: ln_lambda, lambda_, a
    (= lambda * L when L is given), achieved, iterations, visited, skipped,
    status (0 or 6)."""
    if not (0.0 <= target < 1.0):
        raise ValueError("target must be in [0, 1)")
    it = 0

    def ev(x):
        nonlocal it
        it += 1
        v, s = counts_at(delta, x)
        if trace is not None:
            trace.append((x, v, s))
        return v, s

    def out(x, v, s, status):
        lam = math.exp(x)
        return dict(ln_lambda=x, lambda_=lam,
                    a=(lam * L if L is not None else None),
                    achieved=(s / v if v else 0.0), iterations=it,
                    visited=v, skipped=s, status=status)

    v_hi, k_hi = ev(hi)
    s_hi = k_hi / v_hi if v_hi else 0.0
    if s_hi < target:
        return out(hi, v_hi, k_hi, 6)
    v_lo, k_lo = ev(lo)
    if (k_lo / v_lo if v_lo else 0.0) >= target:
        return out(lo, v_lo, k_lo, 0)
    while hi - lo > bracket and s_hi - target > tol and it < max_iter:
        mid = 0.5 * (lo + hi)
        v, k = ev(mid)
        sm = k / v if v else 0.0
        if sm >= target:
            hi, s_hi, v_hi, k_hi = mid, sm, v, k
        else:
            lo = mid
    return out(hi, v_hi, k_hi, 0)


def robust_decisions(delta, trace, target, width):
    """True when every comparison s(x) >= target that the bisection took
    (the evaluations in ``trace``) would come out the same with every delta
    moved by up to ``width``: a computation whose deltas differ from these
    by less than ``width`` then takes exactly the same bisection steps."""
    delta = np.asarray(delta)
    n = delta.size
    if n == 0:
        return True
    for x, _, _ in trace:
        lo_cnt = int(np.count_nonzero(delta < x - width))
        hi_cnt = int(np.count_nonzero(delta < x + width))
        if (lo_cnt / n >= target) != (hi_cnt / n >= target):
            return False
    return True


def deviation(delta_by_length, a, target):
    """|s_L(ln(a / L)) - target| per length L (a dict L -> delta array);
    ln(a/L) is capped at 0 (lambda <= 1)."""
    out = {}
    for L, delta in delta_by_length.items():
        x = min(0.0, math.log(a) - math.log(L))
        out[L] = abs(sparsity_at(delta, x) - target)
    return out
