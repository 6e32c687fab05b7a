"""Threshold calibration over a calibration sample sharded across ranks.

The forward itself needs no communication (every (sequence, KV head) unit is
independent).  The only cross-rank quantity is the pair of skip counters the
calibration bisects on: each rank runs statistics-only passes on its own
shard, the (visited, skipped) counts are summed across ranks, and every rank
takes the same bisection step from the same sums.  The search is the one
blasst_calibrate runs on a single device (smallest ln lambda in [lo, hi]
whose sparsity reaches the target, lambda = a / L with L = Lkv).
"""
from __future__ import annotations

import math
from typing import Callable, Optional

import torch


def _sparsity(vis, skp):
    return skp / vis if vis else 0.0


def calibrate_sharded(count_at: Callable[[float], tuple],
                      target: float, L: int, *, tol: float = 0.002,
                      lo: float = -64.0, hi: float = 0.0, max_iter: int = 100,
                      all_reduce: Optional[Callable[[torch.Tensor], None]] = None):
    """Bisection of ln(lambda) on counts summed over ranks.

    count_at(ln_lambda) -> (visited, skipped) on this rank's shard.
    all_reduce(t) sums the int64 tensor t in place across ranks (None for a
    single process).  Returns a dict like blasst_calibrate's.
    """
    if not (0.0 <= target < 1.0):
        raise ValueError("target must be in [0, 1)")
    it = 0

    def counts(lnl):
        nonlocal it
        it += 1
        v, s = count_at(lnl)
        t = torch.tensor([int(v), int(s)], dtype=torch.int64)
        if all_reduce is not None:
            all_reduce(t)
        return int(t[0]), int(t[1])

    def result(lnl, v, s, status):
        lam = math.exp(lnl)
        return dict(ln_lambda=lnl, lambda_=lam, a=lam * L,
                    achieved=_sparsity(v, s), L=L, iterations=it, visited=v,
                    skipped=s, status=status)

    v_hi, k_hi = counts(hi)
    s_hi = _sparsity(v_hi, k_hi)
    if s_hi < target:
        return result(hi, v_hi, k_hi, 6)  # BLASST_ERR_NO_CONVERGE
    v_lo, k_lo = counts(lo)
    if _sparsity(v_lo, k_lo) >= target:
        return result(lo, v_lo, k_lo, 0)
    while hi - lo > 1e-6 and s_hi - target > tol and it < max_iter:
        mid = 0.5 * (lo + hi)
        v, k = counts(mid)
        sm = _sparsity(v, k)
        if sm >= target:
            hi, s_hi, v_hi, k_hi = mid, sm, v, k
        else:
            lo = mid
    return result(hi, v_hi, k_hi, 0)


def decode_counter(q, k, v, *, Bc=64, num_splits=0, scale=None):
    """count_at for a decode shard on this rank's GPU (statistics-only
    passes of blasst_decode)."""
    from . import blasst as _b
    stats = _b.Stats(device=q.device)

    def count_at(lnl):
        stats.reset()
        _b.blasst_decode(q, k, v, scale=scale, ln_lambda=lnl, Bc=Bc,
                         num_splits=num_splits, stats=stats, stats_only=True)
        return stats.read()

    return count_at
