"""Multi-process host logic on CPU (gloo, world size 2).

* Sharded calibration: two ranks each hold half of the calibration sample;
  with counts summed across ranks, both take the same bisection steps and
  land on the same threshold as one process calibrating the whole sample.
  The skip counts come from the CPU oracle (no GPU here).
* The benchmark's max-over-ranks timing reduction.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from synth import planted_gap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _sample():
    x = planted_gap(4, 8, 2, 1, 2048, 64, decode=True, block=64, gap=8.0,
                    heavy_frac=0.05, seed=12345)
    return x.q, x.k, x.v


def _oracle_counter(q, k, v, S):
    def count_at(lnl):
        r = oracle.decode(q, k, v, 1.0 / 8.0, lnl, 64, S, n_threads=1)
        return r["visited"], r["skipped"]
    return count_at


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from dynamic_block_sparse_fa_b200.sharded import calibrate_sharded
        import bench
        q, k, v = _sample()
        per = q.shape[0] // world
        sl = slice(rank * per, (rank + 1) * per)
        res = calibrate_sharded(_oracle_counter(q[sl], k[sl], v[sl], 2), 0.6,
                                L=2048, all_reduce=dist.all_reduce)
        t = bench.reduce_max(float(10 + rank), dist, torch.device("cpu"))
        out[rank] = (res["ln_lambda"], res["achieved"], res["iterations"], t)
    finally:
        dist.destroy_process_group()


def test_sharded_calibration_matches_single_process():
    from dynamic_block_sparse_fa_b200.sharded import calibrate_sharded
    q, k, v = _sample()
    single = calibrate_sharded(_oracle_counter(q, k, v, 2), 0.6, L=2048)
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    assert r0[:3] == r1[:3], "ranks took different bisection steps"
    assert r0[0] == single["ln_lambda"] and r0[1] == single["achieved"]
    assert r0[3] == r1[3] == 11.0  # max over ranks
    # the calibrated threshold is on the right step of s(ln lambda): the
    # exact quantile from the oracle's margins (margin at ln lambda = 0 is
    # max_r(m~ - m) itself)
    r = oracle.decode(q, k, v, 1.0 / 8.0, 0.0, 64, 2)
    D = r["margin"][r["mask"] > 0]
    frac = float(np.mean(D < single["ln_lambda"]))
    assert frac == pytest.approx(single["achieved"], abs=1e-12)
    assert frac >= 0.6 and frac - 0.6 < 0.02


def test_single_process_calibration_edges():
    from dynamic_block_sparse_fa_b200.sharded import calibrate_sharded
    q, k, v = _sample()
    cnt = _oracle_counter(q, k, v, 1)
    r = calibrate_sharded(cnt, 0.0, L=2048)
    assert r["status"] == 0 and r["ln_lambda"] == -64.0
    r = calibrate_sharded(cnt, 0.999, L=2048)
    assert r["status"] == 6  # not reachable with ln lambda <= 0
    with pytest.raises(ValueError):
        calibrate_sharded(cnt, 1.0, L=2048)
