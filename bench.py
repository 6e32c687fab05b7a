#!/usr/bin/env python
"""Benchmark of the BLASST attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl blasst|reference]

One JSON line on stdout (rank 0).  The headline workload is the decode
configuration: batch 32 per GPU, Hq 32 / Hkv 8 (GQA 4:1), one query token
against a 32K-token contiguous bf16 KV cache, d 128, Bc 64, planted-gap
inputs (gap 8 nats, sink + 3% heavy blocks) with lambda calibrated to 70%
sparsity.  A step is one blasst_decode call (split kernel + merge kernel);
`value` is the algorithmic bytes those calls read and write (all of K, the V
of kept blocks, q, the split partials, o) per second, summed over ranks.

The same line carries:
  * decode at the lambda calibrated for 50% and at the dense path, near-tie
    counts of both from the oracle on sampled sequences;
  * the decode length sweep (batch 148, 8K-128K keys, a fitted at 32K);
  * the tiny prefill configuration (2 heads, 1024 tokens, d 64, ln lambda
    -6) against the full CPU oracle on all host cores and on one;
  * the prefill workload (B 1, Hq 32 / Hkv 8, 32K tokens, d 128, causal,
    128x128 tiles, lambda calibrated to 50% and 70%, and the dense path
    ln lambda = -inf), with the oracle timed on sampled tiles;
  * the prefill calibration sweep (4K-64K, targets 0-90%, deviation of the
    achieved sparsity from the target under lambda = a / L);
  * the roofline of the dominant kernels, the CPU oracle baseline, an
    end-to-end number with host buffers, and the SM clocks sampled (NVML)
    during the timed region.

Under torchrun each rank runs its own replica of the workload (independent
sequences; no collective on the data path) and the reported time is the
maximum over ranks ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("sparse attn latency & dense-equiv TFLOP/s vs λ=0 at 50/70% "
          "sparsity; decode GB/s")

DEC = dict(B=32, Hq=32, Hkv=8, Lkv=32768, d=128, Bc=64, target=0.70,
           window=4096)

# DRAM traffic of the dominant decode kernel per launch, relative to the
# algorithmic bytes of that launch, from one ncu capture of a smaller case
# (dram__bytes_read.sum + dram__bytes_write.sum over the algorithmic bytes of
# the captured launch).  The kernel reads K once and V only for kept blocks,
# so traffic grows with the algorithmic bytes; the ratio is applied to the
# benchmarked launch.  It holds only for the kernel source it was measured
# on (sha256 prefix below); a source without a capture reports null.
DECODE_TRAFFIC = dict(source="dynamic_block_sparse_fa_b200/csrc/decode_mma.cuh",
                      sha256_16="e08531a69c43a4a1",
                      ratio=(950.654720 + 4.106496) / 957.799424)
PRE = dict(B=1, Hq=32, Hkv=8, L=32768, d=128, Br=128, Bc=128, window=4096)
# B200 data-sheet figures, reported beside the measured denominators: HBM3e
# ~8 TB/s, dense bf16 tensor ~2.25 PFLOP/s
NOMINAL = dict(hbm_gbs=8000.0, bf16_tflops=2250.0)


def _measured_traffic(spec, algorithmic_bytes):
    """Bytes of DRAM traffic per launch, or None once the kernel source has
    changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, spec["source"]), "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    if spec["sha256_16"] is None or h != spec["sha256_16"]:
        return None
    return int(round(spec["ratio"] * algorithmic_bytes))


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return (float(pk["hbm_gbs"]), float(pk["bf16_tflops"]),
                float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# clocks (NVML, read only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, index, period_s=0.005):
        self.ok = False
        self.samples = []
        self.reasons = set()
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(
                self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS.items():
                    if r & getattr(nv, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------
def _r(x, nd):
    return None if (x is None or x != x) else round(x, nd)


def decode_bytes(B, Hq, Hkv, Lkv, d, Bc, S, kept_rows):
    """Bytes one decode call must move: all of K, V rows of kept blocks, q,
    split partials (written then read), o and lse."""
    k_bytes = 2 * Lkv * d * B * Hkv
    v_bytes = 2 * d * kept_rows
    q_bytes = 2 * B * Hq * d
    part = B * Hq * S * (d + 1) * 4 * 2
    out = B * Hq * d * 2 + B * Hq * 4
    return k_bytes + v_bytes + q_bytes + part + out


def kept_rows_from_mask(mask, Lkv, Bc):
    """Rows of V read: Bc per kept block, fewer for the ragged last block."""
    nk = mask.shape[-1]
    kept = (mask == 1)
    rows = kept.sum().item() * Bc
    last = Lkv - (nk - 1) * Bc
    if last != Bc:
        rows -= int(kept[..., nk - 1].sum().item()) * (Bc - last)
    return rows


def prefill_flops(visited, kept, Br, Bc, d):
    """Executed tensor FLOPs: QK^T on visited pairs + PV on kept pairs."""
    return 2.0 * Br * Bc * d * (visited + kept)


def dense_equiv_flops(B, Hq, L, d):
    return 4.0 * B * Hq * d * (L * (L + 1) / 2)


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def time_calls(fn, steps, warmup, stream, barrier=None):
    """Runs `warmup` untimed calls then times exactly `steps` calls with
    CUDA events on `stream`; synchronises (and barriers) on both sides.
    Returns the elapsed milliseconds."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return start.elapsed_time(end)


def time_calls_flushed(fn, steps, warmup, stream, flush):
    """Like time_calls for inputs that fit in L2: before each call the
    `flush` buffer (larger than L2) is rewritten, and only the calls are
    timed (a pair of CUDA events around each).  Returns the summed
    milliseconds of the `steps` timed calls."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = []
    for _ in range(steps):
        flush.fill_(1)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        ev.append((a, b))
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev)


def l2_flush_buffer(device, nbytes=256 << 20):
    return torch.empty(nbytes // 4, dtype=torch.float32, device=device)


def reduce_max(value, dist, device):
    """Maximum of a per-rank float over all ranks (the value itself when
    not distributed)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_decode_sample(q, k, v, ln_lambda, S, budget_s=10.0):
    """Times the CPU oracle (as it stands, all host cores) on the decode
    workload's own bytes, one sequence at a time, until about `budget_s`
    seconds of CPU work; returns (GB/s of algorithmic bytes, seconds,
    threads, description of the sample)."""
    import oracle
    d = q.shape[-1]
    threads = os.cpu_count() or 1
    total_bytes, total_t, n = 0, 0.0, 0
    B = q.shape[0]
    while total_t < budget_s and n < 16 * B:
        b = n % B
        qs, ks, vs = q[b:b + 1].cpu(), k[b:b + 1].cpu(), v[b:b + 1].cpu()
        t0 = time.perf_counter()
        res = oracle.decode(qs, ks, vs, 1.0 / math.sqrt(d), ln_lambda,
                            DEC["Bc"], S, n_threads=threads)
        total_t += time.perf_counter() - t0
        kept_rows = kept_rows_from_mask(torch.from_numpy(res["mask"]),
                                        k.shape[2], DEC["Bc"])
        total_bytes += decode_bytes(1, q.shape[1], k.shape[1], k.shape[2], d,
                                    DEC["Bc"], S, kept_rows)
        n += 1
    return total_bytes / total_t / 1e9, total_t, threads, (
        f"{n} sequence passes over the batch of {B} (each: all {k.shape[1]} "
        f"KV heads x {k.shape[2]} keys), same splits and lambda, "
        f"~{budget_s:.0f} s budget")


NEAR_TIE = 1e-3       # |margin| below this: the decision may differ by rounding
DEC_TIE_SEQS = (0, 11, 22, 31)


def _near(margin):
    import numpy as np
    m = np.nan_to_num(margin, nan=1.0, posinf=1.0, neginf=1.0)
    return int((np.abs(m) < NEAR_TIE).sum())


def decode_near_ties(q, k, v, ln_lambda, S, seqs):
    """Near-tie count of the decode decisions on sampled sequences, from the
    oracle's per-pair margins at this ln lambda."""
    import oracle
    d = q.shape[-1]
    n = 0
    for b in seqs:
        if b >= q.shape[0]:
            continue
        r = oracle.decode(q[b:b + 1], k[b:b + 1], v[b:b + 1],
                          1.0 / math.sqrt(d), ln_lambda, DEC["Bc"], S)
        n += _near(r["margin"])
    return n


# ---------------------------------------------------------------------------
# the product arm
# ---------------------------------------------------------------------------
def run_blasst(args):
    import dynamic_block_sparse_fa_b200 as bl
    from synth import config_seed, planted_gap, planted_gap_kv_inplace

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier(device_ids=[local])

    hbm_peak, tf_burst, tf_sust, peak_kind = _peaks()
    stream = torch.cuda.current_stream()

    line = None
    if not args.no_decode:
        line = run_decode(args, bl, dev, stream, world, rank, local, dist,
                          barrier, hbm_peak, peak_kind)
    else:
        line = {"metric": METRIC, "value": None, "unit": "GB/s",
                "n_gpus": world, "note": "decode leg skipped"}

    # ---------------- MQA and MLA decode (rank 0) ----------------
    if rank == 0 and not args.no_mla and not args.no_decode:
        line["decode_mqa"] = run_mqa(args, bl, dev, stream, hbm_peak)
        line["decode_mla"] = run_mla(args, bl, dev, stream, hbm_peak, tf_burst)

    # ---------------- the remaining workloads (rank 0) ----------------
    if rank == 0 and not args.no_sweeps and not args.no_decode:
        line["decode_sweep"] = run_decode_sweep(args, bl, dev, stream, hbm_peak)
    if rank == 0 and not args.no_prefill:
        line["tiny_prefill"] = run_tiny_prefill(args, bl, dev, stream, tf_burst)
        line["prefill"], line["roofline_prefill"] = run_prefill(
            args, bl, dev, stream, tf_burst, peak_kind)
        if not args.no_sweeps:
            line["prefill_sweep"] = run_prefill_sweep(args, bl, dev, stream,
                                                      tf_burst)
    barrier()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_decode(args, bl, dev, stream, world, rank, local, dist, barrier,
               hbm_peak, peak_kind):
    from synth import config_seed, planted_gap_kv_inplace
    B, Hq, Hkv, Lkv, d, Bc = (DEC[x] for x in ("B", "Hq", "Hkv", "Lkv", "d", "Bc"))
    B = args.decode_batch
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=dev)
    k = torch.empty(B, Hkv, Lkv, d, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=Bc, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(1, 1000 * rank))
    if args.decode_lnl is None:
        cal = bl.blasst_calibrate(DEC["target"], mode="decode", q=q, k=k, v=v,
                                  Bc=Bc, tol=0.002)
    else:
        cal = {"ln_lambda": args.decode_lnl, "iterations": 0,
               "a": math.exp(args.decode_lnl) * Lkv}
    lnl = cal["ln_lambda"]
    S = bl.blasst_decode_splits(B, Hkv, Lkv, Bc)
    nk = -(-Lkv // Bc)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(bl.blasst_decode_workspace_size(B, Hq, d, S),
                     dtype=torch.uint8, device=dev)
    st = bl.Stats(device=dev, mask_numel=B * Hkv * nk)
    bl.blasst_decode(q, k, v, ln_lambda=lnl, o=o, lse=lse, workspace=ws, stats=st)
    torch.cuda.synchronize()
    vis, skp = st.read()
    kept_rows = kept_rows_from_mask(st.mask.view(B, Hkv, nk), Lkv, Bc)
    by_call = decode_bytes(B, Hq, Hkv, Lkv, d, Bc, S, kept_rows)
    by_dense = decode_bytes(B, Hq, Hkv, Lkv, d, Bc, S, B * Hkv * Lkv)

    def sparse_call():
        bl.blasst_decode(q, k, v, ln_lambda=lnl, o=o, lse=lse, workspace=ws)

    def dense_call():
        bl.blasst_decode(q, k, v, ln_lambda=-math.inf, o=o, lse=lse, workspace=ws)

    K, W = args.steps, args.warmup
    with ClockSampler(local) as clk:
        ms = time_calls(sparse_call, K, W, stream, barrier)
    ms_max = reduce_max(ms, dist, dev)
    ms_dense = (time_calls(dense_call, K, W, stream, barrier)
                if not args.no_dense else float("nan"))
    t_call = ms_max / K / 1e3
    value = by_call * world / t_call / 1e9  # GB/s over all ranks
    achieved = by_call / t_call / 1e9       # per GPU, per call

    # ---------------- end to end (host buffers) ----------------
    # One pinned staging buffer per direction: q and the new token's K/V
    # rows in, o and lse out, so that each step makes one copy each way.
    qb, kvb = B * Hq * d * 2, 2 * B * Hkv * d * 2
    ob, lb = B * Hq * d * 2, B * Hq * 4
    in_h = torch.empty(qb + kvb, dtype=torch.uint8).pin_memory()
    in_h[:qb].copy_(q.cpu().contiguous().view(-1).view(torch.uint8))
    in_h[qb:].copy_(torch.stack([k[:, :, Lkv - 1], v[:, :, Lkv - 1]]).cpu()
                    .contiguous().view(-1).view(torch.uint8))
    in_d = torch.empty_like(in_h, device=dev)
    q_in = in_d[:qb].view(torch.bfloat16).view(B, Hq, d)
    kv_in = in_d[qb:].view(torch.bfloat16).view(2, B, Hkv, d)
    out_d = torch.empty(ob + lb, dtype=torch.uint8, device=dev)
    o_out = out_d[:ob].view(torch.bfloat16).view(B, Hq, d)
    lse_out = out_d[ob:].view(torch.float32).view(B, Hq)
    out_h = torch.empty(ob + lb, dtype=torch.uint8).pin_memory()

    def e2e_ops():
        in_d.copy_(in_h, non_blocking=True)
        k[:, :, Lkv - 1].copy_(kv_in[0])
        v[:, :, Lkv - 1].copy_(kv_in[1])
        bl.blasst_decode(q_in, k, v, ln_lambda=lnl, o=o_out, lse=lse_out,
                         workspace=ws)
        out_h.copy_(out_d, non_blocking=True)

    # The step's copies and launches as one CUDA graph (captured once,
    # replayed every step): the host pays one launch instead of ~10.
    graph = None
    if not args.no_e2e and not args.no_graph:
        try:
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                for _ in range(2):
                    e2e_ops()
            stream.wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                e2e_ops()
            torch.cuda.synchronize()
        except Exception as exc:  # report and time the launches one by one
            graph = None
            print(f"e2e graph capture failed ({exc}); timing eager steps",
                  file=sys.stderr)

    def e2e_step():
        if graph is not None:
            graph.replay()
        else:
            e2e_ops()
        stream.synchronize()  # the host reads the step's result

    ms_e2e = (time_calls(e2e_step, K, W, stream, barrier)
              if not args.no_e2e else float("nan"))
    e2e_max = reduce_max(ms_e2e, dist, dev)
    e2e_value = by_call * world / (e2e_max / K / 1e3) / 1e9
    h2d = in_h.numel()
    d2h = out_h.numel()

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_max / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "accumulate": "f32",
        "data": "synthetic planted-gap (seeded; gap 8 nats, sink + 3% heavy blocks)",
        "config": {
            "workload": (f"decode B{B} Hq{Hq} Hkv{Hkv} Lkv{Lkv} d{d} Bc{Bc}, " + (
                f"lambda calibrated to {DEC['target']:.0%} sparsity"
                if args.decode_lnl is None else f"fixed ln lambda {lnl}")),
            "global_batch": B * world, "seq_len": Lkv,
            "parallelism": f"replicas{world}", "splits": S,
            "ln_lambda": lnl, "a": cal["a"], "sparsity": skp / vis,
            "l2": "inputs larger than L2 (K+V 4.3 GB per GPU), no flush",
        },
        "decode": {
            "us": round(ms_max / K * 1e3, 2),
            "dense_us": _r(ms_dense / K * 1e3, 2),
            "speedup_vs_dense": _r(ms_dense / ms_max, 4),
            "GBps": round(achieved, 1),
            "dense_GBps": _r(by_dense / (ms_dense / K / 1e3) / 1e9, 1),
            "bytes_per_call": by_call,
            "sparsity": skp / vis,
            "calibration_iterations": cal["iterations"],
        },
        "roofline": {
            "bound": "hbm", "kernel": "decode_mma_kernel (+ merge)",
            "achieved": round(achieved, 1), "peak": hbm_peak,
            "peak_kind": peak_kind + " copy bandwidth", "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4),
            "nominal_peak": NOMINAL["hbm_gbs"],
            "frac_of_nominal": round(achieved / NOMINAL["hbm_gbs"], 4),
            "traffic": _measured_traffic(DECODE_TRAFFIC, by_call),
            "traffic_unit": "bytes per launch",
        },
        "e2e": {"value": _r(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": _r(e2e_max / K, 4),
                "what": "h2d of q and the new token's K/V rows, decode, "
                        "d2h of o and lse, host sync, per step",
                "cuda_graph": graph is not None},
        "gpu_launches": 2 * K,
        "clocks": clk.summary(),
    }

    # ---------------- 50% calibrated sparsity, same inputs ----------------
    if args.no_s50:
        return finish_decode(args, bl, dev, stream, q, k, v, lnl, cal, S, ms_max,
                             by_call, rank, world, line)
    cal50 = bl.blasst_calibrate(0.50, mode="decode", q=q, k=k, v=v, Bc=Bc,
                                tol=0.002)
    st50 = bl.Stats(device=dev, mask_numel=B * Hkv * nk)
    bl.blasst_decode(q, k, v, ln_lambda=cal50["ln_lambda"], o=o, lse=lse,
                     workspace=ws, stats=st50)
    torch.cuda.synchronize()
    v50, k50 = st50.read()
    by50 = decode_bytes(B, Hq, Hkv, Lkv, d, Bc, S,
                        kept_rows_from_mask(st50.mask.view(B, Hkv, nk), Lkv, Bc))
    ms50 = time_calls(lambda: bl.blasst_decode(
        q, k, v, ln_lambda=cal50["ln_lambda"], o=o, lse=lse, workspace=ws),
        K, W, stream, barrier)
    ms50 = reduce_max(ms50, dist, dev)
    line["decode"]["s50"] = {
        "ln_lambda": cal50["ln_lambda"], "a": cal50["a"],
        "sparsity": k50 / v50, "us": round(ms50 / K * 1e3, 2),
        "GBps": round(by50 / (ms50 / K / 1e3) / 1e9, 1),
        "hbm_frac": round(by50 / (ms50 / K / 1e3) / 1e9 / hbm_peak, 4),
        "speedup_vs_dense": _r(ms_dense / ms50, 4)}
    line["decode"]["hbm_frac_dense"] = _r(
        by_dense / (ms_dense / K / 1e3) / 1e9 / hbm_peak, 4)
    # near-ties over the whole batch, from the library's own margins
    lib_ties = {}
    for key, l in (("s70", lnl), ("s50", cal50["ln_lambda"])):
        stm = bl.Stats(device=dev, mask_numel=B * Hkv * nk, margin=True)
        bl.blasst_decode(q, k, v, ln_lambda=l, o=o, lse=lse, workspace=ws,
                         stats=stm)
        torch.cuda.synchronize()
        lib_ties[key] = stm.near_ties()
        del stm
    line["decode"]["near_ties_library"] = dict(
        lib_ties, what=f"all {B * Hkv * nk} pairs of the call, from the "
                       f"library's decision margins (|margin| < {NEAR_TIE})")
    if rank == 0 and not args.no_cpu:
        line["decode"]["near_ties"] = {
            key: decode_near_ties(q, k, v, l, S, DEC_TIE_SEQS)
            for key, l in (("s70", lnl), ("s50", cal50["ln_lambda"]))}
        line["decode"]["near_ties"]["sample"] = (
            f"oracle margins of sequences {DEC_TIE_SEQS} (all heads); a pair "
            f"is a near-tie when |max_r(m~ - m) - ln lambda| < {NEAR_TIE}")

    return finish_decode(args, bl, dev, stream, q, k, v, lnl, cal, S, ms_max,
                         by_call, rank, world, line)


def finish_decode(args, bl, dev, stream, q, k, v, lnl, cal, S, ms_max, by_call,
                  rank, world, line):
    """The decode variants on the same cache, and the CPU oracle baseline."""
    K = args.steps
    if not args.no_paged:
        line["decode_paged"] = run_decode_paged(args, bl, dev, stream, q, k, v,
                                                lnl, cal["a"], S, ms_max / K,
                                                by_call)
    if not args.no_window:
        line["decode_window"] = run_decode_window(args, bl, q, k, v, lnl,
                                                  stream)
        ws = torch.empty(bl.blasst_decode_workspace_size(
            q.shape[0], q.shape[1], q.shape[2], S), dtype=torch.uint8, device=dev)
        line["decode_batched"] = run_decode_batched(args, bl, q, k, v, lnl, S,
                                                    ws, ms_max / K)

    # ---------------- CPU oracle baseline (rank 0, N = 1) ----------------
    if rank == 0 and world == 1 and not args.no_cpu:
        gbs, secs, threads, sample = cpu_oracle_decode_sample(
            q, k, v, lnl, S, budget_s=args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s",
                                "cores": threads, "kind": "oracle",
                                "sample": sample, "seconds": round(secs, 2)}
    return line


def paged_kept_rows(mask, lens, Bc):
    """Rows of V a paged call reads: Bc per kept block, fewer for each
    sequence's ragged last block.  mask [B, Hkv, nk_max]."""
    kept = (mask == 1)
    rows = kept.sum().item() * Bc
    for b, L in enumerate(lens):
        nk = -(-L // Bc)
        last = L - (nk - 1) * Bc
        if nk and last != Bc:
            rows -= int(kept[b, :, nk - 1].sum().item()) * (Bc - last)
    return rows


def run_decode_paged(args, bl, dev, stream, q, k, v, lnl, a, S, ms_contig,
                     by_contig):
    """Paged-cache decode on the same workload: the contiguous cache's tokens
    in a shuffled pool (64- and 16-token pages), then a variable-length
    batch (lengths uniform in [1K, 64K]) with the per-sequence threshold
    lambda = a / L_b."""
    from synth import config_seed, paginate, planted_gap_kv_inplace
    B, Hq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    Bc = DEC["Bc"]
    K, W = args.steps, args.warmup
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    out = {}
    for ps in (64, 16):
        pk = paginate(k, v, [Lkv] * B, ps, seed=config_seed(7, ps))
        ws = torch.empty(bl.blasst_decode_workspace_size(B, Hq, d, S),
                         dtype=torch.uint8, device=dev)
        fn = lambda: bl.blasst_decode_paged(
            q, pk.k_pages, pk.v_pages, pk.block_table, pk.seq_lens,
            max_seq_len=Lkv, ln_lambda=lnl, num_splits=S, o=o, lse=lse,
            workspace=ws)
        ms = time_calls(fn, K, W, stream) / K
        out[f"uniform_page{ps}"] = {
            "workload": f"same tokens as the contiguous run, shuffled pool of "
                        f"{ps}-token pages",
            "us": round(ms * 1e3, 2), "GBps": round(by_contig / (ms / 1e3) / 1e9, 1),
            "vs_contiguous": round(ms_contig / ms, 4)}
        del pk, ws
        torch.cuda.empty_cache()

    # variable lengths
    g = torch.Generator().manual_seed(config_seed(8))
    lens = torch.randint(1024, 65536 + 1, (B,), generator=g).tolist()
    Lmax = max(lens)
    kk = torch.empty(B, Hkv, Lmax, d, dtype=torch.bfloat16, device=dev)
    vv = torch.empty_like(kk)
    qq = torch.empty_like(q)
    planted_gap_kv_inplace(kk, vv, qq, block=Bc, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(8, 1))
    pk = paginate(kk, vv, lens, 16, seed=config_seed(8, 2))
    del kk, vv
    torch.cuda.empty_cache()
    Sv = bl.blasst_decode_splits(B, Hkv, Lmax, Bc)
    nk_max = -(-Lmax // Bc)
    ws = torch.empty(bl.blasst_decode_workspace_size(B, Hq, d, Sv),
                     dtype=torch.uint8, device=dev)
    st = bl.Stats(device=dev, mask_numel=B * Hkv * nk_max)
    ln_a = math.log(a)
    kw = dict(max_seq_len=Lmax, ln_lambda=ln_a, per_length=True,
              num_splits=Sv, o=o, lse=lse, workspace=ws)
    bl.blasst_decode_paged(qq, pk.k_pages, pk.v_pages, pk.block_table,
                           pk.seq_lens, stats=st, **kw)
    torch.cuda.synchronize()
    vis, skp = st.read()
    rows = paged_kept_rows(st.mask.view(B, Hkv, nk_max), lens, Bc)
    by = (2 * d * Hkv * sum(lens) + 2 * d * rows + 2 * B * Hq * d
          + B * Hq * Sv * (d + 1) * 4 * 2 + B * Hq * d * 2 + B * Hq * 4)
    fn = lambda: bl.blasst_decode_paged(qq, pk.k_pages, pk.v_pages,
                                        pk.block_table, pk.seq_lens, **kw)
    ms = time_calls(fn, K, W, stream) / K
    kw_dense = dict(kw, ln_lambda=-math.inf, per_length=False)
    fn_d = lambda: bl.blasst_decode_paged(qq, pk.k_pages, pk.v_pages,
                                          pk.block_table, pk.seq_lens,
                                          **kw_dense)
    ms_d = time_calls(fn_d, K, W, stream) / K
    out["varlen_page16"] = {
        "workload": f"B{B} lengths uniform in [1K, 64K] (sum {sum(lens)}), "
                    f"shuffled pool of 16-token pages, lambda = a / L_b "
                    f"with a = {a:.4g}",
        "splits": Sv, "sparsity": skp / vis, "us": round(ms * 1e3, 2),
        "GBps": round(by / (ms / 1e3) / 1e9, 1), "bytes_per_call": by,
        "dense_us": round(ms_d * 1e3, 2),
        "speedup_vs_dense": round(ms_d / ms, 4)}
    del pk, ws
    torch.cuda.empty_cache()
    return out


def run_prefill(args, bl, dev, stream, tf_peak, peak_kind):
    from synth import config_seed, planted_gap
    B, Hq, Hkv, L, d, Br, Bc = (PRE[x] for x in ("B", "Hq", "Hkv", "L", "d", "Br", "Bc"))
    L = args.prefill_L
    x = planted_gap(B, Hq, Hkv, L, L, d, block=Br, gap=8.0, heavy_frac=0.02,
                    window=512, seed=config_seed(2), device=dev)
    q, k, v = x.q, x.k, x.v
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device=dev)
    K, W = args.prefill_steps, args.warmup
    out = {"workload": f"prefill B{B} Hq{Hq} Hkv{Hkv} L{L} d{d} causal {Br}x{Bc}"}
    dense_flops = dense_equiv_flops(B, Hq, L, d)

    def measure(lnl):
        st = bl.Stats(device=dev)
        bl.blasst_prefill(q, k, v, ln_lambda=lnl, Br=Br, Bc=Bc, o=o, lse=lse,
                          stats=st)
        torch.cuda.synchronize()
        vis, skp = st.read()
        fn = lambda: bl.blasst_prefill(q, k, v, ln_lambda=lnl, Br=Br, Bc=Bc,
                                       o=o, lse=lse)
        ms = time_calls(fn, K, W, stream) / K
        ex = prefill_flops(vis, vis - skp, Br, Bc, d)
        return {"ln_lambda": lnl, "sparsity": skp / vis, "us": round(ms * 1e3, 1),
                "dense_equiv_tflops": round(dense_flops / (ms / 1e3) / 1e12, 1),
                "executed_tflops": round(ex / (ms / 1e3) / 1e12, 1),
                "tensor_frac": round(ex / (ms / 1e3) / 1e12 / tf_peak, 4)}

    if args.prefill_lnl is not None:
        out["fixed"] = measure(args.prefill_lnl)
        r = out["fixed"]
        return out, {"bound": "tensor", "kernel": "prefill2_kernel<128>",
                     "achieved": r["executed_tflops"], "peak": tf_peak,
                     "peak_kind": peak_kind + " bf16 burst", "unit": "TFLOP/s",
                     "frac": r["tensor_frac"],
                     "nominal_peak": NOMINAL["bf16_tflops"],
                     "frac_of_nominal": round(r["executed_tflops"]
                                              / NOMINAL["bf16_tflops"], 4),
                     "traffic": None}
    dense = measure(-math.inf)
    out["dense"] = dense
    # the skipping kernel at a threshold that never skips: the dense path
    # with the vote and the decision hand-offs still in it
    vote = measure(-3.4028234663852886e38)
    out["dense_with_vote"] = vote
    out["vote_overhead"] = round(vote["us"] / dense["us"] - 1.0, 4)
    for tgt, key in ((0.5, "s50"), (0.7, "s70")):
        cal = bl.blasst_calibrate(tgt, mode="prefill", q=q, k=k, v=v, Br=Br,
                                  Bc=Bc, tol=0.002)
        r = measure(cal["ln_lambda"])
        r["a"] = cal["a"]
        r["speedup_vs_dense"] = round(dense["us"] / r["us"], 4)
        out[key] = r
    nq_, nk_ = -(-L // Br), -(-L // Bc)
    for key in ("s50", "s70"):
        stm = bl.Stats(device=dev, mask_numel=B * Hq * nq_ * nk_, margin=True)
        bl.blasst_prefill(q, k, v, ln_lambda=out[key]["ln_lambda"], Br=Br,
                          Bc=Bc, o=o, lse=lse, stats=stm)
        torch.cuda.synchronize()
        out[key]["near_ties_library"] = stm.near_ties()
        del stm
    if not args.no_cpu:
        tiles = [(0, h, i) for h in (0, 17) for i in range(0, 256, 4)]
        for key in ("s50", "s70"):
            _, smp = prefill_oracle_sample(q, k, v, out[key]["ln_lambda"],
                                           tiles, Br)
            out[key]["near_ties_sample"] = smp["near_ties"]
            if key == "s70":
                total_vis = B * Hq * (L // Br) * (L // Br + 1) // 2
                out["cpu_baseline_prefill"] = {
                    "value": round(smp["tflops"], 6), "unit": "TFLOP/s executed",
                    "kind": "oracle", "cores": smp["cores"],
                    "seconds": smp["seconds"],
                    "sample": f"{len(tiles)} query tiles (every 4th tile of "
                              f"heads 0 and 17) at the 70% lambda: "
                              f"{smp['visited']} of {total_vis} visited pairs "
                              f"({smp['visited'] / total_vis:.2%})"}
        out["near_ties_sample"] = (
            "oracle margins on the CPU-baseline tiles; a pair is a near-tie "
            f"when |max_r(m~ - m) - ln lambda| < {NEAR_TIE}")
    if not args.no_window:
        out["window"] = run_prefill_window(args, bl, q, k, v, o, lse,
                                           out["s70"]["ln_lambda"], stream,
                                           tf_peak)
    if not args.no_backward:
        out["backward"] = run_prefill_backward(args, bl, q, k, v,
                                               out["s70"]["ln_lambda"], stream,
                                               tf_peak)
    best = out["s70"]
    roof = {"bound": "tensor", "kernel": "prefill2_kernel<128> at 70%",
            "achieved": best["executed_tflops"], "peak": tf_peak,
            "peak_kind": peak_kind + " bf16 burst", "unit": "TFLOP/s",
            "frac": best["tensor_frac"],
            "nominal_peak": NOMINAL["bf16_tflops"],
            "frac_of_nominal": round(best["executed_tflops"]
                                     / NOMINAL["bf16_tflops"], 4),
            "traffic": None}
    return out, roof


def prefill_oracle_sample(q, k, v, ln_lambda, units, Br=128):
    """The CPU oracle (all host cores) on sampled query tiles of the
    prefill workload: seconds, executed FLOPs per second and the near-tie
    count of the sample, and the sample's share of the visited pairs."""
    import oracle
    d = q.shape[-1]
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    r = oracle.prefill(q, k, v, 1.0 / math.sqrt(d), True, ln_lambda, Br, Br,
                       units=units, n_threads=threads)
    secs = time.perf_counter() - t0
    ex = prefill_flops(r["visited"], r["visited"] - r["skipped"], Br, Br, d)
    return r, {"seconds": round(secs, 3), "cores": threads,
               "tflops": ex / secs / 1e12, "visited": r["visited"],
               "near_ties": _near(r["margin"])}


def run_tiny_prefill(args, bl, dev, stream, tf_peak):
    """The tiny prefill configuration: B 1, Hq = Hkv = 2, L 1024, d 64,
    causal, 64 x 64 tiles, ln lambda = -6, planted gap 8 (sink + 3% heavy
    blocks).  GPU time with L2 flushed between calls; the full CPU oracle
    on all host cores and on one; parity of the GPU result."""
    import numpy as np
    import oracle
    from synth import config_seed, planted_gap
    B, H, L, d, T, lnl = 1, 2, 1024, 64, 64, -6.0
    x = planted_gap(B, H, H, L, L, d, block=T, gap=8.0, heavy_frac=0.03,
                    seed=config_seed(0), device=dev)
    nq = nk = L // T
    st = bl.Stats(device=dev, mask_numel=B * H * nq * nk)
    o, lse = bl.blasst_prefill(x.q, x.k, x.v, ln_lambda=lnl, Br=T, Bc=T,
                               stats=st)
    torch.cuda.synchronize()
    vis, skp = st.read()
    flush = l2_flush_buffer(dev)
    steps = max(args.steps, 100)
    ms = time_calls_flushed(lambda: bl.blasst_prefill(
        x.q, x.k, x.v, ln_lambda=lnl, Br=T, Bc=T, o=o, lse=lse),
        steps, args.warmup, stream, flush) / steps
    od, ld = torch.empty_like(o), torch.empty_like(lse)
    ms_d = time_calls_flushed(lambda: bl.blasst_prefill(
        x.q, x.k, x.v, Br=T, Bc=T, o=od, lse=ld),
        steps, args.warmup, stream, flush) / steps
    del flush
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    ref = oracle.prefill(x.q, x.k, x.v, 1.0 / math.sqrt(d), True, lnl, T, T,
                         n_threads=threads)
    t_all = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.prefill(x.q, x.k, x.v, 1.0 / math.sqrt(d), True, lnl, T, T,
                   n_threads=1)
    t_one = time.perf_counter() - t0
    o_np = o.float().cpu().numpy()
    err = np.concatenate([np.abs(o_np[b, h, i * T:(i + 1) * T] - ref["o"][u])
                          .ravel() for u, (b, h, i) in enumerate(ref["units"])])
    gm = st.mask.cpu().numpy().reshape(B, H, nq, nk)
    got = np.stack([gm[b, h, i] for (b, h, i) in ref["units"]])
    near = np.abs(np.nan_to_num(ref["margin"], nan=1, posinf=1)) < NEAR_TIE
    ex = prefill_flops(vis, vis - skp, T, T, d)
    dense_eq = dense_equiv_flops(B, H, L, d)
    return {
        "workload": f"prefill B{B} Hq{H} Hkv{H} L{L} d{d} causal {T}x{T}, "
                    f"ln lambda {lnl}",
        "l2": "L2 flushed (256 MB write) before every timed call",
        "sparsity": skp / vis, "us": round(ms * 1e3, 2),
        "dense_us": round(ms_d * 1e3, 2),
        "speedup_vs_dense": round(ms_d / ms, 4),
        "dense_equiv_tflops": round(dense_eq / (ms / 1e3) / 1e12, 3),
        "executed_tflops": round(ex / (ms / 1e3) / 1e12, 3),
        "tensor_frac": round(ex / (ms / 1e3) / 1e12 / tf_peak, 5),
        "oracle_seconds_all_cores": round(t_all, 4), "oracle_cores": threads,
        "oracle_seconds_one_core": round(t_one, 4),
        "max_abs_err": float(err.max()), "mean_abs_err": float(err.mean()),
        "mask_mismatch_outside_near_ties": int(((got != ref["mask"]) & ~near).sum()),
        "near_ties": int(near.sum())}


def run_decode_sweep(args, bl, dev, stream, hbm_peak):
    """Decode length sweep: B 148, Hq 32 / Hkv 8, d 128, Bc 64, planted gap 8
    (sink + 3% heavy blocks); a of lambda = a / L calibrated once at 32K for
    70% sparsity and applied at every length.  Per length: achieved
    sparsity, time against the dense path, algorithmic GB/s, near-ties and
    error on 4 sampled sequences from the oracle."""
    import numpy as np
    import oracle
    from synth import config_seed, planted_gap_kv_inplace
    B, Hq, Hkv, d, Bc = 148, 32, 8, 128, 64
    K, W = min(args.steps, 20), args.warmup

    def make(L):
        q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=dev)
        k = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        planted_gap_kv_inplace(k, v, q, block=Bc, gap=8.0, heavy_frac=0.03,
                               seed=config_seed(3, L))
        return q, k, v

    q, k, v = make(32768)
    cal = bl.blasst_calibrate(0.70, mode="decode", q=q, k=k, v=v, Bc=Bc,
                              tol=0.002)
    a = cal["a"]
    del q, k, v
    torch.cuda.empty_cache()
    out = {"workload": f"decode B{B} Hq{Hq} Hkv{Hkv} d{d} Bc{Bc}, lambda = a/L "
                       f"with a fitted at 32K for 70%",
           "a": a, "l2": "inputs larger than L2, no flush"}
    seqs = (0, 37, 101, 147)
    for L in args.sweep_lengths:
        need = 2 * B * Hkv * L * d * 2
        if torch.cuda.mem_get_info(dev)[0] < need * 1.1 + (2 << 30):
            out[str(L)] = {"skipped": "not enough free device memory"}
            continue
        q, k, v = make(L)
        lnl = min(0.0, math.log(a / L))
        S = bl.blasst_decode_splits(B, Hkv, L, Bc)
        nk = -(-L // Bc)
        st = bl.Stats(device=dev, mask_numel=B * Hkv * nk)
        o, lse = bl.blasst_decode(q, k, v, ln_lambda=lnl, stats=st)
        torch.cuda.synchronize()
        vis, skp = st.read()
        mask = st.mask.view(B, Hkv, nk)
        by = decode_bytes(B, Hq, Hkv, L, d, Bc, S,
                          kept_rows_from_mask(mask, L, Bc))
        ms = time_calls(lambda: bl.blasst_decode(q, k, v, ln_lambda=lnl, o=o,
                                                 lse=lse), K, W, stream) / K
        od = torch.empty_like(o)
        ms_d = time_calls(lambda: bl.blasst_decode(q, k, v, o=od), K, W,
                          stream) / K
        ties, errs = 0, []
        for b in seqs:
            r = oracle.decode(q[b:b + 1], k[b:b + 1], v[b:b + 1],
                              1.0 / math.sqrt(d), lnl, Bc, S)
            ties += _near(r["margin"])
            errs.append(np.abs(o[b:b + 1].float().cpu().numpy() - r["o"]).max())
        gbs = by / (ms / 1e3) / 1e9
        out[str(L)] = {"ln_lambda": lnl, "splits": S, "sparsity": skp / vis,
                       "us": round(ms * 1e3, 1), "dense_us": round(ms_d * 1e3, 1),
                       "speedup_vs_dense": round(ms_d / ms, 4),
                       "GBps": round(gbs, 1), "hbm_frac": round(gbs / hbm_peak, 4),
                       "near_ties_4seq": ties,
                       "max_abs_err_4seq": float(max(errs))}
        del q, k, v, o, lse, od, st
        torch.cuda.empty_cache()
    return out


def run_prefill_sweep(args, bl, dev, stream, tf_peak):
    """Prefill sparsity and calibration sweep: B 1, Hq 32 / Hkv 8, d 128,
    causal, 128 x 128 tiles, gap per head uniform in [4, 12] nats, sink +
    2% heavy blocks + 512-token window boost, L in {4K, 16K, 64K}.  For each
    target sparsity a is fitted over the lengths whose calibration reaches
    it (log-space fit of lambda = a / L), then each length runs at
    lambda = a / L: achieved sparsity, deviation from the target, time
    against the dense path.  The 4K case is compared with the oracle."""
    import numpy as np
    import oracle
    from synth import config_seed, planted_gap
    lengths, targets = args.prefill_sweep_lengths, (0.0, 0.3, 0.5, 0.7, 0.9)
    flush = l2_flush_buffer(dev)
    # repetitions per length: short calls are timed more often
    reps_of = {L: max(3, min(20, (20 * 65536) // (L * 4))) for L in lengths}
    xs = {L: planted_gap(1, 32, 8, L, L, 128, block=128, gap_range=(4.0, 12.0),
                         heavy_frac=0.02, window=512, seed=config_seed(4, L),
                         device=dev) for L in lengths}
    dense_ms = {}
    for L, x in xs.items():
        o = torch.empty_like(x.q)
        reps = reps_of[L]
        dense_ms[L] = time_calls_flushed(lambda: bl.blasst_prefill(
            x.q, x.k, x.v, o=o, want_lse=False), reps, 2, stream, flush) / reps
    out = {"workload": "prefill B1 Hq32 Hkv8 d128 causal 128x128, gap per head "
                       "U[4,12] nats, lambda = a/L with a fitted per target "
                       "over the lengths (log space)",
           "l2": "L2 flushed (256 MB write) before every timed call",
           "dense_us": {str(L): round(t * 1e3, 1) for L, t in dense_ms.items()},
           "runs": []}
    devs = []
    for tgt in targets:
        cals = {L: bl.blasst_calibrate(tgt, mode="prefill", q=x.q, k=x.k,
                                       v=x.v, Br=128, Bc=128, tol=0.002,
                                       raise_on_no_converge=False)
                for L, x in xs.items()}
        fit_L = [L for L in lengths if cals[L]["status"] == 0]
        a = None if (tgt == 0.0 or not fit_L) else bl.blasst_fit_a(
            [cals[L]["lambda_"] for L in fit_L], fit_L)
        for L, x in xs.items():
            lnl = -math.inf if a is None else min(0.0, math.log(a / L))
            st = bl.Stats(device=dev)
            bl.blasst_prefill(x.q, x.k, x.v, ln_lambda=lnl, stats=st,
                              stats_only=True)
            torch.cuda.synchronize()
            sp = st.sparsity()
            o = torch.empty_like(x.q)
            reps = reps_of[L]
            ms = time_calls_flushed(lambda: bl.blasst_prefill(
                x.q, x.k, x.v, ln_lambda=lnl, o=o, want_lse=False),
                reps, 2, stream, flush) / reps
            rec = {"L": L, "target": tgt, "a": a, "ln_lambda": lnl,
                   "sparsity": round(sp, 5), "deviation": round(abs(sp - tgt), 5),
                   "calibration_reached_target_at_L": cals[L]["status"] == 0,
                   "us": round(ms * 1e3, 1),
                   "speedup_vs_dense": round(dense_ms[L] / ms, 4),
                   "dense_equiv_tflops": round(dense_equiv_flops(1, 32, L, 128)
                                               / (ms / 1e3) / 1e12, 1)}
            if tgt > 0 and L == 4096 and a is not None and not args.no_cpu:
                r = oracle.prefill(x.q, x.k, x.v, 1 / math.sqrt(128), True,
                                   lnl, 128, 128)
                og, _ = bl.blasst_prefill(x.q, x.k, x.v, ln_lambda=lnl)
                g = og.float().cpu().numpy()
                e = np.concatenate([np.abs(g[b, h, i * 128:(i + 1) * 128]
                                           - r["o"][u]).ravel()
                                    for u, (b, h, i) in enumerate(r["units"])])
                rec.update(max_abs_err=float(e.max()),
                           mean_abs_err=float(e.mean()),
                           near_ties=_near(r["margin"]))
            if tgt > 0 and cals[L]["status"] == 0:
                devs.append(abs(sp - tgt))
            out["runs"].append(rec)
    out["mean_deviation"] = float(np.mean(devs)) if devs else None
    out["max_deviation"] = float(np.max(devs)) if devs else None
    del flush, xs
    torch.cuda.empty_cache()
    return out


def run_mqa(args, bl, dev, stream, hbm_peak):
    """MQA decode, B 32 x 32 query heads on one KV head, 32K keys, d 128:
    blasst_decode (tiles of 8 heads on the tensor core), the same tiles on
    the CUDA cores (blasst_decode_batched with batch 1, one CTA per tile)
    and blasst_decode_wide (the 32 heads as one tile), dense and at
    ln lambda -2.  GB/s counts K and the V of kept blocks."""
    from synth import config_seed, planted_gap_kv_inplace
    B, Hq, Hkv, L, d = 32, 32, 1, 32768, 128
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=dev)
    k = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(10, 4))
    nk = L // 64
    K, W = args.steps, args.warmup
    out = {"workload": f"MQA decode B{B} Hq{Hq} Hkv{Hkv} Lkv{L} d{d} Bc 64"}
    cuda_cores = lambda *a, **kw: bl.blasst_decode_batched(*a, batch=1, **kw)
    for name, fn, rows in (("tiles_of_8", bl.blasst_decode, Hkv * Hq // 8),
                           ("tiles_of_8_cuda_cores", cuda_cores, Hkv * Hq // 8),
                           ("wide", bl.blasst_decode_wide, Hkv)):
        r = {}
        for key, lnl in (("dense", -math.inf), ("lnl_-2", -2.0)):
            st = bl.Stats(device=dev, mask_numel=B * rows * nk)
            o, lse = fn(q, k, v, ln_lambda=lnl, stats=st)
            torch.cuda.synchronize()
            vis, skp = st.read()
            ms = time_calls(lambda: fn(q, k, v, ln_lambda=lnl, o=o, lse=lse),
                            K, W, stream) / K
            byts = B * Hkv * L * d * 2 * (2.0 - skp / vis)
            r[key] = {"us": round(ms * 1e3, 1), "sparsity": skp / vis,
                      "GBps": round(byts / (ms / 1e3) / 1e9, 1),
                      "hbm_frac": round(byts / (ms / 1e3) / 1e9 / hbm_peak, 4)}
        out[name] = r
    return out


def run_mla(args, bl, dev, stream, hbm_peak, tf_peak):
    """MLA decode: B 32 tokens x 128 heads against a latent cache of
    --mla-len keys (32K by default; 576 wide, value = first 512 columns),
    planted-gap rows; dense and at the ln lambda (bisection over
    statistics-only passes) that skips ~50%.
    Algorithmic bytes = the cache (read once; the value is part of the row)
    + q + split partials written and read + o and lse."""
    from synth import config_seed, planted_gap_kv_inplace
    B, H, L, dqk, dv = 32, 128, args.mla_len, 576, 512
    q = torch.empty(B, H, dqk, dtype=torch.bfloat16, device=dev)
    c4 = torch.empty(B, 1, L, dqk, dtype=torch.bfloat16, device=dev)
    planted_gap_kv_inplace(c4, torch.empty_like(c4), q, block=64, gap=8.0,
                           heavy_frac=0.03, seed=config_seed(31))
    cache = c4[:, 0]
    nk = -(-L // 64)
    S = bl.blasst_mla_decode_splits(B, L)
    st = bl.Stats(device=dev, mask_numel=B * nk)

    def sparsity(lnl):
        st.reset()
        bl.blasst_mla_decode(q, cache, ln_lambda=lnl, stats=st, stats_only=True)
        torch.cuda.synchronize()
        v, s_ = st.read()
        return s_ / v
    lo, hi = -64.0, 0.0
    for _ in range(16):
        mid = 0.5 * (lo + hi)
        if sparsity(mid) < 0.5:
            lo = mid
        else:
            hi = mid
    lnl = hi
    o = torch.empty(B, H, dv, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, dtype=torch.float32, device=dev)
    ws = torch.empty(bl.blasst_mla_decode_workspace_size(B, H, S),
                     dtype=torch.uint8, device=dev)
    out = {"workload": f"MLA decode B{B} H{H} L{L} d_qk {dqk} d_v {dv} Bc 64",
           "splits": S}
    K, W = args.steps, args.warmup
    for key, l in (("dense", -math.inf), ("sparse", lnl)):
        sp = sparsity(l)
        fn = lambda: bl.blasst_mla_decode(q, cache, ln_lambda=l, o=o, lse=lse,
                                          workspace=ws)
        ms = time_calls(fn, K, W, stream) / K
        byts = (B * L * dqk * 2 + B * H * dqk * 2 + 2 * B * H * S * (dv + 1) * 4
                + B * H * (dv * 2 + 4))
        kept = (1.0 - sp) * B * nk
        # tensor work issued: each block scored once (its 576 columns split
        # over a CTA pair), P.V of kept blocks (512 value columns, split too)
        issued = (2.0 * 128 * 64 * dqk * B * nk + 2.0 * 128 * 64 * dv * kept)
        out[key] = {"ln_lambda": l, "sparsity": sp, "us": round(ms * 1e3, 1),
                    "GBps": round(byts / (ms / 1e3) / 1e9, 1),
                    "hbm_frac": round(byts / (ms / 1e3) / 1e9 / hbm_peak, 4),
                    "issued_tflops": round(issued / (ms / 1e3) / 1e12, 1),
                    "tensor_frac_issued": round(issued / (ms / 1e3) / 1e12 / tf_peak, 4)}
    out["sparse"]["speedup_vs_dense"] = round(out["dense"]["us"] / out["sparse"]["us"], 4)
    return out


def run_prefill_backward(args, bl, q, k, v, lnl, stream, tf_peak):
    """blasst_prefill_backward on the prefill workload: the dense backward
    (every visible pair) and the backward of the forward at the ln lambda
    calibrated for 70% (its decision bytes as the mask).  Executed FLOPs
    = 5 GEMMs of 128 x 128 x d per kept pair (S^T, dP^T, dV, dK, dQ)."""
    from synth import config_seed, output_gradient
    B, Hq, Lq, d = q.shape
    Br = 128
    nq, nk = -(-Lq // Br), -(-k.shape[2] // Br)
    dout = output_gradient((B, Hq, Lq, d), config_seed(2, 1), device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(bl.blasst_prefill_backward_workspace_size(B, Hq, Lq, d),
                     dtype=torch.uint8, device=q.device)
    K, W = max(3, args.prefill_steps // 2), args.warmup
    res = {"what": "dQ, dK, dV of the forward with its decisions fixed; "
                   "f32 dQ accumulated by TMA bulk reductions"}
    dense_ms = None
    for key, l in (("dense", -math.inf), ("s70", lnl)):
        st = bl.Stats(device=q.device, mask_numel=B * Hq * nq * nk)
        o, lse = bl.blasst_prefill(q, k, v, ln_lambda=l, stats=st)
        torch.cuda.synchronize()
        vis, skp = st.read()
        mask = None if key == "dense" else st.mask

        def fn():
            bl.blasst_prefill_backward(q, k, v, o, lse, dout, mask=mask, dq=dq,
                                       dk=dk, dv=dv, workspace=ws)
        ms = time_calls(fn, K, W, stream) / K
        ex = 10.0 * Br * Br * d * (vis - skp)
        r = {"us": round(ms * 1e3, 1), "sparsity": skp / vis,
             "executed_tflops": round(ex / (ms / 1e3) / 1e12, 1),
             "tensor_frac": round(ex / (ms / 1e3) / 1e12 / tf_peak, 4)}
        if key == "dense":
            dense_ms = ms
        else:
            r["speedup_vs_dense"] = round(dense_ms / ms, 4)
        res[key] = r
    return res


def run_prefill_window(args, bl, q, k, v, o, lse, lnl, stream, tf_peak):
    """Sliding-window prefill on the same inputs: window WIN keys, dense and
    at the ln lambda calibrated for 70% on the full causal problem."""
    B, Hq, L, d = q.shape
    Br = Bc = 128
    K, W = args.prefill_steps, args.warmup
    win = PRE["window"]
    # dense-equivalent FLOPs: 4 d per visible (query, key) pair
    pairs = sum(min(r + 1, win) for r in range(L))
    dense_eq = 4.0 * B * Hq * d * pairs
    res = {"window": win}
    for key, x in (("dense", -math.inf), ("lnl_s70", lnl)):
        st = bl.Stats(device=q.device)
        bl.blasst_prefill_window(q, k, v, window=win, ln_lambda=x, o=o,
                                 lse=lse, stats=st)
        torch.cuda.synchronize()
        vis, skp = st.read()
        fn = lambda: bl.blasst_prefill_window(q, k, v, window=win,
                                              ln_lambda=x, o=o, lse=lse)
        ms = time_calls(fn, K, W, stream) / K
        ex = prefill_flops(vis, vis - skp, Br, Bc, d)
        res[key] = {"ln_lambda": x, "sparsity": skp / vis,
                    "us": round(ms * 1e3, 1),
                    "dense_equiv_tflops": round(dense_eq / (ms / 1e3) / 1e12, 1),
                    "executed_tflops": round(ex / (ms / 1e3) / 1e12, 1),
                    "tensor_frac": round(ex / (ms / 1e3) / 1e12 / tf_peak, 4)}
    res["lnl_s70"]["speedup_vs_dense"] = round(
        res["dense"]["us"] / res["lnl_s70"]["us"], 4)
    return res


def run_decode_batched(args, bl, q, k, v, lnl, S, ws, ms_seq):
    """The batched decision rule (pairs of blocks scored before either is
    decided) on the decode workload at the same ln lambda."""
    B, Hq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    Bc = DEC["Bc"]
    nk = -(-Lkv // Bc)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    st = bl.Stats(device=q.device, mask_numel=B * Hkv * nk)
    bl.blasst_decode_batched(q, k, v, batch=2, ln_lambda=lnl, num_splits=S,
                             o=o, lse=lse, workspace=ws, stats=st)
    torch.cuda.synchronize()
    vis, skp = st.read()
    kept_rows = kept_rows_from_mask(st.mask.view(B, Hkv, nk), Lkv, Bc)
    by = decode_bytes(B, Hq, Hkv, Lkv, d, Bc, S, kept_rows)
    fn = lambda: bl.blasst_decode_batched(q, k, v, batch=2, ln_lambda=lnl,
                                          num_splits=S, o=o, lse=lse,
                                          workspace=ws)
    ms = time_calls(fn, args.steps, args.warmup, torch.cuda.current_stream()) / args.steps
    return {"batch": 2, "ln_lambda": lnl, "sparsity": skp / vis,
            "us": round(ms * 1e3, 2), "GBps": round(by / (ms / 1e3) / 1e9, 1),
            "bytes_per_call": by,
            "speedup_vs_sequential_rule": round(ms_seq / ms, 4)}


def run_decode_window(args, bl, q, k, v, lnl, stream):
    """Sliding-window decode on the decode workload's cache: the last WIN
    keys, at the calibrated ln lambda and dense."""
    B, Hq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    Bc = DEC["Bc"]
    win = DEC["window"]
    K, W = args.steps, args.warmup
    jlo = (Lkv - win) // Bc if 0 < win < Lkv else 0
    S = bl.blasst_decode_splits(B, Hkv, Lkv - jlo * Bc, Bc)
    nk = -(-Lkv // Bc)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    ws = torch.empty(bl.blasst_decode_workspace_size(B, Hq, d, S),
                     dtype=torch.uint8, device=q.device)
    res = {"window": win, "splits": S}
    for key, x in (("dense", -math.inf), ("lnl_s70", lnl)):
        st = bl.Stats(device=q.device, mask_numel=B * Hkv * nk)
        bl.blasst_decode_window(q, k, v, window=win, ln_lambda=x, o=o, lse=lse,
                                workspace=ws, stats=st)
        torch.cuda.synchronize()
        vis, skp = st.read()
        mask = st.mask.view(B, Hkv, nk)
        kept_rows = int((mask == 1).sum().item()) * Bc
        by = (2 * d * B * Hkv * (Lkv - jlo * Bc) + 2 * d * kept_rows
              + 2 * B * Hq * d + B * Hq * S * (d + 1) * 4 * 2
              + B * Hq * (2 * d + 4))
        fn = lambda: bl.blasst_decode_window(q, k, v, window=win, ln_lambda=x,
                                             o=o, lse=lse, workspace=ws)
        ms = time_calls(fn, K, W, stream) / K
        res[key] = {"ln_lambda": x, "sparsity": skp / vis,
                    "us": round(ms * 1e3, 2),
                    "GBps": round(by / (ms / 1e3) / 1e9, 1),
                    "bytes_per_call": by}
    res["lnl_s70"]["speedup_vs_dense"] = round(
        res["dense"]["us"] / res["lnl_s70"]["us"], 4)
    return res


# ---------------------------------------------------------------------------
# the reference arm: the CPU oracle, as it stands, on the host cores
# ---------------------------------------------------------------------------
def auto_splits(B, Hkv, Lkv, Bc, n_sm=148, ctas_per_sm=3):
    """The library's automatic split count (blasst_decode_splits), restated
    so that the reference arm loads no GPU code: >= 2 waves, >= 8 blocks per
    split, best-filled last wave among up to twice the minimum."""
    nk = -(-Lkv // Bc)
    units = B * Hkv
    slots = n_sm * ctas_per_sm
    s_max = max(1, nk // 8)
    s_min = max(1, -(-2 * slots // units))
    if s_min > s_max:
        return s_max
    best, best_eff = s_min, -1.0
    for s in range(s_min, min(2 * s_min, s_max) + 1):
        waves = units * s / slots
        eff = waves / math.ceil(waves)
        if eff > best_eff + 1e-9:
            best, best_eff = s, eff
    return best


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import oracle
    from synth import config_seed, planted_gap

    B, Hq, Hkv, Lkv, d, Bc = (DEC[x] for x in ("B", "Hq", "Hkv", "Lkv", "d", "Bc"))
    n_seq = 4  # bounded sample: four sequences of the batch per step
    x = planted_gap(n_seq, Hq, Hkv, 1, Lkv, d, decode=True, block=Bc, gap=8.0,
                    heavy_frac=0.03, seed=config_seed(1), device="cpu")
    S = auto_splits(B, Hkv, Lkv, Bc)
    scale = 1.0 / math.sqrt(d)
    threads = os.cpu_count() or 1
    # lambda for 70% sparsity from the oracle's own margins (exact quantile)
    r0 = oracle.decode(x.q, x.k, x.v, scale, 0.0, Bc, S, n_threads=threads)
    D = np.sort((r0["margin"]).ravel())  # margin at ln lambda = 0 is D itself
    idx = int(math.ceil(DEC["target"] * D.size)) - 1
    lnl = float(np.nextafter(D[idx], np.inf)) if D[idx] < 0 else 0.0
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        res = oracle.decode(x.q, x.k, x.v, scale, lnl, Bc, S, n_threads=threads)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    kept_rows = kept_rows_from_mask(torch.from_numpy(res["mask"]), Lkv, Bc)
    by = decode_bytes(n_seq, Hq, Hkv, Lkv, d, Bc, S, kept_rows)
    t = sum(times) / len(times)
    val = by / t / 1e9
    sample = (f"{n_seq} of {B} sequences per step (all {Hkv} KV heads x {Lkv} "
              f"keys), {S} splits, lambda from the oracle's margins")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 4),
        "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic planted-gap (seeded)",
        "config": {"workload": (f"decode B{B} Hq{Hq} Hkv{Hkv} Lkv{Lkv} d{d} "
                                f"Bc{Bc}, lambda for {DEC['target']:.0%} sparsity"),
                   "global_batch": B, "seq_len": Lkv, "parallelism": "cpu",
                   "sparsity": res["skipped"] / res["visited"]},
        "cpu_baseline": {"value": round(val, 4), "unit": "GB/s",
                         "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(val, 4), "unit": "GB/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--prefill-steps", type=int, default=10)
    ap.add_argument("--impl", choices=["blasst", "reference"], default="blasst")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode workload (profiling runs only)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-window", action="store_true",
                    help="skip the sliding-window measurements")
    ap.add_argument("--no-mla", action="store_true",
                    help="skip the MLA decode measurements")
    ap.add_argument("--mla-len", type=int, default=32768,
                    help="latent rows per sequence in the MLA decode leg")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the prefill backward measurements")
    ap.add_argument("--no-paged", action="store_true",
                    help="skip the paged-cache decode measurements")
    ap.add_argument("--decode-batch", type=int, default=DEC["B"],
                    help="sequences per GPU (profiling runs use fewer)")
    ap.add_argument("--decode-lnl", type=float, default=None,
                    help="fixed ln(lambda) instead of calibrating")
    ap.add_argument("--prefill-L", type=int, default=PRE["L"])
    ap.add_argument("--prefill-lnl", type=float, default=None,
                    help="measure prefill only at this ln(lambda)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the end-to-end step as separate launches")
    ap.add_argument("--no-s50", action="store_true",
                    help="skip the decode leg at 50%% sparsity (profiling runs)")
    ap.add_argument("--no-sweeps", action="store_true",
                    help="skip the decode length and prefill calibration sweeps")
    ap.add_argument("--sweep-lengths", type=int, nargs="+",
                    default=[8192, 32768, 65536, 131072],
                    help="cache lengths of the B148 decode sweep")
    ap.add_argument("--prefill-sweep-lengths", type=int, nargs="+",
                    default=[4096, 16384, 65536])
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="approximate CPU time budget of the oracle baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_blasst(args)


if __name__ == "__main__":
    main()
