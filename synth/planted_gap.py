"""Seeded planted-gap attention inputs (input synthesis only).

This module is shared by the tests, the benchmark and the smoke check.  It
holds no arithmetic of the attention method itself: it only draws Q, K, V
with a planted score structure, in the shapes of the BLASST kernel
benchmarks (batch 148 / 32K tokens / head dim 128 with GQA, from the
MLSys'26 reading notes, claims table, section 5.3), standing in for the
model activations and datasets (RULER, LongBench) the pages measure on.

Recipe, per sequence b and KV head h (query heads of the group share it):
  * u            : a random unit vector in R^d (the head's "sink" direction);
  * beta         : sqrt(gap * sqrt(d)), so that beta^2 / sqrt(d) = gap nats of
                   scaled score separate planted keys from the rest;
  * Q            : N(0,1) + beta * u             (every query token);
  * K            : N(0,1), plus beta * u on the first Bc-token block (sink)
                   and on a Bernoulli(heavy_frac) subset of the other blocks;
  * V            : N(0,1);
  * window boost : optionally, aligned windows of `window` tokens each get a
                   unit vector u_w orthonormal to u and to the other windows'
                   vectors (reused cyclically when d - 1 vectors run out);
                   beta * u_w is added to Q and K of every token of window w,
                   so each query gains `gap` nats on the keys of its own
                   window that precede it (at most `window` of them).
Everything is drawn in float32 and rounded to bfloat16 (round to nearest
even).  The random stream is torch's counter-based Philox (CUDA) or
Mersenne twister (CPU) seeded with `seed`; the bytes therefore depend on the
device, which is why every comparison feeds the oracle the very bytes the
GPU read.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

CONFIG_SEED_BASE = 0xB1A5500


def beta_for_gap(gap: float, d: int) -> float:
    return math.sqrt(gap * math.sqrt(d))


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    return g


def _directions(n_heads: int, n_vec: int, d: int, g_cpu) -> torch.Tensor:
    """[n_heads, n_vec, d] orthonormal rows (float64), drawn on the CPU."""
    z = torch.randn(n_heads, d, n_vec, generator=g_cpu, dtype=torch.float64)
    qm, r = torch.linalg.qr(z)  # columns orthonormal
    # make the factorisation unique (sign of diag(r) positive)
    sgn = torch.sign(torch.diagonal(r, dim1=-2, dim2=-1))
    sgn[sgn == 0] = 1.0
    qm = qm * sgn[:, None, :]
    return qm.transpose(1, 2).contiguous()


@dataclass
class PlantedInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    heavy: torch.Tensor  # bool [B, Hkv, nblocks]: planted (sink + heavy) blocks
    gap: torch.Tensor    # float [B, Hkv] nats per head


def planted_gap(B, Hq, Hkv, Lq, Lkv, d, *, block=64, gap=8.0, gap_range=None,
                heavy_frac=0.03, window=None, decode=False, seed=0,
                device="cpu") -> PlantedInputs:
    """Draw planted-gap inputs.

    decode=True returns q of shape [B, Hq, d] (one token per sequence, the
    last position); otherwise q is [B, Hq, Lq, d].  k, v are [B, Hkv, Lkv, d].
    gap_range=(lo, hi) draws the gap per (sequence, KV head) uniformly.
    """
    device = torch.device(device)
    assert Hq % Hkv == 0
    G = Hq // Hkv
    g_cpu = _gen("cpu", seed)
    g_dev = _gen(device, seed + 1)
    nblk = -(-Lkv // block)

    if gap_range is not None:
        lo, hi = gap_range
        gaps = lo + (hi - lo) * torch.rand(B, Hkv, generator=g_cpu,
                                           dtype=torch.float64)
    else:
        gaps = torch.full((B, Hkv), float(gap), dtype=torch.float64)
    betas = torch.sqrt(gaps * math.sqrt(d))

    n_win = 0
    if window:
        n_win = -(-max(Lq, Lkv) // window)
    n_vec = 1 + min(max(n_win, 0), d - 1)
    dirs = _directions(B * Hkv, n_vec, d, g_cpu).view(B, Hkv, n_vec, d)
    u = dirs[:, :, 0]  # [B, Hkv, d]

    heavy = torch.rand(B, Hkv, nblk, generator=g_cpu) < heavy_frac
    heavy[:, :, 0] = True  # the sink block

    bu = (betas[:, :, None] * u).to(torch.float32)  # [B, Hkv, d]

    k = torch.randn(B, Hkv, Lkv, d, generator=g_dev, device=device,
                    dtype=torch.float32)
    # planted blocks: + beta*u on every key of the block
    blk = torch.arange(Lkv, device=device) // block
    sel = heavy.to(device)[:, :, blk].to(torch.float32)  # [B, Hkv, Lkv]
    k += sel[..., None] * bu.to(device)[:, :, None, :]
    del sel

    if decode:
        q = torch.randn(B, Hq, d, generator=g_dev, device=device,
                        dtype=torch.float32)
        q += bu.to(device).repeat_interleave(G, dim=1)
    else:
        q = torch.randn(B, Hq, Lq, d, generator=g_dev, device=device,
                        dtype=torch.float32)
        q += bu.to(device).repeat_interleave(G, dim=1)[:, :, None, :]

    if window and not decode:
        uw = (betas[:, :, None, None] * dirs[:, :, 1:]).to(torch.float32)
        uw = uw.to(device)  # [B, Hkv, n_vec-1, d]
        nv = uw.shape[2]
        # query t of Lq sits at key position t + (Lkv - Lq)
        off = Lkv - Lq
        for w in range(n_win):
            vec = uw[:, :, w % nv]  # [B, Hkv, d]
            k0, k1 = w * window, min((w + 1) * window, Lkv)
            if k0 < k1:
                k[:, :, k0:k1] += vec[:, :, None, :]
            q0, q1 = max(k0 - off, 0), min(k1 - off, Lq)
            if q0 < q1:
                q[:, :, q0:q1] += vec.repeat_interleave(G, dim=1)[:, :, None, :]

    v = torch.randn(B, Hkv, Lkv, d, generator=g_dev, device=device,
                    dtype=torch.float32)
    return PlantedInputs(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16),
                         v=v.to(torch.bfloat16), heavy=heavy,
                         gap=gaps.to(torch.float32))


def planted_gap_kv_inplace(k, v, q, *, block=64, gap=8.0, heavy_frac=0.03,
                           seed=0, chunk_tokens=4096):
    """Fill preallocated bf16 decode buffers q [B,Hq,d], k/v [B,Hkv,Lkv,d]
    with the decode recipe above, in token chunks, so that caches of tens of
    GB can be drawn without a float32 copy of the whole tensor."""
    B, Hkv, Lkv, d = k.shape
    Hq = q.shape[1]
    G = Hq // Hkv
    device = k.device
    g_cpu = _gen("cpu", seed)
    g_dev = _gen(device, seed + 1)
    nblk = -(-Lkv // block)
    betas = torch.sqrt(torch.full((B, Hkv), float(gap), dtype=torch.float64)
                       * math.sqrt(d))
    u = _directions(B * Hkv, 1, d, g_cpu).view(B, Hkv, d)
    heavy = torch.rand(B, Hkv, nblk, generator=g_cpu) < heavy_frac
    heavy[:, :, 0] = True
    bu = (betas[:, :, None] * u).to(torch.float32).to(device)
    hv = heavy.to(device)
    for t0 in range(0, Lkv, chunk_tokens):
        t1 = min(t0 + chunk_tokens, Lkv)
        kc = torch.randn(B, Hkv, t1 - t0, d, generator=g_dev, device=device,
                         dtype=torch.float32)
        blk = torch.arange(t0, t1, device=device) // block
        sel = hv[:, :, blk].to(torch.float32)  # [B, Hkv, T]
        kc += sel[..., None] * bu[:, :, None, :]
        k[:, :, t0:t1] = kc.to(torch.bfloat16)
        del kc
        vc = torch.randn(B, Hkv, t1 - t0, d, generator=g_dev, device=device,
                         dtype=torch.float32)
        v[:, :, t0:t1] = vc.to(torch.bfloat16)
        del vc
    qf = torch.randn(B, Hq, d, generator=g_dev, device=device,
                     dtype=torch.float32)
    qf += bu.repeat_interleave(G, dim=1)
    q.copy_(qf.to(torch.bfloat16))
    return heavy


def config_seed(index: int, extra: int = 0) -> int:
    return CONFIG_SEED_BASE + index + extra


def output_gradient(shape, seed, device="cpu") -> torch.Tensor:
    """A seeded standard-normal bf16 tensor: the loss gradient dO fed to the
    backward (drawn on the CPU so that every device gets the same values)."""
    g = _gen("cpu", seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16).to(device)
