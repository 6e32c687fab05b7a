"""Comparison helpers shared by the GPU parity tests.

Acceptance (stated for bf16 inputs with fp32 accumulation): max |o - o_ref|
<= 2e-2 and mean |o - o_ref| <= 2e-3 over the compared outputs; skip masks
bit-exact except where the oracle's margin |max_r(m~ - m) - ln lambda| is
below 1e-3 (near-ties, counted and reported).
"""
import numpy as np
import torch

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 2e-3
NEAR_TIE = 1e-3


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_out(o_gpu, o_ref, what=""):
    """o_gpu, o_ref: arrays of the same shape (float64)."""
    diff = np.abs(o_gpu - o_ref)
    mx, mean = float(diff.max()) if diff.size else 0.0, float(diff.mean()) if diff.size else 0.0
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    assert mx <= MAX_ABS, f"{what}: max abs err {mx:.3e} > {MAX_ABS}"
    assert mean <= MEAN_ABS, f"{what}: mean abs err {mean:.3e} > {MEAN_ABS}"
    return mx, mean


def check_lse(l_gpu, l_ref, what=""):
    diff = np.abs(l_gpu - l_ref)
    mx = float(diff.max()) if diff.size else 0.0
    assert mx <= LSE_ABS, f"{what}: lse max abs err {mx:.3e}"
    return mx


def check_mask(m_gpu, m_ref, margin, what=""):
    """Masks in {0 not visited, 1 kept, 2 skipped}.  Returns the near-tie
    count; raises on any mismatch outside a near-tie."""
    m_gpu = np.asarray(m_gpu)
    m_ref = np.asarray(m_ref)
    near = np.abs(np.nan_to_num(margin, nan=1.0, posinf=1.0, neginf=1.0)) < NEAR_TIE
    bad = (m_gpu != m_ref) & ~near
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} mask mismatches outside near-ties "
        f"(first at {np.argwhere(bad)[:5].tolist()})")
    return int(near.sum())


def sparsity(mask):
    mask = np.asarray(mask)
    v = int((mask > 0).sum())
    return (int((mask == 2).sum()) / v) if v else 0.0
