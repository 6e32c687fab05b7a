"""Independent float64 restatements used to pin the oracle (tests only).

Nothing here shares code with the oracle's C loops: the dense reference is a
whole-matrix numpy softmax, and the skip mask is the closed form that follows
from the method's criterion (a skipped block never raises the running max, so
the running max before block j equals the prefix max of the block maxima).
"""
import numpy as np


def bf16_to_f64(x):
    """bf16 torch tensor -> float64 numpy array (exact)."""
    import torch
    return x.detach().cpu().to(torch.float64).numpy()


def causal_visible(Lq, Lkv):
    """[Lq, Lkv] bool: key c visible to query r iff c <= r + (Lkv - Lq)."""
    r = np.arange(Lq)[:, None]
    c = np.arange(Lkv)[None, :]
    return c <= r + (Lkv - Lq)


def dense_prefill(q, k, v, scale, causal):
    """softmax(scale * Q K^T + mask) V and its log-sum-exp, float64.

    q [B,Hq,Lq,d], k/v [B,Hkv,Lkv,d] float64 arrays."""
    B, Hq, Lq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, Hq, Lq, d))
    lse = np.zeros((B, Hq, Lq))
    vis = causal_visible(Lq, Lkv) if causal else np.ones((Lq, Lkv), bool)
    for b in range(B):
        for h in range(Hq):
            s = scale * (q[b, h] @ k[b, h // G].T)
            s = np.where(vis, s, -np.inf)
            mx = s.max(axis=1, keepdims=True)
            p = np.exp(s - mx)
            den = p.sum(axis=1, keepdims=True)
            o[b, h] = (p @ v[b, h // G]) / den
            lse[b, h] = (mx + np.log(den))[:, 0]
    return o, lse


def dense_decode(q, k, v, scale):
    """q [B,Hq,d], k/v [B,Hkv,Lkv,d] float64 -> o [B,Hq,d], lse [B,Hq]."""
    B, Hq, d = q.shape
    G = Hq // k.shape[1]
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            s = scale * (k[b, h // G] @ q[b, h])
            mx = s.max()
            p = np.exp(s - mx)
            o[b, h] = (p @ v[b, h // G]) / p.sum()
            lse[b, h] = mx + np.log(p.sum())
    return o, lse


def block_row_max(s, Bc):
    """s [R, L] (with -inf for masked) -> [R, nk] per-block row maxima."""
    R, L = s.shape
    nk = -(-L // Bc)
    pad = np.full((R, nk * Bc), -np.inf)
    pad[:, :L] = s
    return pad.reshape(R, nk, Bc).max(axis=2)


def closed_form_decisions(mt, ln_lambda):
    """Tile decisions from the block maxima alone.

    mt [R, nk]: block-local row maxima of one tile (-inf = fully masked).
    Returns (decision [nk] in {0 not visited, 1 kept, 2 skipped},
             D [nk] = max_r (mt - prefix max before the block)).
    """
    R, nk = mt.shape
    prev = np.full((R, nk), -np.inf)
    if nk > 1:
        prev[:, 1:] = np.maximum.accumulate(mt, axis=1)[:, :-1]
    with np.errstate(invalid="ignore"):
        diff = mt - prev                     # +inf where prev = -inf
    diff = np.where(np.isneginf(mt), -np.inf, diff)
    D = diff.max(axis=0)
    visited = ~np.all(np.isneginf(mt), axis=0)
    dec = np.where(~visited, 0, np.where(D < ln_lambda, 2, 1)).astype(np.uint8)
    return dec, D


def prefill_scores(q, k, scale, causal, b, hq, G):
    s = scale * (q[b, hq] @ k[b, hq // G].T)
    if causal:
        s = np.where(causal_visible(q.shape[2], k.shape[2]), s, -np.inf)
    return s


def window_visible(Lq, Lkv, W):
    """[Lq, Lkv] bool: causal sliding window of W keys ending at the
    (bottom-right aligned) diagonal: diag - W < c <= diag."""
    r = np.arange(Lq)[:, None]
    c = np.arange(Lkv)[None, :]
    diag = r + (Lkv - Lq)
    return (c <= diag) & (c > diag - W)


def dense_masked(qh, kh, vh, scale, vis):
    """One head: softmax(scale q k^T where vis, else -inf) v, float64."""
    s = np.where(vis, scale * (qh @ kh.T), -np.inf)
    mx = s.max(axis=1, keepdims=True)
    p = np.exp(s - mx)
    den = p.sum(axis=1, keepdims=True)
    return (p @ vh) / den, (mx + np.log(den))[:, 0]
