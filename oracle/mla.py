"""BLASST decode over a multi-head latent (MLA) cache -- TEST INFRASTRUCTURE
ONLY (the same import rule as the rest of ``oracle``).

MLA decode (the attention form the method is stated to support: MLSys'26
reading notes, claims on MLA / GQA / sliding-window forms; gist.science
summary, section 3): every query head of a token attends to one shared
latent cache row per key, c_t = [latent (d_v) | rope key], d_qk = len(c_t);
the score is scale * q_h . c_t and the value is the latent part c_t[:d_v].
Reading: the decode tile of the method is the group of query heads that
share the KV head (here all H heads of the token), blocks of Bc keys, the
same criterion and online-softmax update as the decode (per split: running
max from -inf, blocks ascending; a block is skipped for the tile iff every
head's block max m~ satisfies m~ - m < ln lambda), split-KV with the
log-sum-exp merge.

Written out with numpy float64 per (sequence, split): one whole-block score
matrix at a time, in the order of the blockwise algorithm; nothing fused.
Pinned in ``tests/test_oracle_mla_pins.py`` against the C decode oracle
(d_v = d_qk, where MLA decode is plain decode with one KV head) and against
numpy softmax attention (dense limit).
"""
import math

import numpy as np

from .backward import _f64

NOT_VISITED, KEPT, SKIPPED = 0, 1, 2


def split_range(nk, S, s):
    """Blocks [j0, j1) of split s of nk blocks cut into S splits."""
    return (s * nk) // S, ((s + 1) * nk) // S


def mla_decode(q, cache, d_v, scale, ln_lambda, Bc, num_splits):
    """q [B,H,d_qk], cache [B,L,d_qk] (bf16 tensors or float arrays).

    Returns o [B,H,d_v], lse [B,H], o_part [B,H,S,d_v], lse_part [B,H,S],
    mask [B,nk] (0 not visited, 1 kept, 2 skipped), margin [B,nk]
    (max_h (m~_h - m_h) - ln lambda), visited, skipped.
    """
    q, c = _f64(q), _f64(cache)
    B, H, dqk = q.shape
    L = c.shape[1]
    nk = -(-L // Bc)
    S = int(num_splits)
    op = np.zeros((B, H, S, d_v))
    lp = np.full((B, H, S), -np.inf)
    mask = np.zeros((B, nk), np.uint8)
    margin = np.zeros((B, nk))
    vis = skp = 0
    for b in range(B):
        for s in range(S):
            j0, j1 = split_range(nk, S, s)
            m = np.full(H, -np.inf)
            l = np.zeros(H)
            acc = np.zeros((H, d_v))
            for j in range(j0, j1):
                kb = c[b, j * Bc:min((j + 1) * Bc, L)]
                sc = scale * (q[b] @ kb.T)          # [H, keys]
                mt = sc.max(axis=1)
                vis += 1
                diff = mt - m                      # +inf where m = -inf
                margin[b, j] = diff.max() - ln_lambda
                skip = ln_lambda > -math.inf and bool(np.all(diff < ln_lambda))
                if skip:
                    skp += 1
                    mask[b, j] = SKIPPED
                    continue
                mask[b, j] = KEPT
                m_new = np.maximum(m, mt)
                alpha = np.where(np.isfinite(m), np.exp(m - m_new), 0.0)
                p = np.exp(sc - m_new[:, None])
                l = alpha * l + p.sum(axis=1)
                acc = alpha[:, None] * acc + p @ kb[:, :d_v]
                m = m_new
            live = l > 0
            op[b, :, s] = np.where(live[:, None], acc / np.where(live, l, 1.0)[:, None], 0.0)
            lp[b, :, s] = np.where(live, m + np.log(np.where(live, l, 1.0)), -np.inf)
    lse = np.full((B, H), -np.inf)
    o = np.zeros((B, H, d_v))
    for b in range(B):
        for h in range(H):
            ls = lp[b, h]
            fin = np.isfinite(ls)
            if not fin.any():
                continue
            mx = ls[fin].max()
            w = np.where(fin, np.exp(ls - mx), 0.0)
            lse[b, h] = mx + math.log(w.sum())
            o[b, h] = (w[:, None] * op[b, h]).sum(axis=0) / w.sum()
    return dict(o=o, lse=lse, o_part=op, lse_part=lp, mask=mask,
                margin=margin, visited=vis, skipped=skp)
