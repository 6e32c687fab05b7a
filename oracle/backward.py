"""Backward of the BLASST prefill forward with its skip decisions held fixed
-- TEST INFRASTRUCTURE ONLY (the same import rule as the rest of
``oracle``: tests, ``__graft_entry__.smoke()`` and bench.py's CPU legs).

Reading: the pages propose fine-tuning with BLASST active (the summary of
"BLASST: Dynamic BLocked Attention Sparsity via Softmax Thresholding" on
gist.science, section 2, "Treinamento Consciente de Esparsidade"; the Hindi
summary, algorithm design, sparsity-aware training), so the backward
differentiates the forward as it ran, its decisions included.  Once the
decisions of a forward are fixed, that forward is attention restricted, per
query tile, to its kept blocks: for a query r of tile i,

    O_r = sum_c P_rc v_c,   P_rc = exp(s_rc - lse_r)  for the visible keys c
                            of the blocks j with mask[i, j] = KEPT, else 0,
    s_rc = scale * q_r . k_c,   lse_r = ln sum_{kept, visible c} exp(s_rc),

because the running-max reference and the lazy rescale of the forward
cancel in O and lse.  A decision is a step function of the inputs (its
derivative is zero wherever it is defined), so the gradient of the forward
is the gradient of this restricted softmax attention.  Written out:

    D_r   = sum_e dO_re O_re
    dV_c  = sum_r P_rc dO_r
    dP_rc = dO_r . v_c
    dS_rc = P_rc (dP_rc - D_r)
    dQ_r  = scale * sum_c dS_rc k_c
    dK_c  = scale * sum_r dS_rc q_r

and for grouped heads a KV head's dK and dV sum over its G query heads.
Each step is one numpy float64 operation on whole (L x L) matrices of one
head, in that order; nothing is blocked or fused.

Parity pins: ``tests/test_oracle_backward_pins.py`` (central finite
differences of an independent numpy forward, with and without a mask, and
the restricted forward against ``oracle.prefill``).
"""
import numpy as np

KEPT = 1


def _f64(x):
    """torch tensor (any float dtype, bf16 exactly) or array -> float64."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if x.dtype.is_floating_point:
            x = x.double()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _u8(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.asarray(x, dtype=np.uint8)


def keep_matrix(mask_bh, Lq, Lkv, Br, Bc, causal):
    """Boolean [Lq, Lkv]: key c takes part in query r's softmax (visible
    under the bottom-right causal mask and in a block the forward kept for
    r's tile)."""
    r = np.arange(Lq)[:, None]
    c = np.arange(Lkv)[None, :]
    keep = mask_bh[r // Br, c // Bc] == KEPT
    if causal:
        keep &= c <= r + (Lkv - Lq)
    return keep


def restricted_forward(q, k, v, mask, scale, causal, Br, Bc):
    """O [B,Hq,Lq,d] and lse [B,Hq,Lq] of attention restricted to the kept
    blocks (float64), the function whose gradient prefill_backward takes."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    mask = _u8(mask)
    B, Hq, Lq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, Hq, Lq, d))
    lse = np.full((B, Hq, Lq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            keep = keep_matrix(mask[b, h], Lq, Lkv, Br, Bc, causal)
            s = scale * (q[b, h] @ k[b, h // G].T)
            s = np.where(keep, s, -np.inf)
            mx = s.max(axis=1, keepdims=True)
            live = np.isfinite(mx[:, 0])
            mx = np.where(np.isfinite(mx), mx, 0.0)
            p = np.exp(s - mx)
            den = p.sum(axis=1, keepdims=True)
            den_safe = np.where(den > 0, den, 1.0)
            o[b, h] = (p @ v[b, h // G]) / den_safe
            lse[b, h] = np.where(live, mx[:, 0] + np.log(den_safe[:, 0]),
                                 -np.inf)
    return o, lse


def prefill_backward(q, k, v, o, lse, do, mask, scale, causal, Br, Bc):
    """dQ [B,Hq,Lq,d], dK and dV [B,Hkv,Lkv,d] (float64) of the forward
    whose output ``o``, log-sum-exp ``lse`` and decisions ``mask``
    ([B,Hq,ceil(Lq/Br),ceil(Lkv/Bc)], 1 = kept) are given, for the output
    gradient ``do``."""
    q, k, v, o, lse, do = (_f64(t) for t in (q, k, v, o, lse, do))
    mask = _u8(mask)
    B, Hq, Lq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kh, vh = k[b, h // G], v[b, h // G]
            keep = keep_matrix(mask[b, h], Lq, Lkv, Br, Bc, causal)
            s = scale * (q[b, h] @ kh.T)
            lse_r = np.where(np.isfinite(lse[b, h]), lse[b, h], 0.0)
            p = np.where(keep, np.exp(np.where(keep, s, 0.0) - lse_r[:, None]),
                         0.0)
            D = (do[b, h] * o[b, h]).sum(axis=1)
            dv[b, h // G] += p.T @ do[b, h]
            dp = do[b, h] @ vh.T
            ds = p * (dp - D[:, None])
            dq[b, h] = scale * (ds @ kh)
            dk[b, h // G] += scale * (ds.T @ q[b, h])
    return dq, dk, dv
