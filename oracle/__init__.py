"""CPU oracle for the BLASST attention forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``dynamic_block_sparse_fa_b200``) neither imports nor links it.

The arithmetic lives in ``blasst_oracle.c`` (plain float64 loops, one query
tile at a time, blocks in ascending order); this module only marshals numpy
arrays into that library.  Every function takes bfloat16 tensors as raw
``uint16`` bit patterns, so the oracle reads exactly the bytes the GPU reads.

Parity pins (see ``tests/test_oracle_pins.py``): dense limit against a
float64 brute-force softmax, an independent closed-form skip mask, the
skipped-mass bound, mask monotonicity in lambda and the split/merge identity.
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None

NOT_VISITED, KEPT, SKIPPED = 0, 1, 2

_dp = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.oracle_prefill.restype = ctypes.c_int
        lib.oracle_prefill.argtypes = [
            _u16p, _u16p, _u16p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
            ctypes.c_double, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, _i32p, _dp, _dp, _u8p, _dp, _i64p, ctypes.c_int]
        lib.oracle_prefill_window.restype = ctypes.c_int
        lib.oracle_prefill_window.argtypes = [
            _u16p, _u16p, _u16p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, _i32p, _dp, _dp, _u8p, _dp, _i64p, ctypes.c_int]
        lib.oracle_decode_window.restype = ctypes.c_int
        lib.oracle_decode_window.argtypes = [
            _u16p, _u16p, _u16p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_double,
            ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp, _u8p, _dp, _i64p,
            ctypes.c_int]
        lib.oracle_decode_batched.restype = ctypes.c_int
        lib.oracle_decode_batched.argtypes = [
            _u16p, _u16p, _u16p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp, _u8p, _dp, _i64p,
            ctypes.c_int]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [
            _u16p, _u16p, _u16p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_int,
            ctypes.c_int, _dp, _dp, _dp, _dp, _u8p, _dp, _i64p, ctypes.c_int]
        lib.oracle_decode_paged.restype = ctypes.c_int
        lib.oracle_decode_paged.argtypes = [
            _u16p, _u16p, _u16p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            _i32p, ctypes.c_int, _i32p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int,
            _dp, _dp, _dp, _dp, _u8p, _dp, _i64p, ctypes.c_int]
        lib.oracle_combine.restype = None
        lib.oracle_combine.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, _dp, _dp]
        lib.oracle_split_begin.restype = ctypes.c_int
        lib.oracle_split_begin.argtypes = [ctypes.c_int] * 3
        _lib = lib
    return _lib


def _ptr(a, t):
    return a.ctypes.data_as(t)


def _bits(x):
    """bf16 tensor/array -> contiguous uint16 numpy array of its bit patterns."""
    if hasattr(x, "detach"):  # torch tensor
        import torch
        assert x.dtype == torch.bfloat16, x.dtype
        x = x.detach().cpu().contiguous().view(torch.int16).numpy()
    x = np.ascontiguousarray(x)
    assert x.dtype in (np.uint16, np.int16), x.dtype
    return x.view(np.uint16)


def n_threads_default():
    return os.cpu_count() or 1


def prefill(q, k, v, scale, causal, ln_lambda, Br, Bc, units=None,
            n_threads=0, window=0):
    """BLASST prefill forward for query tiles ``units`` (list of (b, hq, i)).

    ``window`` > 0 (causal only): query r sees the ``window`` keys ending at
    its diagonal (sliding-window attention); 0 = no window.

    q [B,Hq,Lq,d], k/v [B,Hkv,Lkv,d] bf16.  Returns a dict with
    ``o`` [n_units,Br,d] f64, ``lse`` [n_units,Br], ``mask`` [n_units,nk] u8,
    ``margin`` [n_units,nk], ``visited``, ``skipped``, ``units`` and
    ``threads``.  ``units=None`` means every tile of every head.
    """
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, Lq, d = qb.shape
    _, Hkv, Lkv, _ = kb.shape
    nq = -(-Lq // Br)
    nk = -(-Lkv // Bc)
    if units is None:
        units = [(b, h, i) for b in range(B) for h in range(Hq)
                 for i in range(nq)]
    ua = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 3))
    n = ua.shape[0]
    o = np.zeros((n, Br, d), np.float64)
    lse = np.zeros((n, Br), np.float64)
    mask = np.zeros((n, nk), np.uint8)
    margin = np.zeros((n, nk), np.float64)
    counts = np.zeros(2, np.int64)
    rc = lib.oracle_prefill_window(
        _ptr(qb, _u16p), _ptr(kb, _u16p), _ptr(vb, _u16p),
        B, Hq, Hkv, Lq, Lkv, d, float(scale), int(bool(causal)), int(window),
        float(ln_lambda), Br, Bc, n, _ptr(ua, _i32p),
        _ptr(o, _dp), _ptr(lse, _dp), _ptr(mask, _u8p), _ptr(margin, _dp),
        _ptr(counts, _i64p), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_prefill rejected its arguments")
    threads = n_threads if n_threads > 0 else n_threads_default()
    return dict(o=o, lse=lse, mask=mask, margin=margin,
                visited=int(counts[0]), skipped=int(counts[1]),
                units=ua, threads=threads)


def _tile_heads(Hq, Hkv, tile_heads, *pools):
    """Decode tiles of ``tile_heads`` query heads.  The tile of the method is
    the group of query heads that share a KV head (their rows are voted on
    together); with ``tile_heads`` < G = Hq/Hkv the group is cut into G /
    tile_heads consecutive tiles, which is the same as giving each tile its
    own copy of the KV head.  Returns the number of (virtual) KV heads and
    the pools with each KV head repeated G / tile_heads times (axis 1)."""
    G = Hq // Hkv
    T = G if tile_heads is None else int(tile_heads)
    if T < 1 or G % T != 0:
        raise ValueError("tile_heads must divide Hq / Hkv")
    r = G // T
    if r == 1:
        return Hkv, pools
    return Hkv * r, tuple(np.ascontiguousarray(np.repeat(x, r, axis=1))
                          for x in pools)


def decode(q, k, v, scale, ln_lambda, Bc, num_splits, n_threads=0, window=0,
           tile_heads=None):
    """BLASST decode forward with split-KV and log-sum-exp merge.

    ``window`` > 0: the token sees only the last ``window`` keys (sliding
    window); the splits divide the blocks holding them.  ``tile_heads``:
    query heads per decode tile (default: all Hq/Hkv heads of a KV head).

    q [B,Hq,d], k/v [B,Hkv,Lkv,d] bf16.  Returns ``o`` [B,Hq,d], ``lse``
    [B,Hq], ``o_part`` [B,Hq,S,d], ``lse_part`` [B,Hq,S], ``mask``
    [B,Hkv',nk], ``margin`` [B,Hkv',nk] (Hkv' = Hq / tile_heads), ``visited``,
    ``skipped``.
    """
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, d = qb.shape
    Hkv, (kb, vb) = _tile_heads(Hq, kb.shape[1], tile_heads, kb, vb)
    Lkv = kb.shape[2]
    nk = -(-Lkv // Bc)
    S = int(num_splits)
    o = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    op = np.zeros((B, Hq, S, d), np.float64)
    lp = np.zeros((B, Hq, S), np.float64)
    mask = np.zeros((B, Hkv, nk), np.uint8)
    margin = np.zeros((B, Hkv, nk), np.float64)
    counts = np.zeros(2, np.int64)
    rc = lib.oracle_decode_window(
        _ptr(qb, _u16p), _ptr(kb, _u16p), _ptr(vb, _u16p),
        B, Hq, Hkv, Lkv, d, float(scale), int(window), float(ln_lambda), Bc, S,
        _ptr(o, _dp), _ptr(lse, _dp), _ptr(op, _dp), _ptr(lp, _dp),
        _ptr(mask, _u8p), _ptr(margin, _dp), _ptr(counts, _i64p),
        int(n_threads))
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    threads = n_threads if n_threads > 0 else n_threads_default()
    return dict(o=o, lse=lse, o_part=op, lse_part=lp, mask=mask,
                margin=margin, visited=int(counts[0]),
                skipped=int(counts[1]), threads=threads)


def decode_batched(q, k, v, scale, ln_lambda, Bc, num_splits, batch,
                   n_threads=0, tile_heads=None):
    """Decode with the batched decision rule: blocks of each split are judged
    in batches of ``batch`` against the max over all earlier blocks and the
    whole batch.  ``batch`` = 1 is :func:`decode`.  Same outputs as
    :func:`decode`."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, d = qb.shape
    Hkv, (kb, vb) = _tile_heads(Hq, kb.shape[1], tile_heads, kb, vb)
    Lkv = kb.shape[2]
    nk = -(-Lkv // Bc)
    S = int(num_splits)
    o = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    op = np.zeros((B, Hq, S, d), np.float64)
    lp = np.zeros((B, Hq, S), np.float64)
    mask = np.zeros((B, Hkv, nk), np.uint8)
    margin = np.zeros((B, Hkv, nk), np.float64)
    counts = np.zeros(2, np.int64)
    rc = lib.oracle_decode_batched(
        _ptr(qb, _u16p), _ptr(kb, _u16p), _ptr(vb, _u16p),
        B, Hq, Hkv, Lkv, d, float(scale), float(ln_lambda), Bc, S, int(batch),
        _ptr(o, _dp), _ptr(lse, _dp), _ptr(op, _dp), _ptr(lp, _dp),
        _ptr(mask, _u8p), _ptr(margin, _dp), _ptr(counts, _i64p),
        int(n_threads))
    if rc != 0:
        raise ValueError("oracle_decode_batched rejected its arguments")
    threads = n_threads if n_threads > 0 else n_threads_default()
    return dict(o=o, lse=lse, o_part=op, lse_part=lp, mask=mask,
                margin=margin, visited=int(counts[0]),
                skipped=int(counts[1]), threads=threads)


def _i32(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x), dtype=np.int32)


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale, ln_lambda,
                 num_splits, Bc=64, per_length=False, nk_max=None,
                 page_stride=None, n_threads=0, tile_heads=None):
    """Paged, variable-length decode: gather, then the decode above.

    q [B,Hq,d] bf16.  k_pages / v_pages: either [num_pages,Hkv,page_size,d]
    bf16 (made contiguous), or flat 1-D pools with ``page_stride`` given
    (then pass ``(pool, num_pages, Hkv, page_size, d)`` tuples).
    block_table [B,max_pages] int32, seq_lens [B] int32.  ``per_length``:
    ln_lambda is ln a and sequence b uses min(0, ln a - ln L_b).
    Returns the keys of ``decode`` with mask/margin [B,Hkv',nk_max]
    (``tile_heads`` as in :func:`decode`; 4-D pools only when it is set).
    """
    lib = _load()
    qb = _bits(q)
    B, Hq, d = qb.shape
    if isinstance(k_pages, tuple):
        kp, num_pages, Hkv, ps, d2 = k_pages
        if tile_heads is not None and tile_heads != Hq // Hkv:
            raise ValueError("tile_heads needs [num_pages,Hkv,page,d] pools")
        vp = v_pages[0]
        kb, vb = _bits(kp).reshape(-1), _bits(vp).reshape(-1)
        stride = int(page_stride)
    else:
        kb, vb = _bits(k_pages), _bits(v_pages)
        if (page_stride is not None and tile_heads is not None
                and tile_heads != Hq // kb.shape[1]):
            raise ValueError("tile_heads with a padded page stride")
        Hkv, (kb, vb) = _tile_heads(Hq, kb.shape[1], tile_heads, kb, vb)
        num_pages, _, ps, d2 = kb.shape
        stride = Hkv * ps * d2 if page_stride is None else int(page_stride)
    assert d2 == d
    bt = _i32(block_table)
    sl = _i32(seq_lens).reshape(-1)
    assert sl.shape[0] == B and bt.shape[0] == B
    max_pages = bt.shape[1] if bt.ndim == 2 else 0
    if nk_max is None:
        nk_max = -(-int(max_pages * ps) // Bc)
    S = int(num_splits)
    o = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    op = np.zeros((B, Hq, S, d), np.float64)
    lp = np.zeros((B, Hq, S), np.float64)
    mask = np.zeros((B, Hkv, nk_max), np.uint8)
    margin = np.zeros((B, Hkv, nk_max), np.float64)
    counts = np.zeros(2, np.int64)
    rc = lib.oracle_decode_paged(
        _ptr(qb, _u16p), _ptr(kb, _u16p), _ptr(vb, _u16p), stride,
        int(num_pages), int(ps), _ptr(bt, _i32p), int(max_pages),
        _ptr(sl, _i32p), B, Hq, Hkv, d, float(scale), float(ln_lambda),
        int(bool(per_length)), Bc, S, int(nk_max),
        _ptr(o, _dp), _ptr(lse, _dp), _ptr(op, _dp), _ptr(lp, _dp),
        _ptr(mask, _u8p), _ptr(margin, _dp), _ptr(counts, _i64p),
        int(n_threads))
    if rc != 0:
        raise ValueError("oracle_decode_paged rejected its arguments")
    threads = n_threads if n_threads > 0 else n_threads_default()
    return dict(o=o, lse=lse, o_part=op, lse_part=lp, mask=mask,
                margin=margin, visited=int(counts[0]),
                skipped=int(counts[1]), threads=threads)


def combine(o_part, lse_part):
    """Log-sum-exp merge of split partials: o_part [n,S,d], lse_part [n,S]."""
    lib = _load()
    op = np.ascontiguousarray(o_part, dtype=np.float64)
    lp = np.ascontiguousarray(lse_part, dtype=np.float64)
    n, S, d = op.shape
    o = np.zeros((n, d), np.float64)
    lse = np.zeros(n, np.float64)
    lib.oracle_combine(_ptr(op, _dp), _ptr(lp, _dp), n, S, d, _ptr(o, _dp),
                       _ptr(lse, _dp))
    return o, lse


def split_begin(nk, S, s):
    return _load().oracle_split_begin(nk, S, s)


def sparsity(res):
    return res["skipped"] / res["visited"] if res["visited"] else 0.0


def lambda_fit(lambdas, lengths):
    """Least-squares fit of lambda = a / L in log space: a = exp(mean ln(lambda*L))."""
    vals = [math.log(lam * L) for lam, L in zip(lambdas, lengths)]
    return math.exp(sum(vals) / len(vals))


from .backward import prefill_backward, restricted_forward  # noqa: E402,F401
