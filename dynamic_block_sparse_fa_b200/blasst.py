"""Thin ctypes binding of libblasst.so (include/blasst.h).

Argument marshalling only: every function forwards to the C entry point of
the same name, passing torch tensors as device pointers and the current
CUDA stream.  Outputs the caller does not provide are allocated with torch
(device memory plumbing); all computation runs in the library's kernels.
There is no fallback: if the library is missing, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libblasst.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python dynamic_block_sparse_fa_b200/build.py` (needs nvcc)")

_lib = ctypes.CDLL(LIB_PATH)

BLASST_OK = 0
_STATUS = {
    0: "BLASST_OK", 1: "BLASST_ERR_INVALID_ARG",
    2: "BLASST_ERR_UNSUPPORTED_SHAPE", 3: "BLASST_ERR_MISALIGNED",
    4: "BLASST_ERR_CUDA", 5: "BLASST_ERR_TIMEOUT",
    6: "BLASST_ERR_NO_CONVERGE", 7: "BLASST_ERR_WORKSPACE",
}


class BlasstError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.blasst_strerror(status).decode()
        detail = _lib.blasst_last_error().decode()
        super().__init__(f"{where}: {_STATUS.get(status, status)} ({msg})"
                         + (f": {detail}" if detail and status == 4 else ""))


class SkipStats(ctypes.Structure):
    """Host struct of device pointers (blasst_skip_stats_t)."""
    _fields_ = [("counters", ctypes.c_void_p), ("mask", ctypes.c_void_p),
                ("margin", ctypes.c_void_p)]


class CalibSample(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("q", ctypes.c_void_p),
                ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("B", ctypes.c_int), ("Hq", ctypes.c_int),
                ("Hkv", ctypes.c_int), ("Lq", ctypes.c_int),
                ("Lkv", ctypes.c_int), ("d", ctypes.c_int),
                ("scale", ctypes.c_float), ("causal", ctypes.c_int),
                ("Br", ctypes.c_int), ("Bc", ctypes.c_int),
                ("num_splits", ctypes.c_int)]


class CalibResult(ctypes.Structure):
    _fields_ = [("ln_lambda", ctypes.c_double), ("lambda_", ctypes.c_double),
                ("a", ctypes.c_double), ("achieved", ctypes.c_double),
                ("L", ctypes.c_int), ("iterations", ctypes.c_int),
                ("visited", ctypes.c_ulonglong),
                ("skipped", ctypes.c_ulonglong)]


_vp, _i, _f, _d, _sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float,
                        ctypes.c_double, ctypes.c_size_t)
_lib.blasst_prefill.restype = _i
_lib.blasst_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                _i, _f, _i, _f, _i, _i,
                                ctypes.POINTER(SkipStats), _vp]
_lib.blasst_prefill_window.restype = _i
_lib.blasst_prefill_window.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                       _i, _i, _f, _i, _i, _f, _i, _i,
                                       ctypes.POINTER(SkipStats), _vp]
_lib.blasst_decode.restype = _i
_lib.blasst_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                               _f, _f, _i, _i, _vp, _sz,
                               ctypes.POINTER(SkipStats), _vp]
_lib.blasst_decode_window.restype = _i
_lib.blasst_decode_window.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                      _i, _f, _i, _f, _i, _i, _vp, _sz,
                                      ctypes.POINTER(SkipStats), _vp]
_lib.blasst_decode_batched.restype = _i
_lib.blasst_decode_batched.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                       _i, _f, _f, _i, _i, _i, _vp, _sz,
                                       ctypes.POINTER(SkipStats), _vp]
_lib.blasst_decode_paged.restype = _i
_lib.blasst_decode_paged.argtypes = [_vp, _vp, _vp, ctypes.c_longlong, _i, _i,
                                     _vp, _i, _vp, _i, _vp, _vp, _i, _i, _i,
                                     _i, _f, _f, _i, _i, _vp, _sz,
                                     ctypes.POINTER(SkipStats), _vp]
_lib.blasst_decode_noalloc.restype = _i
_lib.blasst_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                       _i, _f, _f, _i, _i,
                                       ctypes.POINTER(SkipStats), _vp]
_lib.blasst_decode_wide.restype = _i
_lib.blasst_decode_wide.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                    _i, _f, _f, _i, _i, _vp, _sz, _vp, _vp]
_lib.blasst_mla_decode.restype = _i
_lib.blasst_mla_decode.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f,
                                   _f, _i, _vp, _sz, _vp, _vp]
_lib.blasst_mla_decode_workspace_size.restype = _sz
_lib.blasst_mla_decode_workspace_size.argtypes = [_i, _i, _i]
_lib.blasst_mla_decode_splits.restype = _i
_lib.blasst_mla_decode_splits.argtypes = [_i, _i]
_lib.blasst_prefill_backward.restype = _i
_lib.blasst_prefill_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                         _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                         _i, _f, _i, _i, _i, _vp, _sz, _vp]
_lib.blasst_prefill_backward_workspace_size.restype = _sz
_lib.blasst_prefill_backward_workspace_size.argtypes = [_i, _i, _i, _i]
_lib.blasst_decode_workspace_size.restype = _sz
_lib.blasst_decode_workspace_size.argtypes = [_i, _i, _i, _i]
_lib.blasst_decode_splits.restype = _i
_lib.blasst_decode_splits.argtypes = [_i, _i, _i, _i]
_lib.blasst_decode_wide_splits.restype = _i
_lib.blasst_decode_wide_splits.argtypes = [_i, _i, _i, _i]
_lib.blasst_decode_group_splits.restype = _i
_lib.blasst_decode_group_splits.argtypes = [_i, _i, _i, _i, _i]
_lib.blasst_calibrate.restype = _i
_lib.blasst_calibrate.argtypes = [_d, ctypes.POINTER(CalibSample), _d, _vp,
                                  ctypes.POINTER(CalibResult), _vp]
_lib.blasst_fit_a.restype = _d
_lib.blasst_fit_a.argtypes = [_i, ctypes.POINTER(_d), ctypes.POINTER(_i)]
_lib.blasst_skip_stats_reset.restype = _i
_lib.blasst_skip_stats_reset.argtypes = [_vp, _vp]
_lib.blasst_check_device_error.restype = _i
_lib.blasst_check_device_error.argtypes = [ctypes.POINTER(_i)]
_lib.blasst_selftest_wait_timeout.restype = _i
_lib.blasst_selftest_wait_timeout.argtypes = [ctypes.c_longlong, _vp]
_lib.blasst_strerror.restype = ctypes.c_char_p
_lib.blasst_strerror.argtypes = [_i]
_lib.blasst_last_error.restype = ctypes.c_char_p
_lib.blasst_last_error.argtypes = []
_lib.blasst_version.restype = ctypes.c_char_p
_lib.blasst_version.argtypes = []

EXPORTED = ["blasst_prefill", "blasst_decode", "blasst_decode_noalloc",
            "blasst_decode_paged",
            "blasst_decode_workspace_size",
            "blasst_decode_splits", "blasst_decode_wide_splits",
            "blasst_decode_group_splits", "blasst_calibrate", "blasst_fit_a",
            "blasst_skip_stats_reset", "blasst_check_device_error",
            "blasst_selftest_wait_timeout",
            "blasst_strerror", "blasst_last_error", "blasst_version"]


def _check(status, where):
    if status != BLASST_OK:
        raise BlasstError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _arg(t, name, dtype=torch.bfloat16, contiguous=True):
    """Device pointer of a tensor argument after checking what the C ABI
    cannot see: a CUDA tensor, of the given dtype (None: any, for byte
    workspaces), dense in memory (the ABI takes no strides)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor (got {t.device})")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _overlaps(a, b):
    """Whether the storage spans of two tensors intersect (None: never)."""
    if a is None or b is None or a.device != b.device:
        return False
    a0 = a.data_ptr()
    b0 = b.data_ptr()
    a1 = a0 + a.numel() * a.element_size()
    b1 = b0 + b.numel() * b.element_size()
    return a0 < b1 and b0 < a1


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Stats:
    """Device skip counters (uint64[2]: visited, skipped) and an optional
    per-(tile, block) decision mask, allocated with torch."""

    def __init__(self, device="cuda", mask_numel: int = 0,
                 margin: bool = False):
        self.counters = torch.zeros(2, dtype=torch.int64, device=device)
        self.mask = (torch.zeros(mask_numel, dtype=torch.uint8, device=device)
                     if mask_numel else None)
        self.margin = (torch.full((mask_numel,), float("nan"),
                                  dtype=torch.float32, device=device)
                       if margin and mask_numel else None)
        self._c = SkipStats(
            self.counters.data_ptr(),
            self.mask.data_ptr() if self.mask is not None else None,
            self.margin.data_ptr() if self.margin is not None else None)

    @property
    def c_struct(self):
        return ctypes.byref(self._c)

    def reset(self, stream=None):
        blasst_skip_stats_reset(self.counters, stream)
        if self.mask is not None:
            self.mask.zero_()
        if self.margin is not None:
            self.margin.fill_(float("nan"))

    def near_ties(self, width: float = 1e-3) -> int:
        """Visited pairs whose decision margin is within `width` of 0 (the
        margin buffer must have been requested and filled)."""
        if self.margin is None:
            raise ValueError("Stats(margin=True) was not requested")
        m = self.margin
        return int(((self.mask > 0) & (m.abs() < width)).sum().item())

    def read(self):
        v, s = (int(x) for x in self.counters.tolist())
        return v, s

    def sparsity(self):
        v, s = self.read()
        return s / v if v else 0.0


def blasst_version() -> str:
    return _lib.blasst_version().decode()


def blasst_strerror(status: int) -> str:
    return _lib.blasst_strerror(status).decode()


def blasst_last_error() -> str:
    return _lib.blasst_last_error().decode()


def blasst_skip_stats_reset(counters: torch.Tensor, stream=None):
    _check(_lib.blasst_skip_stats_reset(_arg(counters, "counters", torch.int64),
                                        _stream(stream)),
           "blasst_skip_stats_reset")


def blasst_check_device_error():
    """Returns (status, where): status 0, BLASST_ERR_TIMEOUT (5, a wait gave
    up) or BLASST_ERR_INVALID_ARG (1, a paged-decode length or page id out of
    range); for either error `where` is a string naming the first one."""
    where = ctypes.c_int(0)
    st = _lib.blasst_check_device_error(ctypes.byref(where))
    if st not in (0, 1, 5):
        _check(st, "blasst_check_device_error")
    if st in (1, 5):
        return st, f"{where.value}: {blasst_last_error()}"
    return st, where.value


def blasst_selftest_wait_timeout(limit_cycles=1_000_000, stream=None):
    """Launch the diagnostic kernel whose bounded wait is bound to give up."""
    _check(_lib.blasst_selftest_wait_timeout(int(limit_cycles), _stream(stream)),
           "blasst_selftest_wait_timeout")


def blasst_prefill(q, k, v, *, scale=None, causal=True, ln_lambda=-math.inf,
                   Br=128, Bc=128, o=None, lse=None, want_lse=True,
                   stats: Stats | None = None, stats_only=False, stream=None,
                   window=0):
    """BLASST prefill forward.  q [B,Hq,Lq,d], k/v [B,Hkv,Lkv,d] bf16 CUDA.

    window > 0 (causal, 128x128 tiles): each query sees the ``window`` keys
    ending at its diagonal (blasst_prefill_window).  Returns (o, lse); both
    None when stats_only (decisions and counters only)."""
    B, Hq, Lq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if not stats_only:
        if o is None:
            o = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(B, Hq, Lq, dtype=torch.float32, device=q.device)
    else:
        o, lse = None, None
    st = _lib.blasst_prefill_window(
        _arg(q, "q"), _arg(k, "k"), _arg(v, "v"), _arg(o, "o"),
        _arg(lse, "lse", torch.float32), B, Hq, Hkv, Lq, Lkv, d,
        float(scale), int(bool(causal)), int(window), float(ln_lambda), Br, Bc,
        stats.c_struct if stats is not None else None, _stream(stream))
    _check(st, "blasst_prefill_window")
    return o, lse


def blasst_prefill_window(q, k, v, *, window, **kw):
    """blasst_prefill with a causal sliding window of ``window`` keys."""
    return blasst_prefill(q, k, v, window=window, **kw)


def blasst_mla_decode_splits(B, L) -> int:
    return int(_lib.blasst_mla_decode_splits(B, L))


def blasst_mla_decode_workspace_size(B, H, num_splits) -> int:
    return int(_lib.blasst_mla_decode_workspace_size(B, H, num_splits))


def blasst_mla_decode(q, cache, *, d_v=512, scale=None, ln_lambda=-math.inf,
                      num_splits=0, o=None, lse=None, want_lse=True,
                      workspace=None, stats: Stats | None = None,
                      stats_only=False, stream=None):
    """MLA decode.  q [B,H,576], cache [B,L,576] bf16 CUDA (one shared
    latent row per key; value = its first d_v = 512 columns).  Returns
    (o [B,H,512], lse [B,H]); both None when stats_only."""
    B, H, dqk = q.shape
    L = cache.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    S = num_splits if num_splits > 0 else blasst_mla_decode_splits(B, L)
    ws_bytes = 0
    if not stats_only:
        if o is None:
            o = torch.empty(B, H, d_v, dtype=q.dtype, device=q.device)
        if lse is None and want_lse:
            lse = torch.empty(B, H, dtype=torch.float32, device=q.device)
        need = blasst_mla_decode_workspace_size(B, H, S)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8,
                                    device=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    else:
        o, lse, workspace = None, None, None
    st = _lib.blasst_mla_decode(
        _arg(q, "q"), _arg(cache, "cache"), _arg(o, "o"),
        _arg(lse, "lse", torch.float32), B, H, L, dqk, d_v,
        float(scale), float(ln_lambda), S, _arg(workspace, "workspace", None),
        ws_bytes,
        stats.c_struct if stats is not None else None, _stream(stream))
    _check(st, "blasst_mla_decode")
    return o, lse


def blasst_prefill_backward_workspace_size(B, Hq, Lq, d=128) -> int:
    return int(_lib.blasst_prefill_backward_workspace_size(B, Hq, Lq, d))


def blasst_prefill_backward(q, k, v, o, lse, dout, *, mask=None, scale=None,
                            causal=True, Br=128, Bc=128, dq=None, dk=None,
                            dv=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of a blasst_prefill forward with its decisions
    held fixed.  q [B,Hq,Lq,d], k/v [B,Hkv,Lkv,d], o/dout [B,Hq,Lq,d] bf16,
    lse [B,Hq,Lq] f32 (the forward's), mask: the forward's decision bytes
    (Stats.mask) or None for the dense backward."""
    B, Hq, Lq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    # dq also holds the work order of a masked call before it is written
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse),
                    ("dout", dout), ("mask", mask)):
        if _overlaps(dq, t):
            raise ValueError(f"dq overlaps {name}")
    need = blasst_prefill_backward_workspace_size(B, Hq, Lq, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8,
                                device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.blasst_prefill_backward(
        _arg(q, "q"), _arg(k, "k"), _arg(v, "v"), _arg(o, "o"),
        _arg(dout, "dout"), _arg(lse, "lse", torch.float32),
        _arg(mask, "mask", torch.uint8), _arg(dq, "dq"), _arg(dk, "dk"),
        _arg(dv, "dv"), B, Hq, Hkv, Lq, Lkv, d, float(scale),
        int(bool(causal)), Br, Bc, _arg(workspace, "workspace", None), ws_bytes,
        _stream(stream))
    _check(st, "blasst_prefill_backward")
    return dq, dk, dv


def blasst_decode_window(q, k, v, *, window, **kw):
    """blasst_decode over the last ``window`` keys of the cache."""
    return blasst_decode(q, k, v, window=window, **kw)


def blasst_decode_batched(q, k, v, *, batch=2, scale=None,
                          ln_lambda=-math.inf, Bc=64, num_splits=0, o=None,
                          lse=None, want_lse=True, workspace=None,
                          stats: Stats | None = None, stats_only=False,
                          stream=None):
    """Decode with the batched decision rule: blocks are scored in pairs
    and each is judged against the max over earlier blocks and the pair
    (batch = 2; batch = 1 is the sequential rule of blasst_decode, always on
    the CUDA-core kernel).  Returns (o, lse)."""
    B, Hq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    S = num_splits if num_splits > 0 else blasst_decode_splits(B, Hkv, Lkv, Bc)
    ws_bytes = 0
    if not stats_only:
        if o is None:
            o = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
        need = blasst_decode_workspace_size(B, Hq, d, S)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    else:
        o, lse, workspace = None, None, None
    st = _lib.blasst_decode_batched(
        _arg(q, "q"), _arg(k, "k"), _arg(v, "v"), _arg(o, "o"),
        _arg(lse, "lse", torch.float32), B, Hq, Hkv, Lkv, d,
        float(scale), float(ln_lambda), Bc, S, int(batch),
        _arg(workspace, "workspace", None),
        ws_bytes, stats.c_struct if stats is not None else None,
        _stream(stream))
    _check(st, "blasst_decode_batched")
    return o, lse


def blasst_decode_workspace_size(B, Hq, d, num_splits) -> int:
    return int(_lib.blasst_decode_workspace_size(B, Hq, d, num_splits))


def blasst_decode_splits(B, Hkv, Lkv, Bc=64) -> int:
    return int(_lib.blasst_decode_splits(B, Hkv, Lkv, Bc))


def blasst_decode_wide_splits(B, Hkv, Lkv, Bc=64) -> int:
    return int(_lib.blasst_decode_wide_splits(B, Hkv, Lkv, Bc))


def blasst_decode_group_splits(B, Hq, Hkv, Lkv, Bc=64) -> int:
    return int(_lib.blasst_decode_group_splits(B, Hq, Hkv, Lkv, Bc))


def blasst_decode(q, k, v, *, scale=None, ln_lambda=-math.inf, Bc=64,
                  num_splits=0, o=None, lse=None, want_lse=True,
                  workspace=None, stats: Stats | None = None,
                  stats_only=False, stream=None, window=0):
    """BLASST decode forward.  q [B,Hq,d], k/v [B,Hkv,Lkv,d] bf16 CUDA.

    window > 0: the token sees only the last ``window`` keys
    (blasst_decode_window).  Returns (o, lse); both None when stats_only."""
    B, Hq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    jlo = (Lkv - window) // Bc if 0 < window < Lkv else 0
    S = (num_splits if num_splits > 0
         else blasst_decode_group_splits(B, Hq, Hkv, Lkv - jlo * Bc, Bc))
    ws_bytes = 0
    if not stats_only:
        if o is None:
            o = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
        need = blasst_decode_workspace_size(B, Hq, d, S)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    else:
        o, lse, workspace = None, None, None
    st = _lib.blasst_decode_window(
        _arg(q, "q"), _arg(k, "k"), _arg(v, "v"), _arg(o, "o"),
        _arg(lse, "lse", torch.float32), B, Hq, Hkv, Lkv, d,
        float(scale), int(window), float(ln_lambda), Bc, S,
        _arg(workspace, "workspace", None),
        ws_bytes, stats.c_struct if stats is not None else None,
        _stream(stream))
    _check(st, "blasst_decode_window")
    return o, lse


def blasst_decode_wide(q, k, v, *, scale=None, ln_lambda=-math.inf, Bc=64,
                       num_splits=0, o=None, lse=None, want_lse=True,
                       workspace=None, stats: Stats | None = None,
                       stats_only=False, stream=None):
    """Decode on the tensor core with all G = Hq/Hkv (<= 128) heads of a KV
    head as one tile (blasst_decode_wide).  Same arguments and results as
    blasst_decode; the mask layout is [B, Hkv, nk]."""
    B, Hq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    S = (num_splits if num_splits > 0
         else blasst_decode_wide_splits(B, Hkv, Lkv, Bc))
    ws_bytes = 0
    if not stats_only:
        if o is None:
            o = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
        need = blasst_decode_workspace_size(B, Hq, d, S)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    else:
        o, lse, workspace = None, None, None
    st = _lib.blasst_decode_wide(
        _arg(q, "q"), _arg(k, "k"), _arg(v, "v"), _arg(o, "o"),
        _arg(lse, "lse", torch.float32), B, Hq, Hkv, Lkv, d,
        float(scale), float(ln_lambda), Bc, S,
        _arg(workspace, "workspace", None), ws_bytes,
        stats.c_struct if stats is not None else None, _stream(stream))
    _check(st, "blasst_decode_wide")
    return o, lse


def blasst_decode_paged(q, k_pages, v_pages, block_table, seq_lens, *,
                        max_seq_len=None, scale=None, ln_lambda=-math.inf,
                        per_length=False, num_splits=0, o=None, lse=None,
                        want_lse=True, workspace=None,
                        stats: Stats | None = None, stats_only=False,
                        stream=None):
    """BLASST decode over a paged KV cache.

    q [B,Hq,d] bf16.  k_pages / v_pages: [num_pages, Hkv, page_size, d] bf16
    views whose last three dimensions are contiguous (dimension 0 may have
    any stride, e.g. the K and V halves of one interleaved pool
    [num_pages, 2, Hkv, page_size, d]); both must have the same page stride.
    block_table [B, max_pages] int32, seq_lens [B] int32, on the device.
    max_seq_len: host upper bound on seq_lens (default: what the table
    holds, max_pages * page_size; it sizes the split policy and the mask).
    per_length: ln_lambda is ln a and sequence b uses min(0, ln a - ln L_b).
    Returns (o, lse); both None when stats_only.  Bad lengths or page ids
    are caught on the device: see blasst_check_device_error()."""
    B, Hq, d = q.shape
    P, Hkv, ps, d2 = k_pages.shape
    if d2 != d or tuple(v_pages.shape) != tuple(k_pages.shape):
        raise ValueError("k_pages / v_pages shapes")
    for t in (k_pages, v_pages):
        if t.stride()[1:] != (ps * d, d, 1):
            raise ValueError("pages must be contiguous inside a page")
    if k_pages.stride(0) != v_pages.stride(0):
        raise ValueError("k_pages and v_pages must share the page stride")
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_table and seq_lens must be int32")
    block_table = block_table.contiguous()
    seq_lens = seq_lens.contiguous()
    max_pages = block_table.shape[1]
    if max_seq_len is None:
        max_seq_len = max_pages * ps
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    S = num_splits if num_splits > 0 else blasst_decode_splits(
        B, Hkv, max_seq_len, 64)
    ws_bytes = 0
    if not stats_only:
        if o is None:
            o = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
        need = blasst_decode_workspace_size(B, Hq, d, S)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    else:
        o, lse, workspace = None, None, None
    st = _lib.blasst_decode_paged(
        _arg(q, "q"), _arg(k_pages, "k_pages", contiguous=False),
        _arg(v_pages, "v_pages", contiguous=False), int(k_pages.stride(0)), P,
        ps, _arg(block_table, "block_table", torch.int32), max_pages,
        _arg(seq_lens, "seq_lens", torch.int32), int(max_seq_len),
        _arg(o, "o"), _arg(lse, "lse", torch.float32), B, Hq, Hkv, d,
        float(scale), float(ln_lambda), int(bool(per_length)), S,
        _arg(workspace, "workspace", None), ws_bytes,
        stats.c_struct if stats is not None else None, _stream(stream))
    _check(st, "blasst_decode_paged")
    return o, lse


def blasst_decode_noalloc(q, k, v, *, scale=None, ln_lambda=-math.inf, Bc=64,
                          num_splits=0, o=None, lse=None, want_lse=True,
                          stats: Stats | None = None, stats_only=False,
                          stream=None):
    """blasst_decode with the split partials in the library's own fixed
    device array (8 MiB per device) instead of a caller workspace; for
    callers that may not allocate device memory at call time.  Calls that
    could overlap on the GPU share that array and must be serialised."""
    B, Hq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if not stats_only:
        if o is None:
            o = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    else:
        o, lse = None, None
    st = _lib.blasst_decode_noalloc(
        _arg(q, "q"), _arg(k, "k"), _arg(v, "v"), _arg(o, "o"),
        _arg(lse, "lse", torch.float32), B, Hq, Hkv, Lkv, d,
        float(scale), float(ln_lambda), Bc, num_splits,
        stats.c_struct if stats is not None else None, _stream(stream))
    if st == 7:
        raise BlasstError(st, "blasst_decode_noalloc: " + blasst_last_error())
    _check(st, "blasst_decode_noalloc")
    return o, lse


def blasst_calibrate(target, *, mode, q, k, v, scale=None, causal=True,
                     Br=128, Bc=128, num_splits=0, tol=0.002,
                     counters=None, stream=None, raise_on_no_converge=True):
    """Bisection of ln(lambda) until the sample's sparsity reaches `target`.

    mode 'prefill' (q [B,Hq,Lq,d]) or 'decode' (q [B,Hq,d]).  Returns a dict
    with ln_lambda, lambda, a (= lambda * Lkv), achieved, L, iterations,
    visited, skipped, status."""
    m = {"prefill": 0, "decode": 1}[mode]
    d = q.shape[-1]
    B, Hq = q.shape[0], q.shape[1]
    Lq = q.shape[2] if m == 0 else 1
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if counters is None:
        counters = torch.zeros(2, dtype=torch.int64, device=q.device)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _arg(t, n)
    smp = CalibSample(m, q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Hq, Hkv,
                      Lq, Lkv, d, float(scale), int(bool(causal)), Br, Bc,
                      num_splits)
    res = CalibResult()
    st = _lib.blasst_calibrate(float(target), ctypes.byref(smp), float(tol),
                               _arg(counters, "counters", torch.int64),
                               ctypes.byref(res),
                               _stream(stream))
    if st != BLASST_OK and (st != 6 or raise_on_no_converge):
        _check(st, "blasst_calibrate")
    return dict(ln_lambda=res.ln_lambda, lambda_=res.lambda_, a=res.a,
                achieved=res.achieved, L=res.L, iterations=res.iterations,
                visited=res.visited, skipped=res.skipped, status=st)


def blasst_fit_a(lambdas, lengths) -> float:
    n = len(lambdas)
    la = (ctypes.c_double * n)(*lambdas)
    le = (ctypes.c_int * n)(*lengths)
    return float(_lib.blasst_fit_a(n, la, le))
