"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/blasst.h declares, and its host-side logic (argument
validation, split policy, workspace sizing, the lambda = a/L fit) behaves.
No call here reaches a CUDA runtime function: every compute entry point is
given arguments that validation rejects first."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "blasst.h")


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_blasst_build", os.path.join(ROOT, "dynamic_block_sparse_fa_b200",
                                      "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    path = build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(blasst_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("blasst_prefill", "blasst_decode", "blasst_calibrate",
                 "blasst_decode_splits", "blasst_decode_workspace_size",
                 "blasst_skip_stats_reset", "blasst_strerror"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared but not exported"


def test_binding_uses_the_same_names():
    import dynamic_block_sparse_fa_b200 as m
    for name in declared_functions():
        if name == "blasst_last_error":
            continue
        assert hasattr(m, name), f"binding lacks {name}"


def _prefill(lib, q=0x1000, k=0x1000, v=0x1000, o=0x2000, B=1, Hq=2, Hkv=2,
             Lq=128, Lkv=128, d=128, scale=0.088, causal=1, lnl=-1.0, Br=128,
             Bc=128):
    f = lib.blasst_prefill
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 + [
        ctypes.c_float, ctypes.c_int, ctypes.c_float, ctypes.c_int,
        ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    return f(q, k, v, o, None, B, Hq, Hkv, Lq, Lkv, d, scale, causal, lnl, Br,
             Bc, None, None)


def test_prefill_validation(lib):
    assert _prefill(lib, q=None) == 1                  # null input
    assert _prefill(lib, lnl=0.5) == 1                 # ln lambda > 0
    assert _prefill(lib, lnl=float("nan")) == 1
    assert _prefill(lib, Lq=256, Lkv=128) == 1         # causal, Lq > Lkv
    assert _prefill(lib, Hq=3, Hkv=2) == 1             # Hq % Hkv
    assert _prefill(lib, d=96) == 2                    # head dim not built
    assert _prefill(lib, Br=64, Bc=128) == 2           # tile pair not built
    assert _prefill(lib, q=0x1001) == 3                # misaligned
    assert _prefill(lib, B=0) == 1
    assert _prefill(lib, scale=float("inf")) == 1


def _decode(lib, q=0x1000, k=0x1000, v=0x1000, o=0x2000, B=1, Hq=4, Hkv=1,
            Lkv=256, d=128, lnl=-1.0, Bc=64, S=1, ws=None, ws_bytes=0):
    f = lib.blasst_decode
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [
        ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    return f(q, k, v, o, None, B, Hq, Hkv, Lkv, d, 0.088, lnl, Bc, S, ws,
             ws_bytes, None, None)


def test_decode_validation(lib):
    assert _decode(lib, k=None) == 1
    assert _decode(lib, lnl=1.0) == 1
    assert _decode(lib, S=5) == 1                      # more splits than blocks
    assert _decode(lib, d=96) == 2                     # d is 64 or 128
    assert _decode(lib, d=64) == 7                     # d = 64 accepted (no workspace)
    assert _decode(lib, Bc=128) == 2
    assert _decode(lib, Hq=12, Hkv=4) == 2             # G = 3 not built
    assert _decode(lib, v=0x1008) == 3
    assert _decode(lib) == 7                           # no workspace
    assert _decode(lib, ws=0x4000, ws_bytes=64) == 7   # too small


def _noalloc(lib, B, Hq, Hkv, Lkv, S, d=128, o=0x2000):
    f = lib.blasst_decode_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [
        ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_void_p]
    return f(0x1000, 0x1000, 0x1000, o, None, B, Hq, Hkv, Lkv, d, 0.088,
             -1.0, 64, S, None, None)


def test_decode_noalloc_size_guard_needs_no_device(lib):
    """Shapes whose split partials exceed the 8 MiB built-in scratch are
    refused before the library asks the runtime for anything (no device
    here), with a message naming both sizes."""
    # 64 sequences x 64 heads x 8 splits x 129 floats = 16.9 MB of partials
    assert _noalloc(lib, 64, 64, 8, 512, 8) == 7
    lib.blasst_last_error.restype = ctypes.c_char_p
    msg = lib.blasst_last_error().decode()
    assert "scratch holds 8388608" in msg
    assert _noalloc(lib, 0, 64, 8, 512, 8) == 1
    assert _noalloc(lib, 1, 4, 1, 512, -1) == 1


def _mla(lib, q=0x1000, c=0x1000, o=0x2000, B=1, H=8, L=256, dqk=576,
         dv=512, lnl=-1.0, S=1, ws=None, ws_bytes=0):
    f = lib.blasst_mla_decode
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 5 + [
        ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
        ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    return f(q, c, o, None, B, H, L, dqk, dv, 0.04, lnl, S, ws, ws_bytes,
             None, None)


def test_mla_decode_validation(lib):
    """Argument checks of blasst_mla_decode, all taken before any launch."""
    assert _mla(lib, q=None) == 1
    assert _mla(lib, B=0) == 1
    assert _mla(lib, lnl=0.5) == 1                     # ln lambda > 0
    assert _mla(lib, H=129) == 2                       # at most 128 heads
    assert _mla(lib, dqk=512) == 2                     # d_qk 576 only
    assert _mla(lib, dv=256) == 2                      # d_v 512 only
    assert _mla(lib, c=0x1008) == 3                    # misaligned cache
    assert _mla(lib, S=5) == 1                         # 4 blocks of 64 keys
    assert _mla(lib) == 7                              # no workspace
    need = 1 * 8 * 1 * (512 + 1) * 4
    assert _mla(lib, ws=0x4004, ws_bytes=4 * need) == 3  # not 256-aligned


def _wide(lib, q=0x1000, k=0x1000, v=0x1000, o=0x2000, B=1, Hq=32, Hkv=1,
          Lkv=256, d=128, lnl=-1.0, Bc=64, S=1, ws=None, ws_bytes=0):
    f = lib.blasst_decode_wide
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [
        ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    return f(q, k, v, o, None, B, Hq, Hkv, Lkv, d, 0.088, lnl, Bc, S, ws,
             ws_bytes, None, None)


def test_decode_wide_validation(lib):
    """Argument checks of blasst_decode_wide, all taken before any launch."""
    assert _wide(lib, v=None) == 1
    assert _wide(lib, Hq=12, Hkv=5) == 1               # Hq % Hkv
    assert _wide(lib, lnl=float("nan")) == 1
    assert _wide(lib, Hq=256) == 2                     # group above 128 heads
    assert _wide(lib, d=64) == 2
    assert _wide(lib, Bc=128) == 2
    assert _wide(lib, q=0x1002) == 3
    assert _wide(lib, S=5) == 1                        # 4 blocks of 64 keys
    assert _wide(lib) == 7                             # no workspace


def _bwd(lib, ptr=0x1000, dq=0x2000, B=1, Hq=4, Hkv=1, Lq=256, Lkv=256, d=128,
         causal=1, Br=128, Bc=128, ws=None, ws_bytes=0):
    f = lib.blasst_prefill_backward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 10 + [ctypes.c_int] * 6 + [
        ctypes.c_float] + [ctypes.c_int] * 3 + [
        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    return f(ptr, ptr, ptr, ptr, ptr, ptr, None, dq, ptr, ptr, B, Hq, Hkv, Lq,
             Lkv, d, 0.088, causal, Br, Bc, ws, ws_bytes, None)


def test_prefill_backward_validation(lib):
    """Argument checks of blasst_prefill_backward, before any launch."""
    m_ws = lib.blasst_prefill_backward_workspace_size
    m_ws.restype = ctypes.c_size_t
    m_ws.argtypes = [ctypes.c_int] * 4
    need = m_ws(1, 4, 256, 128)
    assert need >= 4 * 256 * 128 * 4 and need % 256 == 0
    assert _bwd(lib, dq=None) == 1
    assert _bwd(lib, Hq=3, Hkv=2) == 1                 # Hq % Hkv
    assert _bwd(lib, Lq=512) == 1                      # causal, Lq > Lkv
    assert _bwd(lib, d=64) == 2                        # d 128 only
    assert _bwd(lib, Br=64, Bc=64) == 2                # 128 x 128 only
    assert _bwd(lib, dq=0x2004) == 3
    assert _bwd(lib) == 7                              # no workspace
    assert _bwd(lib, ws=0x4000, ws_bytes=need - 256) == 7
    assert _bwd(lib, ws=0x4010, ws_bytes=need) == 3    # not 256-aligned


def test_binding_rejects_host_and_mistyped_tensors(lib):
    """The binding passes raw device pointers, so it refuses before the call
    what the C ABI cannot see: host tensors, wrong dtypes, non-tensors."""
    import torch
    import dynamic_block_sparse_fa_b200 as m
    from dynamic_block_sparse_fa_b200 import blasst as b
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        m.blasst_prefill(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        m.blasst_decode(q[:, :, 0].contiguous(), q, q)
    with pytest.raises(TypeError, match="Tensor"):
        b._arg([1, 2], "x")
    assert b._arg(None, "x") is None
    with pytest.raises(ValueError, match="CUDA"):
        b._arg(torch.zeros(4, dtype=torch.float16), "x")


def test_backward_binding_rejects_dq_overlapping_an_input(lib):
    """dq holds the masked backward's work order before it is written, so
    the binding refuses a dq that shares storage with an input (checked on
    the host, before any pointer reaches the library)."""
    import torch
    import dynamic_block_sparse_fa_b200 as m
    from dynamic_block_sparse_fa_b200 import blasst as b
    q = torch.zeros(1, 2, 128, 128, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 128)
    dout = torch.zeros_like(q)
    with pytest.raises(ValueError, match="dq overlaps dout"):
        m.blasst_prefill_backward(q, k, k, q.clone(), lse, dout, dq=dout[:, 1:])
    with pytest.raises(ValueError, match="dq overlaps q"):
        m.blasst_prefill_backward(q, k, k, q.clone(), lse, dout, dq=q)
    flat = torch.zeros(100)
    assert b._overlaps(flat[10:20], flat[19:30])
    assert not b._overlaps(flat[10:20], flat[20:30])
    assert not b._overlaps(flat, None)


def test_split_policy_and_workspace(lib):
    import dynamic_block_sparse_fa_b200 as m
    # batch 32 x 8 KV heads at 32K: 5 splits; batch 148: 1 split
    assert m.blasst_decode_splits(32, 8, 32768, 64) == 5
    assert m.blasst_decode_splits(148, 8, 32768, 64) == 1
    assert m.blasst_decode_splits(1, 1, 64, 64) == 1
    for B, Hkv, L in [(1, 1, 10 ** 6), (7, 3, 1000), (2, 8, 640)]:
        s = m.blasst_decode_splits(B, Hkv, L, 64)
        nk = -(-L // 64)
        assert 1 <= s <= max(1, nk // 8)
    ws = m.blasst_decode_workspace_size(32, 32, 128, 5)
    rows = 32 * 32 * 5
    assert ws >= rows * 129 * 4 + 32 * 4 and ws % 256 == 0
    # partials, lse and the paged work order, each region 256-byte aligned
    assert m.blasst_decode_workspace_size(1, 1, 128, 1) == 512 + 256 + 256


def _wide_policy(B, Hkv, L, Bc=64):
    """The wide-group split policy as include/blasst.h states it: among
    the counts with at least 8 blocks per split, the one minimising
    ceil(B*Hkv*S / 296) * (nk/S + 2), fewest splits on ties."""
    nk = -(-L // Bc)
    best, best_t = 1, None
    for s in range(1, max(1, nk // 8) + 1):
        t = math.ceil(B * Hkv * s / 296) * (nk / s + 2.0)
        if best_t is None or t < best_t - 1e-9:
            best, best_t = s, t
    return best


def test_wide_and_group_split_policies(lib):
    import dynamic_block_sparse_fa_b200 as m
    # MQA batch 32 at 32K: one wave of 288 of the 296 slots
    assert m.blasst_decode_wide_splits(32, 1, 32768, 64) == 9
    assert m.blasst_decode_wide_splits(148, 1, 32768, 64) == 2
    for B in (1, 3, 16, 32, 100, 148, 512):
        for Hkv in (1, 2, 8):
            for L in (64, 500, 4096, 32768, 131072):
                assert (m.blasst_decode_wide_splits(B, Hkv, L, 64)
                        == _wide_policy(B, Hkv, L)), (B, Hkv, L)
    # blasst_decode's choice follows the kernel the group runs on
    for B, Hq, Hkv, L in [(32, 32, 8, 32768), (4, 8, 8, 1000),
                          (2, 256, 1, 4096), (32, 32, 1, 32768),
                          (8, 128, 1, 8192), (8, 64, 4, 5000)]:
        G = Hq // Hkv
        want = (m.blasst_decode_wide_splits(B, Hkv, L, 64) if 8 < G <= 128
                else m.blasst_decode_splits(B, Hkv, L, 64))
        assert m.blasst_decode_group_splits(B, Hq, Hkv, L, 64) == want
    assert m.blasst_decode_group_splits(1, 3, 2, 100, 64) == 1  # Hq % Hkv
    assert m.blasst_decode_group_splits(0, 8, 8, 100, 64) == 1


def test_mla_split_policy(lib):
    """One CTA pair per (sequence, split), one CTA per SM: the count with the
    fewest SM waves per split, at most two waves, 8 blocks per split or
    more, the smaller on a tie."""
    import math
    import dynamic_block_sparse_fa_b200 as m
    assert m.blasst_mla_decode_splits(32, 32768) == 2    # 128 CTAs, one wave
    assert m.blasst_mla_decode_splits(74, 32768) == 1    # 148 CTAs, one wave
    assert m.blasst_mla_decode_splits(200, 32768) == 1   # above two waves
    assert m.blasst_mla_decode_splits(1, 32768) == 64    # capped at nk / 8
    assert m.blasst_mla_decode_splits(1, 640) == 1       # 10 blocks
    for B, L in [(1, 10 ** 6), (3, 4096), (16, 65536), (37, 9000)]:
        s = m.blasst_mla_decode_splits(B, L)
        nk = -(-L // 64)
        assert 1 <= s <= max(1, nk // 8)
        best = min(math.ceil(2 * B * t / 148) / t
                   for t in range(1, max(1, nk // 8) + 1) if 2 * B * t <= 296)
        assert math.ceil(2 * B * s / 148) / s == pytest.approx(best)


def test_fit_a_and_strings(lib):
    import dynamic_block_sparse_fa_b200 as m
    assert m.blasst_fit_a([50 / 4096, 50 / 65536], [4096, 65536]) == \
        pytest.approx(50.0)
    assert m.blasst_fit_a([1e-3, 4e-3], [1000, 1000]) == pytest.approx(2.0)
    assert m.blasst_strerror(0) == "ok"
    assert "aligned" in m.blasst_strerror(3)
    assert m.blasst_version().count(".") == 2


def test_calibrate_validation(lib):
    import dynamic_block_sparse_fa_b200.blasst as b
    smp = b.CalibSample(0, 0x1000, 0x1000, 0x1000, 1, 2, 2, 128, 128, 128,
                        0.088, 1, 128, 128, 0)
    res = b.CalibResult()
    f = b._lib.blasst_calibrate
    assert f(1.5, ctypes.byref(smp), 0.01, ctypes.c_void_p(0x3000),
             ctypes.byref(res), None) == 1
    assert f(0.5, ctypes.byref(smp), 0.01, None, ctypes.byref(res), None) == 1
    smp.mode = 7
    assert f(0.5, ctypes.byref(smp), 0.01, ctypes.c_void_p(0x3000),
             ctypes.byref(res), None) == 1


def test_reference_arm_split_policy_matches_library(lib):
    """bench.py's reference arm restates the automatic split count so that it
    loads no GPU code; both must agree or the arms would run different
    masks."""
    import itertools
    import bench
    import dynamic_block_sparse_fa_b200 as m
    for B, H, L in itertools.product([1, 2, 3, 8, 32, 148], [1, 8],
                                     [64, 1000, 32768, 131072]):
        assert bench.auto_splits(B, H, L, 64) == m.blasst_decode_splits(B, H, L, 64)


def _paged(lib, q=0x1000, kp=0x1000, vp=0x1000, stride=None, P=8, ps=64,
           bt=0x3000, maxp=4, sl=0x4000, maxlen=256, o=0x2000, B=2, Hq=8,
           Hkv=2, d=128, scale=0.088, lnl=-1.0, per_length=0, S=1):
    f = lib.blasst_decode_paged
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_longlong, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_void_p] + [ctypes.c_int] * 4 + [
        ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    if stride is None:
        stride = Hkv * ps * d
    # a workspace of 0 bytes: every shape that passes validation stops at
    # BLASST_ERR_WORKSPACE (7) before any CUDA call
    return f(q, kp, vp, stride, P, ps, bt, maxp, sl, maxlen, o, None, B, Hq,
             Hkv, d, scale, lnl, per_length, S, None, 0, None, None)


def test_paged_decode_validation(lib):
    assert _paged(lib) == 7                            # valid up to workspace
    assert _paged(lib, bt=None) == 1
    assert _paged(lib, sl=None) == 1
    assert _paged(lib, ps=48) == 2                     # page size not built
    assert _paged(lib, ps=8) == 2
    for ps in (16, 32, 64, 128, 256):
        assert _paged(lib, ps=ps, maxp=max(1, 256 // ps)) == 7
    assert _paged(lib, maxlen=257) == 1                # beyond the table
    assert _paged(lib, stride=2 * 64 * 128 - 8) == 1   # pages overlap
    assert _paged(lib, stride=2 * 64 * 128 + 4) == 1   # not 16-byte multiple
    assert _paged(lib, stride=2 * 2 * 64 * 128) == 7   # interleaved K/V pool
    assert _paged(lib, lnl=0.5) == 1                   # ln lambda > 0 ...
    assert _paged(lib, lnl=3.5, per_length=1) == 7     # ... but ln a may be
    assert _paged(lib, lnl=float("nan"), per_length=1) == 1
    assert _paged(lib, lnl=float("inf"), per_length=1) == 1
    assert _paged(lib, lnl=-math.inf, per_length=1) == 7
    assert _paged(lib, S=5) == 1                       # more splits than blocks
    assert _paged(lib, Hq=24, Hkv=2) == 2              # G = 12 not built
    assert _paged(lib, d=64) == 7                      # d 64 with G <= 8 ...
    assert _paged(lib, d=64, Hq=32, Hkv=2) == 2        # ... not with G = 16
    assert _paged(lib, d=96) == 2
    assert _paged(lib, kp=0x1008) == 3                 # misaligned pool
    assert _paged(lib, P=0) == 1
