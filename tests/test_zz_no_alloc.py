"""blasst_decode_noalloc: the decode entry point for callers that may not
allocate device memory when they run the decode (for example an
inference-engine plugin whose enqueue step must not allocate, or a
latency-critical decode loop that cannot take cudaMalloc's device-wide
synchronisation) and so cannot pass a workspace.  Its split partials live in
the library's own fixed device array.

The test calls it through the C ABI twice in a row, on two different inputs,
and compares each result with blasst_decode given a caller workspace, within
the tolerance of the other decode parity tests.  It also checks that shapes
too large for the fixed array are refused before any launch.  This file is
named so that pytest collects it last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from synth import config_seed, planted_gap
from tests import _parity as P

pytestmark = pytest.mark.gpu


def _c_noalloc(b, q, k, v, o, lse, ln_lambda, S, stats=None):
    B, Hq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    return b._lib.blasst_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, Lkv, d,
        1.0 / math.sqrt(d), ln_lambda, 64, S,
        stats.c_struct if stats is not None else None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_decode_noalloc_matches_decode_twice():
    import dynamic_block_sparse_fa_b200 as m
    from dynamic_block_sparse_fa_b200 import blasst as b

    cases = [  # (B, Hq, Hkv, Lkv, ln_lambda, splits)
        (4, 32, 8, 8192, -4.0, 0),
        (2, 16, 8, 3000, -2.0, 3),
    ]
    for i, (B, Hq, Hkv, Lkv, lnl, S) in enumerate(cases):
        x = planted_gap(B, Hq, Hkv, 1, Lkv, 128, decode=True, block=64,
                        gap=8.0, heavy_frac=0.03,
                        seed=config_seed(1, 7000 + i), device="cuda")
        o_ref, lse_ref = m.blasst_decode(x.q, x.k, x.v, ln_lambda=lnl,
                                         num_splits=S)
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        st = m.Stats()
        rc = _c_noalloc(b, x.q, x.k, x.v, o, lse, lnl, S, st)
        assert rc == 0, m.blasst_last_error()
        torch.cuda.synchronize()
        P.check_out(P.to_np(o), P.to_np(o_ref), f"noalloc call {i}")
        P.check_lse(P.to_np(lse), P.to_np(lse_ref), f"noalloc call {i}")
        vis, skp = st.read()
        assert vis == B * Hkv * (-(-Lkv // 64)) and skp > 0


def test_decode_noalloc_rejects_oversized_partials():
    import dynamic_block_sparse_fa_b200 as m
    from dynamic_block_sparse_fa_b200 import blasst as b

    # 64 sequences x 64 heads x 8 splits x 129 floats > 8 MiB of partials
    B, Hq, Hkv, Lkv = 64, 64, 8, 4096
    q = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    rc = b._lib.blasst_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(o.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, Lkv, 128, 0.088, -1.0,
        64, 8, None, None)
    assert rc == 7
    assert "scratch holds" in m.blasst_last_error()
