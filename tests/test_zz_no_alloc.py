"""blasst_decode_noalloc: the decode entry point for callers that may not
allocate device memory when they run the decode (for example an
inference-engine plugin whose enqueue step must not allocate, or a
latency-critical decode loop that cannot take cudaMalloc's device-wide
synchronisation) and so cannot pass a workspace.  Its split partials live in
the library's own fixed device array.

The test calls it through the C ABI on three inputs one after the other
(and the first once more at the end, after the array holds another call's
partials), and checks each result against the CPU oracle and against
blasst_decode given a caller workspace, within the tolerance of the other
decode parity tests.  One input has 16 query heads per KV head, so the
tiled path (two CTAs of 8 heads per KV head) runs through the shared
array too.  Shapes too large for the array are refused before any launch:
the refusal is checked on buffers of the full declared size, so that even
a regression of that check would meet a second one (blasst_decode's own
workspace-size check) before any kernel could write past the array.  This
file is named so that pytest collects it last.
"""
import ctypes
import math

import pytest
import torch

import oracle
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


CASES = [  # (B, Hq, Hkv, Lkv, ln_lambda, splits)
    (4, 32, 8, 8192, -4.0, 0),
    (2, 16, 8, 3000, -2.0, 3),
    (2, 32, 2, 4096, -3.0, 0),    # 16 heads per KV head: tiles of 8
]


def _run_case(m, b, i):
    B, Hq, Hkv, Lkv, lnl, S = CASES[i]
    x = planted_gap(B, Hq, Hkv, 1, Lkv, 128, decode=True, block=64,
                    gap=8.0, heavy_frac=0.03,
                    seed=config_seed(1, 7000 + i), device="cuda")
    S_res = S if S else m.blasst_decode_group_splits(B, Hq, Hkv, Lkv, 64)
    o_ref, lse_ref = m.blasst_decode(x.q, x.k, x.v, ln_lambda=lnl,
                                     num_splits=S)
    o = torch.full_like(o_ref, float("nan"))
    lse = torch.full_like(lse_ref, float("nan"))
    st = m.Stats()
    rc = _c_noalloc(b, x.q, x.k, x.v, o, lse, lnl, S, st)
    assert rc == 0, m.blasst_last_error()
    torch.cuda.synchronize()
    assert m.blasst_check_device_error()[0] == 0
    G = Hq // Hkv
    tile = min(G, 8)
    orc = oracle.decode(x.q, x.k, x.v, 1 / math.sqrt(128), lnl, 64, S_res,
                        tile_heads=tile)
    P.check_out(P.to_np(o), orc["o"], f"noalloc call {i} vs oracle")
    P.check_lse(P.to_np(lse), orc["lse"], f"noalloc call {i} vs oracle")
    P.check_out(P.to_np(o), P.to_np(o_ref), f"noalloc call {i} vs decode")
    P.check_lse(P.to_np(lse), P.to_np(lse_ref), f"noalloc call {i} vs decode")
    vis, skp = st.read()
    nk = -(-Lkv // 64)
    assert vis == B * Hkv * (G // tile) * nk == orc["visited"]
    assert skp > 0
    near = int((abs(orc["margin"][orc["mask"] > 0]) < P.NEAR_TIE).sum())
    assert abs(skp - orc["skipped"]) <= near


def test_decode_noalloc_matches_oracle_and_decode():
    import dynamic_block_sparse_fa_b200 as m
    from dynamic_block_sparse_fa_b200 import blasst as b
    for i in range(len(CASES)):
        _run_case(m, b, i)
    _run_case(m, b, 0)  # the array now holds the previous call's partials


def test_decode_noalloc_rejects_oversized_partials():
    import dynamic_block_sparse_fa_b200 as m
    from dynamic_block_sparse_fa_b200 import blasst as b

    # 64 sequences x 64 heads x 8 splits x 129 floats = 16.9 MB > 8 MiB
    B, Hq, Hkv, Lkv, S = 64, 64, 8, 512, 8
    assert m.blasst_decode_workspace_size(B, Hq, 128, S) > 8 << 20
    q = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(B, Hkv, Lkv, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    rc = _c_noalloc(b, q, k, k, o, lse, -1.0, S)
    assert rc == 7
    assert "scratch holds" in m.blasst_last_error()
    torch.cuda.synchronize()
    assert m.blasst_check_device_error()[0] == 0
