"""GPU parity of the paged, variable-length decode against the CPU oracle,
called through the C ABI.

The logical caches are seeded planted-gap inputs; the test scatters them
into a page pool in a seeded random order and fills every pool row that no
sequence owns with poison (large K and V values), so that a read outside a
sequence's own rows changes its output visibly.  Checks: outputs within
max 2e-2 / mean 2e-3, lse, skip decisions bit-exact except near-ties,
counters, the statistics-only pass, page sizes 16..256, every GQA ratio,
empty and one-token sequences, splits with no blocks, the interleaved K/V
pool, the per-sequence threshold lambda = a / L_b, agreement bit for bit
with the contiguous kernel on the same tokens, out-of-range lengths and
page ids reported as invalid arguments, and the full-size decode workload
(batch 32, 32K cache) in a shuffled pool.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import config_seed, paginate, planted_gap, planted_gap_kv_inplace
from tests import _parity as P

pytestmark = pytest.mark.gpu

POISON = (6.0, 500.0)


@pytest.fixture(scope="module")
def blasst():
    import dynamic_block_sparse_fa_b200 as m
    return m


def _pool(pk, layout):
    """Separate K and V pools, or one interleaved pool [P, 2, Hkv, ps, d]."""
    if layout == "separate":
        return pk.k_pages, pk.v_pages
    both = torch.stack([pk.k_pages, pk.v_pages], dim=1).contiguous()
    return both[:, 0], both[:, 1]


def _check_paged(m, q, kp, vp, pk, lens, ln_lambda, S_req, per_length,
                 max_seq_len=None):
    B, Hq, d = q.shape
    Hkv = kp.shape[1]
    if max_seq_len is None:
        max_seq_len = pk.block_table.shape[1] * pk.page_size
    nk_max = -(-max_seq_len // 64)
    S = S_req if S_req > 0 else m.blasst_decode_splits(B, Hkv, max_seq_len, 64)
    scale = 1.0 / math.sqrt(d)
    stats = m.Stats(mask_numel=B * Hkv * nk_max)
    o, lse = m.blasst_decode_paged(q, kp, vp, pk.block_table, pk.seq_lens,
                                   max_seq_len=max_seq_len, scale=scale,
                                   ln_lambda=ln_lambda, per_length=per_length,
                                   num_splits=S_req, stats=stats)
    torch.cuda.synchronize()
    st, where = m.blasst_check_device_error()
    assert st == 0, f"device error word set ({where})"
    ref = oracle.decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                              pk.seq_lens, scale, ln_lambda, S,
                              per_length=per_length, nk_max=nk_max)
    og, lg = P.to_np(o), P.to_np(lse)
    live = [b for b in range(B) if lens[b] > 0]
    for b in range(B):
        if lens[b] == 0:
            assert np.all(og[b] == 0.0) and np.all(np.isneginf(lg[b]))
    P.check_out(og[live], ref["o"][live], "paged o")
    P.check_lse(lg[live], ref["lse"][live], "paged lse")
    mask = stats.mask.cpu().numpy().reshape(B, Hkv, nk_max)
    ties = P.check_mask(mask, ref["mask"], ref["margin"], "paged mask")
    vis, skp = stats.read()
    assert vis == Hkv * sum(-(-L // 64) for L in lens)
    assert skp == int((mask == 2).sum())
    if ties == 0:
        assert (vis, skp) == (ref["visited"], ref["skipped"])
    st2 = m.Stats(mask_numel=B * Hkv * nk_max)
    r2 = m.blasst_decode_paged(q, kp, vp, pk.block_table, pk.seq_lens,
                               max_seq_len=max_seq_len, scale=scale,
                               ln_lambda=ln_lambda, per_length=per_length,
                               num_splits=S_req, stats=st2, stats_only=True)
    assert r2 == (None, None)
    assert torch.equal(st2.mask, stats.mask)
    assert st2.read() == (vis, skp)
    return o, lse, mask


PAGED_CASES = [
    # Hq, Hkv, lens, page_size, ln_lambda, splits, per_length, layout
    (32, 8, [1000, 64, 65, 4096], 16, -3.0, 0, False, "separate"),
    (8, 2, [777, 2048, 1], 32, -2.0, 3, False, "separate"),
    (16, 8, [3000, 1500], 64, -4.0, 4, False, "interleaved"),
    (64, 8, [2048, 0, 300], 128, -3.0, 2, False, "separate"),
    (4, 1, [5000, 130], 256, math.log(60.0), 5, True, "separate"),
    (8, 8, [63, 64, 129, 1000], 64, -math.inf, 2, False, "separate"),
    (32, 8, [4096, 4096], 64, 0.0, 7, False, "interleaved"),
    (32, 8, [2500, 40, 7000, 64, 3333], 16, math.log(20.0), 0, True,
     "interleaved"),
]


@pytest.mark.parametrize("case", PAGED_CASES)
def test_paged_decode_matches_oracle(blasst, case):
    Hq, Hkv, lens, ps, ln_lambda, S, per_length, layout = case
    B = len(lens)
    Lmax = max(max(lens), 1)
    x = planted_gap(B, Hq, Hkv, 1, Lmax, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.03, seed=config_seed(1, 7 * Lmax + Hq + ps),
                    device="cuda")
    pk = paginate(x.k, x.v, lens, ps, seed=Lmax + ps, spare_pages=7,
                  poison=POISON)
    kp, vp = _pool(pk, layout)
    o, lse, mask = _check_paged(blasst, x.q, kp, vp, pk, lens, ln_lambda, S,
                                per_length)
    if ln_lambda == -math.inf:
        assert (mask == 2).sum() == 0


PAGED_D64_CASES = [
    # head dimension 64 (the warp-MMA kernel, up to 8 heads per KV head)
    (8, 2, [1000, 64, 65, 3000], 16, -3.0, 0, False, "separate"),
    (4, 4, [2048, 129], 64, -2.0, 3, False, "interleaved"),
    (8, 1, [700, 5000], 32, math.log(40.0), 2, True, "separate"),
]


@pytest.mark.parametrize("case", PAGED_D64_CASES)
def test_paged_decode_d64_matches_oracle(blasst, case):
    Hq, Hkv, lens, ps, ln_lambda, S, per_length, layout = case
    B = len(lens)
    Lmax = max(lens)
    x = planted_gap(B, Hq, Hkv, 1, Lmax, 64, decode=True, block=64, gap=8.0,
                    heavy_frac=0.03, seed=config_seed(1, 3 * Lmax + Hq + ps),
                    device="cuda")
    pk = paginate(x.k, x.v, lens, ps, seed=Lmax + ps + 1, spare_pages=5,
                  poison=POISON)
    kp, vp = _pool(pk, layout)
    _check_paged(blasst, x.q, kp, vp, pk, lens, ln_lambda, S, per_length)


def test_paged_d64_equals_contiguous_bitwise(blasst):
    """Head dimension 64, same tokens, same splits: the paged and the
    contiguous warp-MMA kernels give the same bits; 16 query heads per KV
    head at d 64 (the CUDA-core kernel, d 128 only) is refused."""
    m = blasst
    B, Hq, Hkv, L = 3, 16, 4, 2000
    x = planted_gap(B, Hq, Hkv, 1, L, 64, decode=True, block=64, gap=8.0,
                    heavy_frac=0.03, seed=config_seed(1, 98), device="cuda")
    pk = paginate(x.k, x.v, [L] * B, 16, seed=4, spare_pages=2,
                  poison=POISON)
    for lnl in (-math.inf, -3.0):
        o1, l1 = m.blasst_decode(x.q, x.k, x.v, ln_lambda=lnl, num_splits=3)
        o2, l2 = m.blasst_decode_paged(x.q, pk.k_pages, pk.v_pages,
                                       pk.block_table, pk.seq_lens,
                                       max_seq_len=L, ln_lambda=lnl,
                                       num_splits=3)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
    q16 = torch.zeros(1, 16, 64, dtype=torch.bfloat16, device="cuda")
    kp = torch.zeros(4, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    sl = torch.tensor([100], dtype=torch.int32, device="cuda")
    with pytest.raises(m.BlasstError, match="UNSUPPORTED"):
        m.blasst_decode_paged(q16, kp, kp, bt, sl)


@pytest.mark.parametrize("ps", [16, 64])
def test_paged_nan_rows_past_the_sequence_never_reach_the_output(blasst, ps):
    """Pool rows no sequence owns hold NaN: the kernel may bring the rest of
    a sequence's last page (or stale rows) into shared memory, but masks
    those keys and zeroes those V rows, so the outputs stay finite and
    match the oracle (which reads only the sequences' own rows)."""
    lens = [1000, 65, 1, 2047]
    B = len(lens)
    x = planted_gap(B, 8, 2, 1, max(lens), 128, decode=True, block=64,
                    gap=8.0, heavy_frac=0.05, seed=config_seed(1, 4242 + ps),
                    device="cuda")
    nan = float("nan")
    pk = paginate(x.k, x.v, lens, ps, seed=ps, spare_pages=3,
                  poison=(nan, nan))
    o, lse, _ = _check_paged(blasst, x.q, pk.k_pages, pk.v_pages, pk, lens,
                             -2.0, 0, False)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("ps", [16, 64, 256])
def test_paged_equals_contiguous_bitwise(blasst, ps):
    """Same tokens, same splits: the paged kernel reads the same bytes in the
    same order as the contiguous one (both the warp-MMA kernel), so the
    results agree bit for bit; the CUDA-core kernel (blasst_decode_batched
    with batch 1, same decisions) agrees within the parity tolerance."""
    m = blasst
    B, Hq, Hkv, L = 6, 32, 8, 4096 + 64 * 3
    x = planted_gap(B, Hq, Hkv, 1, L, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.03, seed=config_seed(1, 99), device="cuda")
    pk = paginate(x.k, x.v, [L] * B, ps, seed=3, spare_pages=2,
                  poison=POISON)
    for lnl in (-math.inf, -3.0):
        o1, l1 = m.blasst_decode(x.q, x.k, x.v, ln_lambda=lnl, num_splits=3)
        o2, l2 = m.blasst_decode_paged(x.q, pk.k_pages, pk.v_pages,
                                       pk.block_table, pk.seq_lens,
                                       max_seq_len=L, ln_lambda=lnl,
                                       num_splits=3)
        o3, l3 = m.blasst_decode_batched(x.q, x.k, x.v, batch=1,
                                         ln_lambda=lnl, num_splits=3)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        P.check_out(P.to_np(o3), P.to_np(o2), "CUDA-core vs paged")
        P.check_lse(P.to_np(l3), P.to_np(l2), "CUDA-core vs paged")


def test_paged_bad_table_and_length_are_reported(blasst):
    """Out-of-range values in the device-resident table and lengths are
    caught by the kernel before any copy through them is issued.  The pool
    passed to the call is a view into a larger allocation with 8 poisoned
    guard pages on each side, so that the bad page ids used here (-1 and
    num_pages + 5) would still address allocated memory if the check ever
    failed to stop a copy."""
    m = blasst
    B, Hq, Hkv, L = 2, 8, 2, 1000
    x = planted_gap(B, Hq, Hkv, 1, L, 128, decode=True, block=64, gap=8.0,
                    heavy_frac=0.03, seed=5, device="cuda")
    pk = paginate(x.k, x.v, [L, L], 64, seed=1, poison=POISON)
    GUARD = 8
    P_ = pk.num_pages
    kg = torch.full((P_ + 2 * GUARD,) + tuple(pk.k_pages.shape[1:]),
                    POISON[0], dtype=torch.bfloat16, device="cuda")
    vg = torch.full_like(kg, POISON[1])
    kg[GUARD:GUARD + P_] = pk.k_pages
    vg[GUARD:GUARD + P_] = pk.v_pages
    kp, vp = kg[GUARD:GUARD + P_], vg[GUARD:GUARD + P_]
    assert kp.shape[0] == P_ and kp.data_ptr() > kg.data_ptr()
    o_good, _ = m.blasst_decode_paged(x.q, kp, vp, pk.block_table,
                                      pk.seq_lens, ln_lambda=-2.0)
    assert m.blasst_check_device_error()[0] == 0
    bt = pk.block_table.clone()
    bt[1, 3] = P_ + 5
    assert P_ + 5 < P_ + GUARD
    m.blasst_decode_paged(x.q, kp, vp, bt, pk.seq_lens, ln_lambda=-2.0)
    st, where = m.blasst_check_device_error()
    assert st == 1 and "page id" in where and "sequence 1" in where
    bt[1, 3] = -1
    m.blasst_decode_paged(x.q, kp, vp, bt, pk.seq_lens, ln_lambda=-2.0)
    st, where = m.blasst_check_device_error()
    assert st == 1 and "page id" in where
    # a length past what the table holds: the table is a view of a larger
    # one (an extra row of -1), so an entry read past its end stays inside
    # the allocation
    tb = torch.full((B + 1, pk.block_table.shape[1]), -1, dtype=torch.int32,
                    device="cuda")
    tb[:B] = pk.block_table
    lens = torch.tensor([L, 16 * 64 + 1], dtype=torch.int32, device="cuda")
    assert pk.block_table.shape[1] * 64 == 16 * 64
    m.blasst_decode_paged(x.q, kp, vp, tb[:B], lens, ln_lambda=-2.0)
    st, where = m.blasst_check_device_error()
    assert st == 1 and "length" in where
    # the context is still usable and a good call is clean afterwards
    o2, _ = m.blasst_decode_paged(x.q, kp, vp, pk.block_table, pk.seq_lens,
                                  ln_lambda=-2.0)
    assert m.blasst_check_device_error()[0] == 0
    assert torch.equal(o2, o_good)


def test_paged_rejects_bad_arguments(blasst):
    m = blasst
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    kp = torch.zeros(4, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    sl = torch.tensor([100], dtype=torch.int32, device="cuda")
    with pytest.raises(blasst.BlasstError, match="INVALID_ARG"):
        m.blasst_decode_paged(q, kp, kp, bt, sl, ln_lambda=0.5)
    with pytest.raises(blasst.BlasstError, match="INVALID_ARG"):
        m.blasst_decode_paged(q, kp, kp, bt, sl, max_seq_len=257)
    kp48 = torch.zeros(4, 1, 48, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(blasst.BlasstError, match="UNSUPPORTED"):
        m.blasst_decode_paged(q, kp48, kp48, bt, sl)
    with pytest.raises(ValueError):
        m.blasst_decode_paged(q, kp, kp, bt.long(), sl)


def test_paged_full_size_shuffled_pool(blasst):
    """Batch 32, Hq 32 / Hkv 8, 32K cache, d 128 in a shuffled pool of
    64-token pages, lambda calibrated to 70% sparsity on the contiguous
    cache: decisions and outputs equal the contiguous kernel's bit for bit,
    and 3 sampled sequences match the oracle."""
    m = blasst
    B, Hq, Hkv, L, d = 32, 32, 8, 32768, 128
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(1))
    cal = m.blasst_calibrate(0.70, mode="decode", q=q, k=k, v=v, Bc=64)
    lnl = cal["ln_lambda"]
    nk = L // 64
    pk = paginate(k, v, [L] * B, 64, seed=11, spare_pages=64)
    s1 = m.Stats(mask_numel=B * Hkv * nk)
    s2 = m.Stats(mask_numel=B * Hkv * nk)
    o1, l1 = m.blasst_decode(q, k, v, ln_lambda=lnl, stats=s1)
    o2, l2 = m.blasst_decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                                   pk.seq_lens, max_seq_len=L, ln_lambda=lnl,
                                   stats=s2)
    torch.cuda.synchronize()
    assert m.blasst_check_device_error()[0] == 0
    assert torch.equal(s1.mask, s2.mask) and s1.read() == s2.read()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    del k, v
    S = m.blasst_decode_splits(B, Hkv, L, 64)
    mask = s2.mask.cpu().numpy().reshape(B, Hkv, nk)
    for b in (0, 17, 31):
        ids = pk.block_table[b].long()
        kb = pk.k_pages[ids].transpose(0, 1).reshape(1, Hkv, L, d)
        vb = pk.v_pages[ids].transpose(0, 1).reshape(1, Hkv, L, d)
        ref = oracle.decode(q[b:b + 1], kb, vb, 1 / math.sqrt(d), lnl, 64, S)
        P.check_out(P.to_np(o2[b:b + 1]), ref["o"], f"seq {b}")
        P.check_lse(P.to_np(l2[b:b + 1]), ref["lse"], f"seq {b}")
        P.check_mask(mask[b:b + 1], ref["mask"], ref["margin"], f"seq {b}")


def test_paged_varlen_per_length_sampled(blasst):
    """Batch 32 of lengths 1K..64K (mean about 32K) in a shuffled pool of
    16-token pages, per-sequence threshold lambda = a / L_b with a the value
    calibrated for 70% at 32K; 3 sampled sequences against the oracle."""
    m = blasst
    B, Hq, Hkv, d = 32, 32, 8, 128
    g = torch.Generator().manual_seed(config_seed(6))
    lens = torch.randint(1024, 65536 + 1, (B,), generator=g).tolist()
    lens[0], lens[1] = 65536, 1023
    Lmax = max(lens)
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, Lmax, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(6, 1))
    ln_a = math.log(math.exp(-8.0) * 32768)  # any a: parity is what counts
    pk = paginate(k, v, lens, 16, seed=12, spare_pages=100, poison=POISON)
    del k, v
    nk_max = -(-Lmax // 64)
    stats = m.Stats(mask_numel=B * Hkv * nk_max)
    o, lse = m.blasst_decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                                   pk.seq_lens, max_seq_len=Lmax,
                                   ln_lambda=ln_a, per_length=True,
                                   stats=stats)
    torch.cuda.synchronize()
    assert m.blasst_check_device_error()[0] == 0
    vis, skp = stats.read()
    assert vis == Hkv * sum(-(-L // 64) for L in lens)
    S = m.blasst_decode_splits(B, Hkv, Lmax, 64)
    mask = stats.mask.cpu().numpy().reshape(B, Hkv, nk_max)
    for b in (0, 1, 20):
        L = lens[b]
        npg = -(-L // 16)
        ids = pk.block_table[b, :npg].long()
        kb = pk.k_pages[ids].transpose(0, 1).reshape(Hkv, npg * 16, d)[:, :L]
        vb = pk.v_pages[ids].transpose(0, 1).reshape(Hkv, npg * 16, d)[:, :L]
        lnl = min(0.0, ln_a - math.log(L))
        ref = oracle.decode(q[b:b + 1], kb[None], vb[None], 1 / math.sqrt(d),
                            lnl, 64, S)
        P.check_out(P.to_np(o[b:b + 1]), ref["o"], f"seq {b}")
        P.check_lse(P.to_np(lse[b:b + 1]), ref["lse"], f"seq {b}")
        nk = -(-L // 64)
        P.check_mask(mask[b:b + 1, :, :nk], ref["mask"], ref["margin"],
                     f"seq {b}")
        assert np.all(mask[b, :, nk:] == 0)


def test_paged_varlen_work_order_is_invisible(blasst):
    """Batch 32 of lengths 1K..64K (one tie) in 16-token pages, 5 splits:
    1280 work items, more than the GPU holds at once, so the call sorts the
    sequences by length and decodes the longest first.  Every sequence's
    output, lse and decisions equal, bit for bit, a contiguous decode of that
    sequence alone (40 work items, natural order), and the counters add up;
    o and lse are poisoned with NaN first, so a sequence that no CTA decoded
    would show."""
    m = blasst
    B, Hq, Hkv, d, S, lnl = 32, 32, 8, 128, 5, -5.5
    g = torch.Generator().manual_seed(config_seed(6, 7))
    lens = torch.randint(1024, 65536 + 1, (B,), generator=g).tolist()
    lens[3] = lens[9]  # equal lengths: the index orders them
    Lmax = max(lens)
    assert B * Hkv * S > 148 * 3
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, Lmax, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(6, 8))
    pk = paginate(k, v, lens, 16, seed=14, spare_pages=8, poison=POISON)
    del k, v
    nk_max = -(-Lmax // 64)
    st = m.Stats(mask_numel=B * Hkv * nk_max)
    o = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16,
                   device="cuda")
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32,
                     device="cuda")
    m.blasst_decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                          pk.seq_lens, max_seq_len=Lmax, ln_lambda=lnl,
                          num_splits=S, o=o, lse=lse, stats=st)
    torch.cuda.synchronize()
    assert m.blasst_check_device_error()[0] == 0
    mask = st.mask.view(B, Hkv, nk_max)
    vis = skp = 0
    for b in range(B):
        L = lens[b]
        npg, nk = -(-L // 16), -(-L // 64)
        ids = pk.block_table[b, :npg].long()
        kb = pk.k_pages[ids].transpose(0, 1).reshape(Hkv, npg * 16, d)[:, :L]
        vb = pk.v_pages[ids].transpose(0, 1).reshape(Hkv, npg * 16, d)[:, :L]
        sb = m.Stats(mask_numel=Hkv * nk)
        ob, lb = m.blasst_decode(q[b:b + 1], kb[None].contiguous(),
                                 vb[None].contiguous(), ln_lambda=lnl,
                                 num_splits=S, stats=sb)
        torch.cuda.synchronize()
        assert torch.equal(ob, o[b:b + 1]) and torch.equal(lb, lse[b:b + 1]), b
        assert torch.equal(sb.mask.view(Hkv, nk), mask[b, :, :nk]), b
        assert not mask[b, :, nk:].any(), b
        v1, s1 = sb.read()
        vis, skp = vis + v1, skp + s1
    assert st.read() == (vis, skp)


def test_paged_varlen_work_order_cuda_core_kernel(blasst):
    """The same work order on the CUDA-core paged kernel (16 query heads per
    KV head, two tiles of 8): batch 32 of lengths 1K..16K, 5 splits, 640
    work items.  Every sequence equals, bit for bit, the contiguous CUDA-core
    kernel (blasst_decode_batched with batch 1) on that sequence alone."""
    m = blasst
    B, Hq, Hkv, d, S, lnl = 32, 32, 2, 128, 5, -4.0
    g = torch.Generator().manual_seed(config_seed(6, 9))
    lens = torch.randint(1024, 16384 + 1, (B,), generator=g).tolist()
    Lmax = max(lens)
    assert B * Hkv * 2 * S > 148 * 3
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, Lmax, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(6, 10))
    pk = paginate(k, v, lens, 16, seed=15, spare_pages=8, poison=POISON)
    del k, v
    o = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16,
                   device="cuda")
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32,
                     device="cuda")
    m.blasst_decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                          pk.seq_lens, max_seq_len=Lmax, ln_lambda=lnl,
                          num_splits=S, o=o, lse=lse)
    torch.cuda.synchronize()
    assert m.blasst_check_device_error()[0] == 0
    for b in range(B):
        L = lens[b]
        npg = -(-L // 16)
        ids = pk.block_table[b, :npg].long()
        kb = pk.k_pages[ids].transpose(0, 1).reshape(Hkv, npg * 16, d)[:, :L]
        vb = pk.v_pages[ids].transpose(0, 1).reshape(Hkv, npg * 16, d)[:, :L]
        ob, lb = m.blasst_decode_batched(q[b:b + 1], kb[None].contiguous(),
                                         vb[None].contiguous(), batch=1,
                                         ln_lambda=lnl, num_splits=S)
        torch.cuda.synchronize()
        assert torch.equal(ob, o[b:b + 1]) and torch.equal(lb, lse[b:b + 1]), b


def test_paged_work_order_many_sequences(blasst):
    """600 sequences of 64..4096 keys (ties included), 4 query heads on one
    KV head, one split: 600 work items, so the work order is computed by
    three blocks of the ordering kernel (ranks counted across 256-length
    tiles).  No output row is left unwritten (o and lse start as NaN, so a
    sequence missing from the permutation would show), and sampled
    sequences equal a contiguous decode of each alone bit for bit."""
    m = blasst
    B, Hq, Hkv, d, S, lnl = 600, 4, 1, 128, 1, -4.0
    g = torch.Generator().manual_seed(config_seed(6, 11))
    lens = torch.randint(64, 4096 + 1, (B,), generator=g).tolist()
    for i in range(0, B, 50):  # runs of equal lengths
        lens[i + 1] = lens[i]
    Lmax = max(lens)
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, Hkv, Lmax, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    planted_gap_kv_inplace(k, v, q, block=64, gap=8.0, heavy_frac=0.03,
                           seed=config_seed(6, 12))
    pk = paginate(k, v, lens, 16, seed=16, spare_pages=8, poison=POISON)
    del k, v
    o = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16,
                   device="cuda")
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32,
                     device="cuda")
    m.blasst_decode_paged(q, pk.k_pages, pk.v_pages, pk.block_table,
                          pk.seq_lens, max_seq_len=Lmax, ln_lambda=lnl,
                          num_splits=S, o=o, lse=lse)
    torch.cuda.synchronize()
    assert m.blasst_check_device_error()[0] == 0
    assert not torch.isnan(o.float()).any() and not torch.isnan(lse).any()
    order = sorted(range(B), key=lambda i: (-lens[i], i))
    picks = sorted({order[0], order[1], order[255], order[256], order[511],
                    order[512], order[-1], 0})
    for b in picks:
        L = lens[b]
        npg = -(-L // 16)
        ids = pk.block_table[b, :npg].long()
        kb = pk.k_pages[ids].transpose(0, 1).reshape(Hkv, npg * 16, d)[:, :L]
        vb = pk.v_pages[ids].transpose(0, 1).reshape(Hkv, npg * 16, d)[:, :L]
        ob, lb = m.blasst_decode(q[b:b + 1], kb[None].contiguous(),
                                 vb[None].contiguous(), ln_lambda=lnl,
                                 num_splits=S)
        torch.cuda.synchronize()
        assert torch.equal(ob, o[b:b + 1]) and torch.equal(lb, lse[b:b + 1]), b
