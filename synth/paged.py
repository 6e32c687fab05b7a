"""Seeded page-pool layout of a KV cache (input synthesis only).

Serving engines keep the decode KV cache in a pool of fixed-size pages and
give each sequence a block table of page ids; a sequence's pages are
scattered over the pool in whatever order they were allocated.  This module
turns logical per-sequence caches into such a pool so that the tests and the
benchmark can feed the paged decode the same tokens as the contiguous one.
It holds none of the attention method's arithmetic.

Pool layout: [num_pages, Hkv, page_size, d] -- inside a page, one KV head's
tokens are contiguous rows of d elements.  Physical page ids are a seeded
random permutation; ``spare_pages`` extra pages belong to no sequence.
Table entries past a sequence's last page are -1.  ``poison`` fills every
pool row that no sequence owns (spare pages and the rows past the end of a
sequence's last page), so that a kernel reading out of bounds of a sequence
changes its result visibly.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass
class PagedKV:
    k_pages: torch.Tensor      # [P, Hkv, page_size, d] bf16
    v_pages: torch.Tensor      # [P, Hkv, page_size, d] bf16
    block_table: torch.Tensor  # [B, max_pages] int32, -1 past a sequence
    seq_lens: torch.Tensor     # [B] int32
    page_size: int
    num_pages: int


def paginate(k: torch.Tensor, v: torch.Tensor, seq_lens, page_size: int, *,
             seed: int, spare_pages: int = 0, poison=(0.0, 0.0),
             max_pages: int | None = None) -> PagedKV:
    """Scatter logical caches k, v [B, Hkv, Lmax, d] into a page pool.

    Rows of sequence b at or past seq_lens[b] are not copied (their pool
    rows hold ``poison``).  Everything is built on k's device.
    """
    B, Hkv, Lmax, d = k.shape
    dev = k.device
    lens = [int(x) for x in (seq_lens.tolist() if torch.is_tensor(seq_lens)
                             else seq_lens)]
    assert len(lens) == B and all(0 <= L <= Lmax for L in lens)
    ps = int(page_size)
    npg = [-(-L // ps) for L in lens]
    mp = max(npg + [1]) if max_pages is None else int(max_pages)
    assert mp >= max(npg + [0])
    total = sum(npg) + int(spare_pages)
    g = torch.Generator().manual_seed(int(seed) & ((1 << 63) - 1))
    perm = torch.randperm(max(total, 1), generator=g)[:total]

    pk, pv = float(poison[0]), float(poison[1])
    k_pages = torch.full((max(total, 1), Hkv, ps, d), pk, dtype=k.dtype,
                         device=dev)
    v_pages = torch.full((max(total, 1), Hkv, ps, d), pv, dtype=v.dtype,
                         device=dev)
    table = torch.full((B, mp), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        L, n = lens[b], npg[b]
        if n == 0:
            continue
        ids = perm[off:off + n]
        table[b, :n] = ids.to(torch.int32)
        off += n
        full = L // ps  # pages filled completely
        if full:
            src_k = k[b, :, :full * ps].reshape(Hkv, full, ps, d).transpose(0, 1)
            src_v = v[b, :, :full * ps].reshape(Hkv, full, ps, d).transpose(0, 1)
            idx = ids[:full].to(dev)
            k_pages[idx] = src_k
            v_pages[idx] = src_v
        rem = L - full * ps
        if rem:
            pid = int(ids[full])
            k_pages[pid, :, :rem] = k[b, :, full * ps:L]
            v_pages[pid, :, :rem] = v[b, :, full * ps:L]
    return PagedKV(k_pages, v_pages, table.to(dev),
                   torch.tensor(lens, dtype=torch.int32, device=dev), ps,
                   max(total, 1))
