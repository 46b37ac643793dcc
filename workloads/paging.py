"""Paged-cache layout for the seeded inputs: logical caches scattered into a shuffled
page pool, as a paged-attention serving engine holds them.

Pure data movement (no arithmetic of the method).  A pool holds the pages every
sequence needs plus `spare` unused pages filled with a large constant, so that a
kernel reading a page it was not given shows up in the results.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass
class PagedCache:
    page_size: int
    block_table: torch.Tensor   # [B, max_blocks] int32, -1 past a sequence's last page
    seq_lens: torch.Tensor      # [B] int32
    num_pages: int


def make_block_table(seq_lens, Lmax: int, page_size: int, seed: int, spare: int = 3):
    """A seeded random assignment of distinct pool pages to every sequence's blocks."""
    B = len(seq_lens)
    max_blocks = max(1, -(-Lmax // page_size))
    need = [-(-int(L) // page_size) for L in seq_lens]
    num_pages = sum(need) + spare
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    at = 0
    for b, nb in enumerate(need):
        table[b, :nb] = perm[at:at + nb]
        at += nb
    return PagedCache(page_size, table, torch.tensor([int(x) for x in seq_lens], dtype=torch.int32),
                      num_pages)


def scatter_to_pages(x: torch.Tensor, pc: PagedCache, fill=0) -> torch.Tensor:
    """x [B, Hkv, Lmax, ...] -> pool [num_pages, Hkv, page_size, ...] holding the first
    seq_lens[b] positions of each sequence at its block-table pages; every other
    slot holds `fill`."""
    B, Hkv, Lmax = x.shape[:3]
    ps = pc.page_size
    pool = torch.full((pc.num_pages, Hkv, ps) + tuple(x.shape[3:]), fill, dtype=x.dtype,
                      device=x.device)
    if Lmax % ps == 0 and all(int(L) == Lmax for L in pc.seq_lens):
        # every sequence full: one indexed copy of all blocks
        nb = Lmax // ps
        rest = tuple(x.shape[3:])
        blocks = x.reshape((B, Hkv, nb, ps) + rest).transpose(1, 2).reshape((B * nb, Hkv, ps) + rest)
        pool[pc.block_table[:, :nb].reshape(-1).long().to(x.device)] = blocks
        return pool
    for b in range(B):
        L = int(pc.seq_lens[b])
        for blk in range(-(-L // ps)):
            page = int(pc.block_table[b, blk])
            lo, hi = blk * ps, min(L, (blk + 1) * ps)
            pool[page, :, :hi - lo] = x[b, :, lo:hi]
    return pool
