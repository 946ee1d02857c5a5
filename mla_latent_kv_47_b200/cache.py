"""Contiguous per-sequence latent cache on the device (allocation and bookkeeping).

Row layout per token: [c^KV (d_c) | k^R (d_R)] in the storage dtype, or the
E4M3 row of mla_cache_format (bytes); sequence s owns rows
[seq_start[s], seq_start[s] + capacity[s]).  Writes go through the
library (mla_cache_append / mla_decode / mla_prefill).
"""
from __future__ import annotations

import torch

from . import make_cache, MLA_FP32, CACHE_E4M3, cache_row_bytes

POISON_BF16 = 0x7FC1          # a quiet NaN; rows never written keep this pattern
POISON_FP32 = 0x7FC00001
POISON_BYTE = 0x7F            # E4M3 rows: a NaN code (and a NaN-free pattern elsewhere)


def _row_storage(dims):
    """(torch dtype, elements per row) of a cache row of these dims."""
    if dims.cache_format == CACHE_E4M3:
        return torch.uint8, cache_row_bytes(dims)
    return (torch.float32 if dims.dtype == MLA_FP32 else torch.bfloat16), dims.d_c + dims.d_R


def _poison(data):
    if data.dtype == torch.bfloat16:
        data.view(torch.int16).fill_(POISON_BF16)
    elif data.dtype == torch.uint8:
        data.fill_(POISON_BYTE)
    else:
        data.view(torch.int32).fill_(POISON_FP32)


class LatentCache:
    def __init__(self, dims, capacities, device="cuda", poison=False, gap=0):
        self.dims = dims
        self.dtype, self.row = _row_storage(dims)
        caps = [int(c) for c in capacities]
        starts, s = [], 0
        for c in caps:
            starts.append(s)
            s += c + gap
        self.total_rows = s
        self.capacity = torch.tensor(caps, dtype=torch.int32, device=device)
        self.seq_start = torch.tensor(starts, dtype=torch.int64, device=device)
        self.data = torch.empty((max(s, 1), self.row), dtype=self.dtype, device=device)
        if poison:
            self.poison_()
        self.handle = make_cache(self.data, self.seq_start, self.capacity)

    def poison_(self):
        _poison(self.data)

    def rows_of(self, seq, n):
        s = int(self.seq_start[seq].item())
        return self.data[s:s + n]


class PagedLatentCache:
    """Latent cache as a pool of pages of `block_size` rows with a block table.

    Sequence s owns pages block_table[s, :ceil(capacity[s] / block_size)];
    token p of sequence s lives in row block_table[s, p // block_size] *
    block_size + p % block_size.  Pages are handed out in the order of
    `page_order` (a permutation of the pool, e.g. shuffled so that a
    sequence's pages are scattered), and the pool may hold spare pages.
    """

    def __init__(self, dims, capacities, block_size=64, device="cuda", poison=False, spare_pages=0,
                 page_order=None):
        self.dims = dims
        self.dtype, self.row = _row_storage(dims)
        self.block_size = int(block_size)
        caps = [int(c) for c in capacities]
        need = [(c + self.block_size - 1) // self.block_size for c in caps]
        self.max_blocks = max(1, max(need))
        n_pages = sum(need) + int(spare_pages)
        order = list(range(n_pages)) if page_order is None else [int(x) for x in page_order]
        assert sorted(order) == list(range(n_pages))
        table = [[-1] * self.max_blocks for _ in caps]
        k = 0
        for s, n in enumerate(need):
            for j in range(n):
                table[s][j] = order[k]
                k += 1
        self.table_host = table
        self.block_table = torch.tensor(table, dtype=torch.int32, device=device)
        self.capacity = torch.tensor(caps, dtype=torch.int32, device=device)
        self.total_rows = n_pages * self.block_size
        self.data = torch.empty((max(self.total_rows, 1), self.row), dtype=self.dtype, device=device)
        if poison:
            self.poison_()
        self.handle = make_cache(self.data, None, self.capacity, block_table=self.block_table,
                                 block_size=self.block_size)

    def poison_(self):
        _poison(self.data)

    def row_of(self, seq, p):
        return self.table_host[seq][p // self.block_size] * self.block_size + p % self.block_size
