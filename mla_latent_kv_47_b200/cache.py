"""Contiguous per-sequence latent cache on the device (allocation and bookkeeping).

Row layout per token: [c^KV (d_c) | k^R (d_R)] in the storage dtype; sequence s
owns rows [seq_start[s], seq_start[s] + capacity[s]).  Writes go through the
library (mla_cache_append / mla_decode / mla_prefill).
"""
from __future__ import annotations

import torch

from . import make_cache, MLA_FP32

POISON_BF16 = 0x7FC1          # a quiet NaN; rows never written keep this pattern
POISON_FP32 = 0x7FC00001


class LatentCache:
    def __init__(self, dims, capacities, device="cuda", poison=False, gap=0):
        self.dims = dims
        self.dtype = torch.float32 if dims.dtype == MLA_FP32 else torch.bfloat16
        self.row = dims.d_c + dims.d_R
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
        if self.dtype == torch.bfloat16:
            self.data.view(torch.int16).fill_(POISON_BF16)
        else:
            self.data.view(torch.int32).fill_(POISON_FP32)

    def rows_of(self, seq, n):
        s = int(self.seq_start[seq].item())
        return self.data[s:s + n]
