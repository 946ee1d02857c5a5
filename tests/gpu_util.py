"""Shared helpers of the GPU parity tests: device copies of the synthetic inputs,
cache filling through the library, and the parity gate."""
from __future__ import annotations

import numpy as np
import torch

import synth

BF16_GATE_MAX = 1e-2    # max|d| <= 1e-2 max|ref|
BF16_GATE_MEAN = 2e-3   # mean|d| <= 2e-3 max|ref|


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        bits = synth.to_bf16_bits(np.asarray(x, dtype=np.float32))
        return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def to_host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def gate(u_gpu: np.ndarray, u_ref: np.ndarray) -> dict:
    d = np.abs(np.asarray(u_gpu, np.float64) - u_ref)
    mx = float(np.max(np.abs(u_ref)))
    return {
        "max_rel": float(d.max() / mx),
        "mean_rel": float(d.mean() / mx),
        "sum_rel": float(d.sum() / np.abs(u_ref).sum()),
        "finite": bool(np.all(np.isfinite(u_gpu))),
    }


def assert_gate(stats: dict, max_rel=BF16_GATE_MAX, mean_rel=BF16_GATE_MEAN):
    assert stats["finite"], stats
    assert stats["max_rel"] <= max_rel, stats
    assert stats["mean_rel"] <= mean_rel, stats


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """|a - b| in units in the last place, for bf16 bit patterns of equal sign
    (sign-magnitude mapped onto a monotone integer line)."""
    def key(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)
    return np.abs(key(a_bits) - key(b_bits))


def device_weights(p: synth.Preset, seed=0):
    Wh = synth.weights(p, seed=seed)
    return Wh, {k: to_dev(v, p.dims.dtype) for k, v in Wh.items()}


def fill_cache(m, dims, Wd, cache, ws, seqs_h: dict, lengths, p, gen_seed=1234, chunk=32768):
    """Appends tokens 0..L_b-1 of every sequence b.  Sequences listed in
    `seqs_h` use those host hidden states (oracle-checked); the others get
    device-drawn N(0,1) states that no oracle looks at."""
    wts = m.make_weights(Wd)
    g = torch.Generator(device="cuda")
    g.manual_seed(gen_seed)
    tdt = torch.float32 if p.dims.dtype == "fp32" else torch.bfloat16
    for b, L in enumerate(lengths):
        for t0 in range(0, L, chunk):
            n = min(chunk, L - t0)
            if b in seqs_h:
                h = to_dev(seqs_h[b][t0:t0 + n], p.dims.dtype)
            else:
                h = torch.randn((n, p.dims.d_model), generator=g, device="cuda", dtype=torch.float32).to(tdt)
            seq = torch.full((n,), b, dtype=torch.int32, device="cuda")
            pos = torch.arange(t0, t0 + n, dtype=torch.int32, device="cuda")
            m.cache_append(dims, wts, h, seq, pos, cache.handle, ws)
