"""Seeded synthetic inputs for the MLA latent-KV hot path.

This module only draws numbers: the workload presets, hidden states h_t,
weight matrices and per-sequence cache lengths. It holds none of the
method's arithmetic (no projection, RoPE, softmax or attention), so the
fp64 oracle and the CUDA path can both be fed from it without sharing any
of the computation they are compared on.

Workloads follow the DeepSeek-V2 dimensions given in "DeepSeek-V2 summary"
(7shi.hateblo.jp) §3.1.2 (n_h=128, d_h=128, d_c=512, d_c'=1536, per-head
rotary width 64, d=5120) and App. B.1 for V2-Lite (d=2048, n_h=16, no query
compression).  Value distributions: weights N(0, 0.02), hidden states
N(0, 1), both rounded to the storage dtype (round-to-nearest-even bf16, or
fp32 for the tiny preset).

Every tensor is drawn from its own numpy Generator seeded with
(seed, preset id, tensor id, sequence), so any subset of sequences can be
regenerated without drawing the rest.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = [
    "Dims", "Preset", "PRESETS", "preset", "ragged_lengths", "weights",
    "hidden", "to_bf16_bits", "bf16_bits_to_f32", "round_bf16",
    "WEIGHT_NAMES",
]


@dataclasses.dataclass(frozen=True)
class Dims:
    d_model: int
    n_h: int
    d_h: int
    d_R: int
    d_c: int
    d_cq: int          # 0: no query compression (W_UQ / W_QR act on h directly)
    rope_base: float = 10000.0
    dtype: str = "bf16"  # storage dtype of h, weights and cache: "bf16" | "fp32"
    yarn: tuple | None = None  # (s, alpha, beta, L0) of YaRN, or None for plain RoPE
    cache: str = "dtype"       # latent cache rows: "dtype" (storage dtype) or "e4m3" (low-bit c^KV)

    @property
    def row_elems(self) -> int:
        """Elements per cached token per layer: [c_KV (d_c) | k^R (d_R)]."""
        return self.d_c + self.d_R


@dataclasses.dataclass(frozen=True)
class Preset:
    name: str
    pid: int
    dims: Dims
    batch: int
    seqlen: tuple | None   # cached tokens per sequence before the new one (decode)
    prefill_T: int = 0     # tokens of a causal prefill (prefill preset only)


V2 = Dims(d_model=5120, n_h=128, d_h=128, d_R=64, d_c=512, d_cq=1536)
V2_LITE = Dims(d_model=2048, n_h=16, d_h=128, d_R=64, d_c=512, d_cq=0)
TINY = Dims(d_model=64, n_h=4, d_h=16, d_R=8, d_c=32, d_cq=48, dtype="fp32")


def ragged_lengths(seed: int = 0, batch: int = 128, max_len: int = 131072) -> np.ndarray:
    """Per-sequence cache lengths drawn log-uniform in [1, max_len].

    L = clip(floor(exp(U(0, ln max_len))), 1, max_len) from
    numpy.random.default_rng(seed).  For seed 0 and batch 128 this gives
    sum 2,007,088, max 126,832 and median 679.
    """
    rng = np.random.default_rng(seed=seed)
    u = rng.uniform(0.0, np.log(max_len), batch)
    return np.clip(np.floor(np.exp(u)), 1, max_len).astype(np.int64)


PRESETS = {
    "tiny": Preset("tiny", 1, TINY, 1, (64,)),
    "lite": Preset("lite", 2, V2_LITE, 32, (4096,) * 32),
    "v2": Preset("v2", 3, V2, 64, (8192,) * 64),
    "ragged": Preset("ragged", 4, V2, 128, tuple(int(x) for x in ragged_lengths(0))),
    "prefill": Preset("prefill", 5, V2, 1, None, prefill_T=16384),
}


def preset(name: str) -> Preset:
    return PRESETS[name]


WEIGHT_NAMES = ("W_DQ", "W_UQ", "W_QR", "W_DKV", "W_UK", "W_UV", "W_KR", "W_O")
_TENSOR_ID = {n: i + 1 for i, n in enumerate(WEIGHT_NAMES)}
_H_ID = 100


def weight_shapes(d: Dims) -> dict:
    """Shapes [out, in] of the weight matrices (y = W x)."""
    qin = d.d_cq if d.d_cq else d.d_model
    shapes = {
        "W_UQ": (d.n_h * d.d_h, qin),
        "W_QR": (d.n_h * d.d_R, qin),
        "W_DKV": (d.d_c, d.d_model),
        "W_UK": (d.n_h * d.d_h, d.d_c),
        "W_UV": (d.n_h * d.d_h, d.d_c),
        "W_KR": (d.d_R, d.d_model),
        "W_O": (d.d_model, d.n_h * d.d_h),
    }
    if d.d_cq:
        shapes["W_DQ"] = (d.d_cq, d.d_model)
    return shapes


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Values of x rounded to bf16 (RNE), returned as float32."""
    return bf16_bits_to_f32(to_bf16_bits(np.asarray(x, dtype=np.float32)))


def _rng(seed: int, pid: int, tid: int, seq: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, pid, tid, seq])


def _draw(rng: np.random.Generator, shape, std: float, dtype: str) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32) * np.float32(std)
    return round_bf16(x) if dtype == "bf16" else x


def weights(p: Preset, seed: int = 0, std: float = 0.02) -> dict:
    """The layer's weight matrices as float32 arrays holding storage-exact values."""
    out = {}
    for name, shape in weight_shapes(p.dims).items():
        out[name] = _draw(_rng(seed, p.pid, _TENSOR_ID[name]), shape, std, p.dims.dtype)
    return out


def hidden(p: Preset, seq: int, n_tokens: int, seed: int = 0, first: int = 0) -> np.ndarray:
    """Hidden states h_t of one sequence, tokens [first, first + n_tokens).

    Token t of sequence `seq` is always the same vector whatever range is
    asked for: each token row has its own generator keyed by its index.
    Rows are drawn in blocks of 256 tokens to keep this cheap.
    """
    d = p.dims.d_model
    blk = 256
    out = np.empty((n_tokens, d), dtype=np.float32)
    t = first
    while t < first + n_tokens:
        b0 = (t // blk) * blk
        rng = _rng(seed, p.pid, _H_ID, seq * 1_000_003 + b0 // blk)
        block = _draw(rng, (blk, d), 1.0, p.dims.dtype)
        lo = t - b0
        hi = min(blk, first + n_tokens - b0)
        out[t - first:t - first + (hi - lo)] = block[lo:hi]
        t = b0 + hi
    return out
