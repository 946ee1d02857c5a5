"""Low-bit latent-cache storage for the oracle.

TEST INFRASTRUCTURE ONLY, under the same rules as ``oracle/mla.py``: only
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU leg may import it,
and it shares no code with the CUDA path.

What the pages say.  The deployed model quantises each element of the KV
cache to about 6 bits on average ("DeepSeek-V2 summary" (7shi.hateblo.jp),
§3.2.3), and the recommended serving example runs an FP8 E5M2 KV cache
("딥시크 V2" (downcodes.com), §8, inference with SGLang).  Neither gives a
scheme.

Reading taken.  A cache row's c^KV part, and optionally its k^R part, is
stored as elements of one small-float format times one power-of-two scale
per row and part.  The element formats are the OCP 8-bit and 6-bit floats
(all with subnormals):

    name   exponent  mantissa  bias   largest finite   non-finite codes
    e5m2      5         2       15       57344         exponent all ones (inf, NaN)
    e4m3      4         3        7         448         S.1111.111 (NaN)
    e3m2      3         2        3          28         none
    e2m3      2         3        1         7.5         none

An element is the representable value nearest to x / 2^k, ties to the even
code (the code whose last mantissa bit is 0).  The row's scale 2^k is the
smallest power of two with amax / 2^k <= largest finite (amax: the largest
magnitude of the row's part), so no element saturates and the largest one
keeps the format's full relative precision.  An all-zero part has k = 0.
Decoding multiplies the element value by 2^k exactly.
"""
from __future__ import annotations

import math

import numpy as np

from oracle.mla import decode_absorbed, decode_unabsorbed, latent_rows, round_bf16_f64

__all__ = ["FORMATS", "code_values", "max_finite", "encode", "decode", "row_scale_exp",
           "quantize_rows", "dequantize_rows", "store_rows", "decode_lowbit"]

# name -> (exponent bits, mantissa bits, bias)
FORMATS = {
    "e5m2": (5, 2, 15),
    "e4m3": (4, 3, 7),
    "e3m2": (3, 2, 3),
    "e2m3": (2, 3, 1),
}


def _fields(fmt):
    if fmt not in FORMATS:
        raise ValueError(f"unknown element format {fmt!r}")
    return FORMATS[fmt]


def code_values(fmt: str) -> np.ndarray:
    """Value of every code 0 .. 2^(1+E+M) - 1 (sign bit highest), NaN where
    the code is not a finite number."""
    E, M, bias = _fields(fmt)
    n = 1 << (1 + E + M)
    out = np.empty(n, dtype=np.float64)
    for c in range(n):
        s = -1.0 if (c >> (E + M)) & 1 else 1.0
        e = (c >> M) & ((1 << E) - 1)
        m = c & ((1 << M) - 1)
        if fmt == "e5m2" and e == (1 << E) - 1:
            out[c] = np.nan                      # inf and NaN codes: never produced by encode
        elif fmt == "e4m3" and e == (1 << E) - 1 and m == (1 << M) - 1:
            out[c] = np.nan
        elif e == 0:
            out[c] = s * math.ldexp(m, 1 - bias - M)
        else:
            out[c] = s * math.ldexp((1 << M) + m, e - bias - M)
    return out


def max_finite(fmt: str) -> float:
    v = code_values(fmt)
    return float(np.nanmax(v))


def encode(x, fmt: str) -> np.ndarray:
    """Codes (uint8) of the values nearest to x, ties to the even code.
    Magnitudes above the largest finite value take it (callers scale so
    that this does not happen); x must not be NaN."""
    E, M, bias = _fields(fmt)
    x = np.asarray(x, dtype=np.float64)
    if np.any(np.isnan(x)):
        raise ValueError("NaN has no code in the cache formats as used here")
    top = max_finite(fmt)
    sign = np.signbit(x)
    a = np.minimum(np.abs(x), top)
    # quantum of the binade of a (the subnormal quantum below the smallest normal)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, 1 - bias)
    quantum = np.ldexp(1.0, (e - M).astype(np.int64))
    q = np.round(a / quantum) * quantum          # numpy rounds halves to even
    q = np.minimum(q, top)
    # value -> code through the table of non-negative finite values
    vals = code_values(fmt)[: 1 << (E + M)]
    finite = np.isfinite(vals)
    pos_codes = np.nonzero(finite)[0]
    pos_vals = vals[finite]
    idx = np.searchsorted(pos_vals, q)
    if not np.all(pos_vals[np.minimum(idx, len(pos_vals) - 1)] == q):
        raise AssertionError("rounded value off the format's grid")
    codes = pos_codes[idx] | (sign.astype(np.int64) << (E + M))
    return codes.astype(np.uint8)


def decode(codes, fmt: str) -> np.ndarray:
    return code_values(fmt)[np.asarray(codes, dtype=np.int64)]


def row_scale_exp(amax, fmt: str) -> np.ndarray:
    """k per row: the smallest integer with amax / 2^k <= largest finite (0 for amax = 0)."""
    amax = np.asarray(amax, dtype=np.float64)
    top = max_finite(fmt)
    k = np.zeros(amax.shape, dtype=np.int64)
    nz = amax > 0
    k[nz] = np.ceil(np.log2(amax[nz] / top)).astype(np.int64)
    # guard the log2 rounding at exact powers of two
    over = nz & (np.ldexp(top, k) < amax)
    k[over] += 1
    under = nz & (np.ldexp(top, k - 1) >= amax)
    k[under] -= 1
    return k


def quantize_rows(x, fmt: str):
    """(codes [n, d] uint8, k [n] int64) of rows x [n, d]."""
    x = np.asarray(x, dtype=np.float64)
    k = row_scale_exp(np.max(np.abs(x), axis=1), fmt)
    codes = encode(np.ldexp(x, -k[:, None]), fmt)
    return codes, k


def dequantize_rows(codes, k, fmt: str) -> np.ndarray:
    return np.ldexp(decode(codes, fmt), np.asarray(k)[:, None])


def store_rows(c_kv, k_r, fmt_c: str, fmt_r: str | None = None):
    """The cache rows as the low-bit cache holds them, returned in fp64:
    c^KV in fmt_c with a per-row scale; k^R in fmt_r likewise, or rounded
    to bf16 when fmt_r is None."""
    c_codes, c_k = quantize_rows(c_kv, fmt_c)
    c_store = dequantize_rows(c_codes, c_k, fmt_c)
    if fmt_r is None:
        r_store = round_bf16_f64(k_r)
    else:
        r_codes, r_k = quantize_rows(k_r, fmt_r)
        r_store = dequantize_rows(r_codes, r_k, fmt_r)
    return c_store, r_store


def decode_lowbit(W: dict, h_seq, dims, fmt_c: str, fmt_r: str | None = None, absorbed: bool = False):
    """u of the App. C decode step over a cache stored in the low-bit format:
    the exact latent rows, stored and read back by store_rows, then the
    un-absorbed formulas of oracle.mla (or, with `absorbed`, the absorbed form,
    which is pinned to them and far cheaper for long sequences)."""
    h_seq = np.asarray(h_seq, dtype=np.float64)
    pos = np.arange(h_seq.shape[0], dtype=np.float64)
    c_kv, k_r = latent_rows(W, h_seq, pos, dims)
    rows = store_rows(c_kv, k_r, fmt_c, fmt_r)
    if absorbed:
        return decode_absorbed(W, h_seq, dims, cache_rows=rows)
    return decode_unabsorbed(W, h_seq, dims, cache_rows=rows)
