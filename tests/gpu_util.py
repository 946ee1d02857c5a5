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


def cache_value_check(got_bits: np.ndarray, Wh: dict, h: np.ndarray, pos: np.ndarray, dims) -> float:
    """Checks stored bf16 cache rows against the exact rows [c^KV | RoPE(k^R)].

    Bound per element: rounding to bf16 (half an ulp <= 2^-8 |x|) plus the
    noise of an fp32 dot product of length K = d_model, taken as
    16 sqrt(K) 2^-24 ||w o h||_2 (a generous multiple of the random-walk size of
    fp32 summation error); a rotated k^R element carries the noise of both
    members of its pair plus a few fp32 roundings of the rotation.
    Returns the largest |error| / bound (must be <= 1)."""
    from oracle import mla as om
    c_kv, k_r = om.latent_rows(Wh, h, pos, dims)
    exact = np.concatenate([c_kv, k_r], axis=1)
    got = synth.bf16_bits_to_f32(got_bits).astype(np.float64)
    K = dims.d_model
    u = 2.0 ** -24
    h2 = np.asarray(h, np.float64) ** 2
    noise_c = np.sqrt(h2 @ (np.asarray(Wh["W_DKV"], np.float64) ** 2).T)
    if "g_kv" in Wh:
        # RMSNorm on c^KV: the fp32 noise of each element is divided by the
        # row's RMS and multiplied by its gain
        raw = np.asarray(h, np.float64) @ np.asarray(Wh["W_DKV"], np.float64).T
        rms = np.sqrt(np.mean(raw * raw, axis=1, keepdims=True) + 1e-6)
        g = np.abs(np.asarray(Wh["g_kv"], np.float64))[None, :]
        noise_c = noise_c * g / rms
    pre_r = np.asarray(h, np.float64) @ np.asarray(Wh["W_KR"], np.float64).T
    noise_r = np.sqrt(h2 @ (np.asarray(Wh["W_KR"], np.float64) ** 2).T)
    pair = noise_r.reshape(noise_r.shape[0], -1, 2).sum(-1).repeat(2, axis=1)
    pair_mag = np.abs(pre_r).reshape(pre_r.shape[0], -1, 2).sum(-1).repeat(2, axis=1)
    acc = 16.0 * np.sqrt(K) * u * np.concatenate([noise_c, pair], axis=1)
    rot = np.concatenate([np.zeros_like(noise_c), 8 * u * pair_mag], axis=1)
    bound = 2.0 ** -8 * np.abs(exact) + (1 + 2.0 ** -8) * acc + rot
    if "g_kv" in Wh:
        # the norm's own fp32 arithmetic (a sum of squares over d_c, rsqrt, two
        # products) and the noise of the RMS itself: well under 2^-14 relative
        bound[:, :c_kv.shape[1]] += 2.0 ** -14 * np.abs(c_kv)
    return float(np.max(np.abs(got - exact) / bound))


def e4m3_row_check(got_bytes: np.ndarray, Wh: dict, h: np.ndarray, pos: np.ndarray, dims) -> float:
    """Checks stored E4M3 cache rows (bytes of the mla_cache_format layout)
    against the exact rows.  c^KV: the decoded value code * 2^k must be within
    half a code spacing of the exact value (2^-4 relative for normal codes,
    2^(k-10) absolute below the smallest normal, 2^(k-6)) plus the fp32 noise
    of the down-projection; the scale exponent must be the oracle's rule
    applied to the row; the 15 padding bytes must be zero.  k^R: bf16 within
    half an ulp plus the rotation's fp32 noise.  Returns the largest
    |error| / bound (must be <= 1)."""
    from oracle import lowbit as lb
    from oracle import mla as om
    d_c, d_R = dims.d_c, dims.d_R
    c_kv, k_r = om.latent_rows(Wh, h, pos, dims)
    g = np.asarray(got_bytes, dtype=np.uint8)
    k = g[:, d_c + 2 * d_R].view(np.int8).astype(np.int64)
    assert np.all(g[:, d_c + 2 * d_R + 1:d_c + 2 * d_R + 16] == 0), "padding bytes"
    # the scale rule on the exact row may differ by one where amax sits on a power-of-two edge
    k_ref = lb.row_scale_exp(np.max(np.abs(c_kv), axis=1), "e4m3")
    assert np.all(np.abs(k - k_ref) <= 1), "scale exponent"
    dec = lb.dequantize_rows(g[:, :d_c], k, "e4m3")
    u = 2.0 ** -24
    h2 = np.asarray(h, np.float64) ** 2
    noise = 16.0 * np.sqrt(dims.d_model) * u * np.sqrt(h2 @ (np.asarray(Wh["W_DKV"], np.float64) ** 2).T)
    bound_c = 2.0 ** -4 * np.abs(c_kv) + np.ldexp(1.0, k - 10)[:, None] + 2 * noise
    ratio = float(np.max(np.abs(dec - c_kv) / bound_c))
    kr = bf16_bits_to_f64(g[:, d_c:d_c + 2 * d_R].copy().view(np.uint16))
    bound_r = 2.0 ** -8 * np.abs(k_r) + 1e-4 * (1.0 + np.abs(k_r))
    return max(ratio, float(np.max(np.abs(kr - k_r) / bound_r)))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)
