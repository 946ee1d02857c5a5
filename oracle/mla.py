"""Plain fp64 CPU oracle of DeepSeek-V2 Multi-head Latent Attention (MLA).

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports this file;
only tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of the
benchmark do.  It shares no code with the CUDA path.

Source of every formula: "DeepSeek-V2 summary" (7shi.hateblo.jp), App. C
"Full Formulas of MLA", with the notation of its §2.1.1-§2.1.3:

    c^Q_t   = W^{DQ} h_t                       (query compression, width d_c')
    q^C_t   = W^{UQ} c^Q_t                     (per head d_h)
    q^R_t   = RoPE(W^{QR} c^Q_t)               (per head d_R, decoupled RoPE)
    c^KV_t  = W^{DKV} h_t                      (cached latent, width d_c)
    k^C_t   = W^{UK} c^KV_t                    (per head d_h)
    k^R_t   = RoPE(W^{KR} h_t)                 (width d_R, one key shared by all heads, cached)
    v^C_t   = W^{UV} c^KV_t                    (per head d_h)
    q_{t,i} = [q^C_{t,i}; q^R_{t,i}],  k_{j,i} = [k^C_{j,i}; k^R_j]
    o_{t,i} = sum_{j<=t} softmax_j(q_{t,i}.k_{j,i} / sqrt(d_h + d_R)) v^C_{j,i}
    u_t     = W^O [o_{t,1}; ...; o_{t,n_h}]

Readings taken where the pages are silent or garbled (each is listed in the
design notes of this repository):
  * RoPE pairs interleaved components (2m, 2m+1) and rotates them by
    phi = pos * base^(-2m/d_R) (the RoFormer definition; the pages only say
    "RoPE").  Positions are 0-based token indices within the sequence.
  * The rotary key is shared by all heads ("shared key" in §2.1.3); App. C's
    per-head superscript on it is taken as a typo.
  * Concatenation order inside q and k does not change a dot product; the
    cache row is [c^KV | k^R].
  * Without query compression (V2-Lite, App. B.1) W^{UQ} and W^{QR} act on
    h_t directly.
  * RMSNorm on the latents (§3.1.2) is not part of App. C.  It is applied
    only when the weights carry its gains: "g_kv" [d_c] normalises c^KV
    before it is cached, and "g_q" [d_cq] normalises c^Q before the
    up-projections (RMS over the latent's own width, eps = RMS_EPS; the pages
    give neither the placement nor eps).
  * YaRN (§3.1.4) is not part of App. C either.  It is applied only when
    dims carries `yarn` = (s, alpha, beta, L0): the rotary frequencies of q^R
    and k^R ramp from theta/s to theta as L0 holds between alpha and beta of
    their wavelengths (the published YaRN rule; the pages give s = 40,
    alpha = 1, beta = 32 and the 4K pre-training length), and every score is
    multiplied by t with sqrt(t) = 0.0707 ln s + 1.

Weights use the pages' shapes W in R^{out x in} with y = W x.  Head i owns rows
[i d_h, (i+1) d_h) of W^{UQ}, W^{UK}, W^{UV}, rows [i d_R, (i+1) d_R) of W^{QR}
and columns [i d_h, (i+1) d_h) of W^O.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rope", "yarn_theta", "yarn_score_factor", "score_scale", "rmsnorm", "RMS_EPS", "latent_rows", "queries", "keys_values", "softmax", "attend",
    "decode_unabsorbed", "decode_absorbed", "prefill_unabsorbed",
    "round_bf16_f64", "cache_row_elems",
]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def cache_row_elems(d_c: int, d_R: int) -> int:
    """Elements cached per token per layer: only c^KV and k^R (App. C, blue boxes)."""
    return d_c + d_R


def rope(x, pos, base: float, theta=None):
    """Rotary position embedding on the last axis (width d_R, even).

    Pair m = (x[2m], x[2m+1]) is rotated by phi = pos * theta_m with
    theta_m = base^(-2m/d_R) unless `theta` gives the frequencies:
    (a, b) -> (a cos phi - b sin phi, a sin phi + b cos phi).
    `pos` broadcasts against x's leading axes.
    """
    x = _f64(x)
    d_R = x.shape[-1]
    if theta is None:
        m = np.arange(d_R // 2, dtype=np.float64)
        theta = np.power(float(base), -2.0 * m / d_R)
    theta = _f64(theta)
    phi = _f64(pos)[..., None] * theta
    c, s = np.cos(phi), np.sin(phi)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, phi.shape[:-1] + (d_R,)), dtype=np.float64)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def yarn_theta(d_R: int, base: float, yarn):
    """YaRN rotary frequencies for yarn = (s, alpha, beta, L0).

    Pair m keeps theta_m = base^(-2m/d_R) when the pre-training length L0
    spans more than beta of its wavelengths 2 pi / theta_m, takes theta_m / s
    (position interpolation) below alpha of them, and ramps linearly in
    between.
    """
    s, alpha, beta, L0 = yarn
    m = np.arange(d_R // 2, dtype=np.float64)
    theta = np.power(float(base), -2.0 * m / d_R)
    r = L0 * theta / (2.0 * np.pi)            # wavelengths inside L0
    ramp = np.clip((r - alpha) / (beta - alpha), 0.0, 1.0)
    return (1.0 - ramp) * theta / s + ramp * theta


def yarn_score_factor(s: float) -> float:
    """t with sqrt(t) = 0.0707 ln s + 1, the factor on every attention score."""
    return (0.0707 * np.log(s) + 1.0) ** 2


def _theta(dims):
    y = getattr(dims, "yarn", None)
    return None if y is None else yarn_theta(dims.d_R, dims.rope_base, y)


def score_scale(dims) -> float:
    """Softmax scale: 1/sqrt(d_h + d_R), times YaRN's t when dims carries yarn."""
    y = getattr(dims, "yarn", None)
    return (1.0 if y is None else yarn_score_factor(y[0])) / np.sqrt(dims.d_h + dims.d_R)


RMS_EPS = 1e-6


def rmsnorm(x, g, eps=None):
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    x = _f64(x)
    eps = RMS_EPS if eps is None else eps
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * _f64(g)


def latent_rows(W: dict, h, pos, dims):
    """The cached vectors of tokens h [T, d] at positions pos [T].

    Returns (c_kv [T, d_c], k_r [T, d_R]): c^KV = W^{DKV} h (RMS-normalised
    with gains W["g_kv"] when present), k^R = RoPE(W^{KR} h).
    """
    h = _f64(h)
    c_kv = h @ _f64(W["W_DKV"]).T
    if "g_kv" in W:
        c_kv = rmsnorm(c_kv, W["g_kv"])
    k_r = rope(h @ _f64(W["W_KR"]).T, pos, dims.rope_base, _theta(dims))
    return c_kv, k_r


def queries(W: dict, h, pos, dims):
    """Per-head query parts: q^C [T, n_h, d_h] and q^R [T, n_h, d_R] (c^Q
    RMS-normalised with gains W["g_q"] when present)."""
    h = _f64(h)
    T = h.shape[0]
    c_q = h @ _f64(W["W_DQ"]).T if dims.d_cq else h
    if dims.d_cq and "g_q" in W:
        c_q = rmsnorm(c_q, W["g_q"])
    q_c = (c_q @ _f64(W["W_UQ"]).T).reshape(T, dims.n_h, dims.d_h)
    q_r = rope((c_q @ _f64(W["W_QR"]).T).reshape(T, dims.n_h, dims.d_R),
               _f64(pos)[:, None], dims.rope_base, _theta(dims))
    return q_c, q_r


def keys_values(W: dict, c_kv, k_r, dims):
    """Un-absorbed per-head keys [T, n_h, d_h + d_R] and values [T, n_h, d_h].

    k_{j,i} = [W^{UK}_i c^KV_j ; k^R_j], v_{j,i} = W^{UV}_i c^KV_j.
    """
    c_kv = _f64(c_kv)
    T = c_kv.shape[0]
    k_c = (c_kv @ _f64(W["W_UK"]).T).reshape(T, dims.n_h, dims.d_h)
    v = (c_kv @ _f64(W["W_UV"]).T).reshape(T, dims.n_h, dims.d_h)
    k_rh = np.broadcast_to(_f64(k_r)[:, None, :], (T, dims.n_h, dims.d_R))
    return np.concatenate([k_c, k_rh], axis=-1), v


def softmax(s, axis=-1):
    """exp(s - max) / sum exp(s - max) along `axis`."""
    s = _f64(s)
    e = np.exp(s - np.max(s, axis=axis, keepdims=True))
    return e / np.sum(e, axis=axis, keepdims=True)


def attend(q, k, v, scale):
    """One query per head over keys j: q [n_h, dq], k [L, n_h, dq], v [L, n_h, dv].

    Returns (o [n_h, dv], p [n_h, L]).
    """
    s = np.einsum("hd,jhd->hj", _f64(q), _f64(k)) * scale
    p = softmax(s, axis=-1)
    o = np.einsum("hj,jhd->hd", p, _f64(v))
    return o, p


def _output(W, o, dims):
    """u = W^O [o_1; ...; o_{n_h}]."""
    return _f64(W["W_O"]) @ o.reshape(-1)


def decode_unabsorbed(W: dict, h_seq, dims, cache_rows=None):
    """u for the last token of one sequence, by the naive App. C formulas.

    h_seq [L+1, d]: hidden states of the cached tokens 0..L-1 and of the new
    token L (position L).  The query attends over j = 0..L (itself included).
    If `cache_rows` = (c_kv, k_r) is given it replaces the recomputed latents
    (used to feed the oracle storage-rounded cache values).
    """
    h_seq = _f64(h_seq)
    L1 = h_seq.shape[0]
    pos = np.arange(L1, dtype=np.float64)
    c_kv, k_r = latent_rows(W, h_seq, pos, dims) if cache_rows is None else cache_rows
    k, v = keys_values(W, c_kv, k_r, dims)
    q_c, q_r = queries(W, h_seq[-1:], pos[-1:], dims)
    q = np.concatenate([q_c[0], q_r[0]], axis=-1)
    o, _ = attend(q, k, v, score_scale(dims))
    return _output(W, o, dims)


def decode_absorbed(W: dict, h_seq, dims, return_parts=False, cache_rows=None):
    """Same result as decode_unabsorbed, with W^{UK} and W^{UV} absorbed.

    Associativity (App. C, last paragraph): q^C_i . (W^{UK}_i c_j) =
    (W^{UK}_i^T q^C_i) . c_j, and W^{UV}_i sum_j p_j c_j = sum_j p_j W^{UV}_i c_j,
    so keys and values are never formed: every head scores against the cached
    [c^KV_j ; k^R_j] row with q_lat_i = [W^{UK}_i^T q^C_i ; q^R_i].  The
    identity holds for any cached rows, so `cache_rows` = (c_kv, k_r) may
    replace the recomputed latents as in decode_unabsorbed.
    """
    h_seq = _f64(h_seq)
    L1 = h_seq.shape[0]
    pos = np.arange(L1, dtype=np.float64)
    c_kv, k_r = latent_rows(W, h_seq, pos, dims) if cache_rows is None else (_f64(cache_rows[0]), _f64(cache_rows[1]))
    q_c, q_r = queries(W, h_seq[-1:], pos[-1:], dims)
    W_UK = _f64(W["W_UK"]).reshape(dims.n_h, dims.d_h, dims.d_c)
    W_UV = _f64(W["W_UV"]).reshape(dims.n_h, dims.d_h, dims.d_c)
    q_abs = np.einsum("hdc,hd->hc", W_UK, q_c[0])                      # [n_h, d_c]
    q_lat = np.concatenate([q_abs, q_r[0]], axis=-1)                   # [n_h, d_c + d_R]
    rows = np.concatenate([c_kv, k_r], axis=-1)                        # [L+1, d_c + d_R]
    s = (q_lat @ rows.T) * score_scale(dims)                          # [n_h, L+1]
    p = softmax(s, axis=-1)
    o_lat = p @ c_kv                                                   # [n_h, d_c]
    o = np.einsum("hdc,hc->hd", W_UV, o_lat)                           # [n_h, d_h]
    u = _output(W, o, dims)
    if return_parts:
        return u, dict(q_lat=q_lat, o_lat=o_lat, rows=rows, p=p, o=o)
    return u


def prefill_unabsorbed(W: dict, h, dims, start_pos: int = 0, h_prefix=None, rows=None):
    """u for the tokens of a causal prefill, by the naive App. C formulas.

    h [T, d] are tokens at positions start_pos .. start_pos+T-1; h_prefix
    [start_pos, d] are the hidden states of the tokens already cached.
    Token t attends over every j <= t.  `rows` (indices into h) limits which
    outputs are formed; the result then has one row per entry of `rows`.
    """
    h = _f64(h)
    T = h.shape[0]
    h_all = h if h_prefix is None else np.concatenate([_f64(h_prefix), h], axis=0)
    assert h_all.shape[0] == start_pos + T
    pos_all = np.arange(start_pos + T, dtype=np.float64)
    c_kv, k_r = latent_rows(W, h_all, pos_all, dims)
    k, v = keys_values(W, c_kv, k_r, dims)
    rows = list(range(T)) if rows is None else [int(r) for r in rows]
    q_c, q_r = queries(W, h[rows], pos_all[start_pos:][rows], dims)
    q = np.concatenate([q_c, q_r], axis=-1)                            # [len(rows), n_h, dq]
    scale = score_scale(dims)
    u = np.empty((len(rows), dims.d_model), dtype=np.float64)
    for i, t in enumerate(rows):
        n = start_pos + t + 1
        o, _ = attend(q[i], k[:n], v[:n], scale)
        u[i] = _output(W, o, dims)
    return u


def round_bf16_f64(x):
    """fp64 values rounded to the nearest bf16 (ties to even), returned as fp64.

    Rounds directly from fp64 (no fp32 intermediate), so it is the bf16
    nearest to the exact value.
    """
    x = _f64(x)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    scaled = np.ldexp(m, 8)                  # 8 significant bits in |scaled| in [128, 256)
    r = np.round(scaled)                     # numpy rounds half to even
    return np.ldexp(r, e - 8)
