"""Pure-Python brute force of MLA for tiny inputs (lists and `math` only).

Written independently of the numpy oracle: every sum is an explicit loop, every
formula is retyped from "DeepSeek-V2 summary" (7shi.hateblo.jp) App. C, and the
rotary embedding is the RoFormer rotation of interleaved pairs.
"""
import math


def matvec(W, x):
    return [sum(W[r][c] * x[c] for c in range(len(x))) for r in range(len(W))]


def rope_vec(x, pos, base):
    d = len(x)
    out = list(x)
    for m in range(d // 2):
        phi = pos * base ** (-2.0 * m / d)
        a, b = x[2 * m], x[2 * m + 1]
        out[2 * m] = a * math.cos(phi) - b * math.sin(phi)
        out[2 * m + 1] = a * math.sin(phi) + b * math.cos(phi)
    return out


def mla_token_output(W, hs, t, dims):
    """u_t for token t of the sequence hs (list of lists), attending to j <= t."""
    n_h, d_h, d_R = dims.n_h, dims.d_h, dims.d_R
    Wl = {k: [list(map(float, r)) for r in v] for k, v in W.items()}
    h_t = [float(v) for v in hs[t]]
    c_q = matvec(Wl["W_DQ"], h_t) if dims.d_cq else h_t
    q_c = matvec(Wl["W_UQ"], c_q)
    q_r_all = matvec(Wl["W_QR"], c_q)
    keys, vals = [], []
    for j in range(t + 1):
        h_j = [float(v) for v in hs[j]]
        c = matvec(Wl["W_DKV"], h_j)
        k_r = rope_vec(matvec(Wl["W_KR"], h_j), j, dims.rope_base)
        keys.append((matvec(Wl["W_UK"], c), k_r))
        vals.append(matvec(Wl["W_UV"], c))
    o = []
    for i in range(n_h):
        q = q_c[i * d_h:(i + 1) * d_h] + rope_vec(q_r_all[i * d_R:(i + 1) * d_R], t, dims.rope_base)
        scores = []
        for j in range(t + 1):
            k = keys[j][0][i * d_h:(i + 1) * d_h] + keys[j][1]
            scores.append(sum(q[e] * k[e] for e in range(d_h + d_R)) / math.sqrt(d_h + d_R))
        mx = max(scores)
        ex = [math.exp(s - mx) for s in scores]
        z = sum(ex)
        for e in range(d_h):
            o.append(sum(ex[j] / z * vals[j][i * d_h + e] for j in range(t + 1)))
    return matvec(Wl["W_O"], o)
