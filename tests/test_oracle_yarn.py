"""Pins of the oracle's optional YaRN rotary scaling.

"DeepSeek-V2 summary" (7shi.hateblo.jp) §3.1.4 extends the 4K context with
YaRN on the decoupled rotary key (s = 40, alpha = 1, beta = 32) and scales
the attention by t with sqrt(t) = 0.0707 ln s + 1.  The oracle applies this
only when dims carries `yarn`.  Pins: s = 1 is plain RoPE; rotary pairs with
many wavelengths inside the pre-training length keep their frequency, pairs
with less than one are plain RoPE at position / s; the ramp between is
monotone; rotations keep norms and relative-position invariance; the factor
t enters every score exactly as a query scaled by t would; and decode
depends only on relative positions, which fails when queries and keys
rotate differently.
"""
import math
import types

import numpy as np
import pytest

from oracle import mla as om
from synth import Dims
from tests.test_oracle_pins import rand_h, rand_weights

V2_YARN = (40.0, 1.0, 32.0, 4096.0)
SMALLY = Dims(d_model=8, n_h=2, d_h=4, d_R=8, d_c=6, d_cq=5, rope_base=10000.0, dtype="fp32")


def with_yarn(dims, yarn):
    d = types.SimpleNamespace(**{k: getattr(dims, k) for k in dims.__dataclass_fields__})
    d.yarn = yarn
    return d


def _classes(d_R, base, yarn):
    s, alpha, beta, L0 = yarn
    theta = np.power(base, -2.0 * np.arange(d_R // 2) / d_R)
    r = L0 * theta / (2 * np.pi)
    return r > beta, r < alpha


def test_s1_is_plain_rope():
    for d_R in (8, 64):
        assert np.allclose(om.yarn_theta(d_R, 10000.0, (1.0, 1.0, 32.0, 4096.0)),
                           np.power(10000.0, -2.0 * np.arange(d_R // 2) / d_R), rtol=1e-15, atol=0)
    assert om.yarn_score_factor(1.0) == 1.0
    W = rand_weights(SMALLY, 41)
    h = rand_h(SMALLY, 6, 41)
    a = om.decode_absorbed(W, h, with_yarn(SMALLY, (1.0, 1.0, 32.0, 4096.0)))
    assert np.allclose(a, om.decode_absorbed(W, h, SMALLY), rtol=1e-13, atol=1e-15)


def test_fast_pairs_keep_their_frequency_and_slow_pairs_interpolate():
    d_R, base = 64, 10000.0                      # the V2 rotary width
    fast, slow = _classes(d_R, base, V2_YARN)
    assert fast.any() and slow.any() and (~fast & ~slow).any()   # all three regimes occur at V2 dims
    rng = np.random.default_rng(3)
    x = rng.standard_normal((9, d_R))
    pos = rng.uniform(0, 160000, 9)
    y = om.rope(x, pos, base, om.yarn_theta(d_R, base, V2_YARN))
    plain = om.rope(x, pos, base)
    interp = om.rope(x, pos / V2_YARN[0], base)
    for m in np.nonzero(fast)[0]:
        assert np.allclose(y[:, 2 * m:2 * m + 2], plain[:, 2 * m:2 * m + 2], rtol=1e-12, atol=1e-12)
    for m in np.nonzero(slow)[0]:
        assert np.allclose(y[:, 2 * m:2 * m + 2], interp[:, 2 * m:2 * m + 2], rtol=1e-9, atol=1e-9)


def test_ramp_is_monotone_between_the_two_regimes():
    d_R, base = 64, 10000.0
    s = V2_YARN[0]
    theta = np.power(base, -2.0 * np.arange(d_R // 2) / d_R)
    ratio = om.yarn_theta(d_R, base, V2_YARN) / theta       # 1 for fast pairs, 1/s for slow ones
    assert np.all(ratio <= 1 + 1e-15) and np.all(ratio >= 1 / s - 1e-15)
    assert np.all(np.diff(ratio) <= 1e-15)                   # slower pairs are interpolated more


def test_rotation_keeps_norms_and_relative_positions():
    d_R, base = 64, 10000.0
    th = om.yarn_theta(d_R, base, V2_YARN)
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(d_R), rng.standard_normal(d_R)
    assert np.isclose(np.linalg.norm(om.rope(q, 1234.0, base, th)), np.linalg.norm(q), rtol=1e-13)
    dots = [om.rope(q, i + 50.0, base, th) @ om.rope(k, j + 50.0, base, th) for i, j in [(900, 100), (1800, 1000), (100800, 100000)]]
    assert np.allclose(dots, dots[0], rtol=1e-8)


def test_score_factor_enters_every_score():
    """With no rotary part (W_QR = W_KR = 0) YaRN changes only the scores'
    scale, exactly as scaling W_UQ by t does without it."""
    W = rand_weights(SMALLY, 42)
    W["W_QR"] = np.zeros_like(W["W_QR"])
    W["W_KR"] = np.zeros_like(W["W_KR"])
    h = rand_h(SMALLY, 7, 42)
    t = om.yarn_score_factor(V2_YARN[0])
    assert 1.5 < t < 1.7                                     # (0.0707 ln 40 + 1)^2
    W2 = dict(W)
    W2["W_UQ"] = np.asarray(W["W_UQ"]) * t
    got = om.decode_unabsorbed(W, h, with_yarn(SMALLY, V2_YARN))
    assert np.allclose(got, om.decode_unabsorbed(W2, h, SMALLY), rtol=1e-11, atol=1e-13)


def _decode_at(W, h, dims, shift):
    """decode_unabsorbed with every position moved by `shift`."""
    L1 = h.shape[0]
    pos = np.arange(L1, dtype=np.float64) + shift
    c_kv, k_r = om.latent_rows(W, h, pos, dims)
    k, v = om.keys_values(W, c_kv, k_r, dims)
    q_c, q_r = om.queries(W, h[-1:], pos[-1:], dims)
    o, _ = om.attend(np.concatenate([q_c[0], q_r[0]], axis=-1), k, v, om.score_scale(dims))
    return om._output(W, o, dims)


def test_decode_depends_on_relative_positions_only():
    W = rand_weights(SMALLY, 43)
    h = rand_h(SMALLY, 6, 43)
    d = with_yarn(SMALLY, (40.0, 1.0, 32.0, 64.0))
    assert np.allclose(_decode_at(W, h, d, 0.0), _decode_at(W, h, d, 12345.0), rtol=1e-8, atol=1e-10)
    assert np.allclose(_decode_at(W, h, d, 0.0), om.decode_unabsorbed(W, h, d), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- planted mistakes

_ORIG_THETA = om.yarn_theta
_ORIG_T = om.yarn_score_factor
_ORIG_ROPE = om.rope
_ORIG_LATENT = om.latent_rows


def _reversed_ramp(d_R, base, yarn):
    s, alpha, beta, L0 = yarn
    theta = np.power(float(base), -2.0 * np.arange(d_R // 2) / d_R)
    ramp = np.clip((L0 * theta / (2 * np.pi) - alpha) / (beta - alpha), 0.0, 1.0)
    return ramp * theta / s + (1 - ramp) * theta


def _keys_plain(W, h, pos, dims):
    d = types.SimpleNamespace(**{k: getattr(dims, k) for k in ("d_model", "n_h", "d_h", "d_R", "d_c", "d_cq", "rope_base", "dtype")})
    return _ORIG_LATENT(W, h, pos, d)


MUTANTS = {
    "ramp_reversed": ("yarn_theta", _reversed_ramp, test_fast_pairs_keep_their_frequency_and_slow_pairs_interpolate),
    "sqrt_t_on_scores": ("yarn_score_factor", lambda s: math.sqrt(_ORIG_T(s)), test_score_factor_enters_every_score),
    "yarn_on_queries_only": ("latent_rows", _keys_plain, test_decode_depends_on_relative_positions_only),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn, pin = MUTANTS[name]
    monkeypatch.setattr(om, attr, fn)
    with pytest.raises(AssertionError):
        pin()


def test_yarn_moves_v2_decode_by_more_than_the_gpu_gate():
    """At DeepSeek-V2 dims and positions past the 4K pre-training length, YaRN
    changes u by several times the GPU parity gate (1e-2 of max|u|), so the GPU
    YaRN parity tests cannot pass with plain RoPE."""
    import dataclasses
    import synth
    p = synth.preset("v2")
    W = synth.weights(p)
    h = synth.hidden(p, 1, 6001)
    a = om.decode_absorbed(W, h, dataclasses.replace(p.dims, yarn=V2_YARN))
    b = om.decode_absorbed(W, h, p.dims)
    assert np.max(np.abs(a - b)) > 5e-2 * np.max(np.abs(a))
