"""Pins of the oracle's optional RMSNorm on the compressed latents.

The pages add RMSNorm layers after the compressed latent vectors (§3.1.2 of
"DeepSeek-V2 summary" (7shi.hateblo.jp)); App. C has none, so the oracle
applies them only when the weights carry the gains g_kv / g_q.  Pins: an
independent pure-Python RMSNorm, the unit-RMS and scale-invariance
properties, invariance of the whole decode and prefill to scaling the
compression weights once the norm is on, the unchanged default path, and
planted mistakes.
"""
import math

import numpy as np
import pytest

from oracle import mla as om
from tests.test_oracle_pins import SMALL, rand_h, rand_weights


def _brute_rmsnorm(row, g, eps):
    ms = sum(v * v for v in row) / len(row)
    inv = 1.0 / math.sqrt(ms + eps)
    return [v * inv * gi for v, gi in zip(row, g)]


def _with_gains(W, dims, seed):
    rng = np.random.default_rng(seed)
    W = dict(W)
    W["g_kv"] = 0.5 + rng.random(dims.d_c)
    W["g_q"] = 0.5 + rng.random(dims.d_cq)
    return W


def test_rmsnorm_matches_brute_force():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 7)) * np.array([[1e-3], [1.0], [30.0], [1.0], [2.0]])
    g = rng.random(7) + 0.5
    for eps in (0.0, 1e-6, 0.1):
        got = om.rmsnorm(x, g, eps)
        ref = np.array([_brute_rmsnorm(list(r), list(g), eps) for r in x])
        assert np.allclose(got, ref, rtol=1e-13, atol=0)


def test_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((6, 32))
    y = om.rmsnorm(x, np.ones(32), 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    for a in (1e-4, 0.3, 7.0, 1e5):
        assert np.allclose(om.rmsnorm(a * x, np.ones(32), 0.0), y, rtol=1e-13)
    assert np.allclose(om.rmsnorm(-x, np.ones(32), 0.0), -y, rtol=1e-14)


def test_default_path_is_unchanged():
    """Without gains the oracle is App. C exactly (the brute force knows no norm)."""
    from tests import bruteforce_mla as bf
    W = rand_weights(SMALL, 31)
    h = rand_h(SMALL, 4, 31)
    ref = np.array(bf.mla_token_output(W, h.tolist(), 3, SMALL))
    assert np.allclose(om.decode_unabsorbed(W, h, SMALL), ref, rtol=1e-10, atol=1e-12)


def test_normed_latents_have_the_gains_as_rms(monkeypatch):
    monkeypatch.setattr(om, "RMS_EPS", 0.0)
    W = _with_gains(rand_weights(SMALL, 32), SMALL, 32)
    h = rand_h(SMALL, 5, 32)
    c_kv, _ = om.latent_rows(W, h, np.arange(5.0), SMALL)
    assert np.allclose(np.sqrt(np.mean((c_kv / W["g_kv"]) ** 2, axis=-1)), 1.0, rtol=1e-13)


@pytest.mark.parametrize("which", ["W_DKV", "W_DQ"])
def test_output_ignores_the_scale_of_the_compression(which, monkeypatch):
    """With the norm on, scaling W_DKV (or W_DQ) by a > 0 changes no output:
    the norm removes it before anything downstream sees the latent."""
    monkeypatch.setattr(om, "RMS_EPS", 0.0)
    W = _with_gains(rand_weights(SMALL, 33), SMALL, 33)
    h = rand_h(SMALL, 6, 33)
    W2 = dict(W)
    W2[which] = np.asarray(W[which]) * 5.5
    assert np.allclose(om.decode_absorbed(W2, h, SMALL), om.decode_absorbed(W, h, SMALL), rtol=1e-11, atol=1e-13)
    assert np.allclose(om.prefill_unabsorbed(W2, h, SMALL), om.prefill_unabsorbed(W, h, SMALL), rtol=1e-11, atol=1e-13)
    # without gains the same scaling does change the output
    W.pop("g_kv"), W.pop("g_q"), W2.pop("g_kv"), W2.pop("g_q")
    assert not np.allclose(om.decode_absorbed(W2, h, SMALL), om.decode_absorbed(W, h, SMALL), rtol=1e-6)


def test_absorbed_and_unabsorbed_agree_with_the_norm():
    W = _with_gains(rand_weights(SMALL, 34), SMALL, 34)
    h = rand_h(SMALL, 7, 34)
    a = om.decode_absorbed(W, h, SMALL)
    b = om.decode_unabsorbed(W, h, SMALL)
    assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))


_ORIG = om.rmsnorm

MUTANTS = {
    "eps_outside_sqrt": lambda x, g, eps=None: np.asarray(x, float) / (np.sqrt(np.mean(np.asarray(x, float) ** 2, axis=-1, keepdims=True)) + (om.RMS_EPS if eps is None else eps)) * g,
    "norm_without_gain": lambda x, g, eps=None: _ORIG(x, np.ones_like(np.asarray(g, float)), eps),
    "std_instead_of_rms": lambda x, g, eps=None: (np.asarray(x, float) - np.mean(x, axis=-1, keepdims=True)) / np.sqrt(np.var(x, axis=-1, keepdims=True) + (om.RMS_EPS if eps is None else eps)) * g,
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(om, "rmsnorm", MUTANTS[name])
    with pytest.raises(AssertionError):
        test_rmsnorm_matches_brute_force()


def test_gains_move_v2_decode_by_more_than_the_gpu_gate():
    """At DeepSeek-V2 dims, RMSNorm with gains in [0.5, 1.5) changes u by
    several times the GPU parity gate (1e-2 of max|u|), so the GPU RMSNorm
    tests cannot pass with the norm skipped."""
    import synth
    p = synth.preset("v2")
    W = synth.weights(p)
    rng = np.random.default_rng(17)
    Wg = dict(W, g_kv=synth.round_bf16((0.5 + rng.random(p.dims.d_c)).astype(np.float32)),
              g_q=synth.round_bf16((0.5 + rng.random(p.dims.d_cq)).astype(np.float32)))
    h = synth.hidden(p, 2, 700)
    a = om.decode_absorbed(Wg, h, p.dims)
    b = om.decode_absorbed(W, h, p.dims)
    assert np.max(np.abs(a - b)) > 5e-2 * np.max(np.abs(a))
