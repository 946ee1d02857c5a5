"""Pins of the fp64 oracle to facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: the
cache-size figures printed on the pages, an independent pure-Python brute
force, closed forms, invariants of softmax and RoPE, and library routines the
special cases reduce to.  The mutation tests at the end plant typical mistakes
in the oracle and check that a pin catches each of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import mla as om
from synth import Dims, PRESETS, ragged_lengths, round_bf16, to_bf16_bits, bf16_bits_to_f32
from tests import bruteforce_mla as bf

HERE = os.path.dirname(os.path.abspath(__file__))

SMALL = Dims(d_model=8, n_h=2, d_h=4, d_R=4, d_c=6, d_cq=5, rope_base=100.0, dtype="fp32")
SMALL_NOQ = Dims(d_model=8, n_h=3, d_h=4, d_R=2, d_c=6, d_cq=0, rope_base=50.0, dtype="fp32")


def rand_weights(dims, seed, std=0.3):
    from synth import weight_shapes
    rng = np.random.default_rng(seed)
    return {k: rng.standard_normal(s) * std for k, s in weight_shapes(dims).items()}


def rand_h(dims, n, seed):
    return np.random.default_rng(seed + 1000).standard_normal((n, dims.d_model))


# ---------------------------------------------------------------- pages' figures

def test_cache_row_is_4p5_dh_and_gqa_2p25_groups():
    """§2.1.4: MLA caches (d_c + d_R) per token per layer = 4.5 d_h, i.e. the
    cache of GQA with 2.25 groups (GQA caches 2 n_g d_h: keys and values)."""
    g = json.load(open(os.path.join(HERE, "golden", "page_dims.json")))
    for name in ("v2", "lite"):
        d = g[name]
        row = om.cache_row_elems(d["d_c"], d["d_R"])
        assert row == 576
        assert row == 4.5 * d["d_h"]
        assert row == 2 * g["gqa_equivalent_groups"] * d["d_h"]
    for p in PRESETS.values():
        assert p.dims.row_elems == om.cache_row_elems(p.dims.d_c, p.dims.d_R)


def test_presets_match_page_dims():
    g = json.load(open(os.path.join(HERE, "golden", "page_dims.json")))
    for name, key in (("v2", "v2"), ("lite", "lite")):
        d = PRESETS[name].dims
        for f in ("d_model", "n_h", "d_h", "d_c", "d_cq", "d_R"):
            assert getattr(d, f) == g[key][f], (name, f)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("dims", [SMALL, SMALL_NOQ], ids=["qcomp", "noqcomp"])
def test_bruteforce_4_tokens(dims):
    """The numpy oracle equals an independent pure-Python brute force."""
    W = rand_weights(dims, 1)
    h = rand_h(dims, 4, 1)
    for t in range(4):
        ref = np.array(bf.mla_token_output(W, h.tolist(), t, dims))
        u = om.decode_unabsorbed(W, h[: t + 1], dims)
        assert np.max(np.abs(u - ref)) <= 1e-13 * max(1.0, np.max(np.abs(ref)))
    up = om.prefill_unabsorbed(W, h, dims)
    for t in range(4):
        ref = np.array(bf.mla_token_output(W, h.tolist(), t, dims))
        assert np.max(np.abs(up[t] - ref)) <= 1e-13 * max(1.0, np.max(np.abs(ref)))


# ---------------------------------------------------------------- absorption identity

@pytest.mark.parametrize("dims,L", [(SMALL, 9), (SMALL_NOQ, 7), (PRESETS["tiny"].dims, 64)])
def test_absorbed_equals_unabsorbed(dims, L):
    """App. C: absorbing W^{UK} into the query and W^{UV} into the output is exact."""
    W = rand_weights(dims, 2, std=0.2)
    h = rand_h(dims, L + 1, 2)
    u0 = om.decode_unabsorbed(W, h, dims)
    u1 = om.decode_absorbed(W, h, dims)
    assert np.max(np.abs(u0 - u1)) <= 1e-12 * np.max(np.abs(u0))


@pytest.mark.parametrize("preset,L", [("v2", 100), ("ragged", 40)])
def test_absorbed_equals_unabsorbed_at_v2_dims(preset, L):
    """The absorbed form, which the long ragged parity cases are checked
    against, equals the un-absorbed App. C form at the DeepSeek-V2 dims and
    with the presets' own weights and hidden states, not only on small
    layers."""
    import synth
    p = synth.preset(preset)
    W = synth.weights(p)
    h = synth.hidden(p, 3, L + 1)
    u0 = om.decode_unabsorbed(W, h, p.dims)
    u1 = om.decode_absorbed(W, h, p.dims)
    assert np.max(np.abs(u0 - u1)) <= 1e-12 * np.max(np.abs(u0))


def test_softmax_rows_sum_to_one():
    dims = PRESETS["tiny"].dims
    W = rand_weights(dims, 3, std=0.3)
    h = rand_h(dims, 40, 3)
    _, parts = om.decode_absorbed(W, h, dims, return_parts=True)
    p = parts["p"]
    assert np.all(p >= 0)
    assert np.max(np.abs(p.sum(axis=-1) - 1.0)) <= 1e-15 * p.shape[-1]
    s = np.random.default_rng(0).standard_normal((5, 33)) * 30
    assert np.max(np.abs(om.softmax(s).sum(-1) - 1)) < 1e-15 * 33


# ---------------------------------------------------------------- closed forms

def test_single_token_closed_form():
    """With nothing cached the softmax is 1, so u = W^O blockdiag(W^{UV}) c^KV_new."""
    dims = SMALL
    W = rand_weights(dims, 4)
    h = rand_h(dims, 1, 4)
    c = [sum(W["W_DKV"][r][k] * h[0][k] for k in range(dims.d_model)) for r in range(dims.d_c)]
    o = [sum(W["W_UV"][r][k] * c[k] for k in range(dims.d_c)) for r in range(dims.n_h * dims.d_h)]
    u_ref = [sum(W["W_O"][r][k] * o[k] for k in range(len(o))) for r in range(dims.d_model)]
    u = om.decode_unabsorbed(W, h, dims)
    assert np.max(np.abs(u - np.array(u_ref))) <= 1e-13


def test_uniform_attention_closed_form():
    """W^{QR} = W^{KR} = 0 and identical h_j: every score is equal, p = 1/(L+1),
    and u equals the single-token value."""
    dims = SMALL
    W = rand_weights(dims, 5)
    W["W_QR"] = np.zeros_like(W["W_QR"])
    W["W_KR"] = np.zeros_like(W["W_KR"])
    h1 = rand_h(dims, 1, 5)
    h = np.repeat(h1, 12, axis=0)
    _, parts = om.decode_absorbed(W, h, dims, return_parts=True)
    assert np.max(np.abs(parts["p"] - 1.0 / 12)) < 1e-15
    assert np.max(np.abs(om.decode_unabsorbed(W, h, dims) - om.decode_unabsorbed(W, h1, dims))) < 1e-13


def test_mha_special_case_matches_library_attention():
    """W^{QR} = 0 removes the rotary score term: MLA is then textbook multi-head
    attention over the up-projected keys/values, with scale 1/sqrt(d_h + d_R)."""
    torch = pytest.importorskip("torch")
    dims = SMALL
    W = rand_weights(dims, 6)
    W["W_QR"] = np.zeros_like(W["W_QR"])
    L1 = 10
    h = rand_h(dims, L1, 6)
    c_q = h @ W["W_DQ"].T
    q = (c_q[-1] @ W["W_UQ"].T).reshape(dims.n_h, 1, dims.d_h)
    c = h @ W["W_DKV"].T
    k = (c @ W["W_UK"].T).reshape(L1, dims.n_h, dims.d_h).transpose(1, 0, 2)
    v = (c @ W["W_UV"].T).reshape(L1, dims.n_h, dims.d_h).transpose(1, 0, 2)
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        scale=1.0 / math.sqrt(dims.d_h + dims.d_R)).numpy()
    u_ref = W["W_O"] @ o.reshape(-1)
    assert np.max(np.abs(om.decode_unabsorbed(W, h, dims) - u_ref)) < 1e-13


# ---------------------------------------------------------------- RoPE

def test_rope_explicit_values():
    """d_R = 4, base 100: pair 0 turns by pos rad, pair 1 by pos/10 rad."""
    x = np.array([1.0, 2.0, 3.0, -4.0])
    y = om.rope(x, 3, 100.0)
    c0, s0, c1, s1 = math.cos(3), math.sin(3), math.cos(0.3), math.sin(0.3)
    ref = [1 * c0 - 2 * s0, 1 * s0 + 2 * c0, 3 * c1 + 4 * s1, 3 * s1 - 4 * c1]
    assert np.max(np.abs(y - ref)) < 1e-15


def test_rope_invariants():
    rng = np.random.default_rng(7)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    assert np.allclose(om.rope(q, 0, 10000.0), q, atol=0)
    for pos in (1, 77, 131071):
        assert abs(np.linalg.norm(om.rope(q, pos, 10000.0)) - np.linalg.norm(q)) < 1e-12
    # the score depends only on the position difference
    a = om.rope(q, 1000, 10000.0) @ om.rope(k, 990, 10000.0)
    b = om.rope(q, 130010, 10000.0) @ om.rope(k, 130000, 10000.0)
    assert abs(a - b) < 1e-9


def test_shift_invariance_of_decode_scores():
    """Shifting every position by the same amount leaves the scores unchanged:
    RoPE_m(q).RoPE_n(k) depends only on m - n."""
    dims = SMALL
    W = rand_weights(dims, 8)
    h = rand_h(dims, 6, 8)
    pos = np.arange(6.0)
    c, kr = om.latent_rows(W, h, pos, dims)
    c2, kr2 = om.latent_rows(W, h, pos + 500, dims)
    qc, qr = om.queries(W, h[-1:], pos[-1:], dims)
    qc2, qr2 = om.queries(W, h[-1:], pos[-1:] + 500, dims)
    s1 = np.einsum("hd,jd->hj", qr[0], kr)
    s2 = np.einsum("hd,jd->hj", qr2[0], kr2)
    assert np.max(np.abs(s1 - s2)) < 1e-12


# ---------------------------------------------------------------- invariances

def test_prefill_row_equals_decode():
    dims = SMALL
    W = rand_weights(dims, 9)
    h = rand_h(dims, 7, 9)
    up = om.prefill_unabsorbed(W, h, dims)
    for t in range(7):
        assert np.max(np.abs(up[t] - om.decode_unabsorbed(W, h[: t + 1], dims))) < 1e-13
    # a prefill on top of a cached prefix gives the same rows
    up2 = om.prefill_unabsorbed(W, h[3:], dims, start_pos=3, h_prefix=h[:3])
    assert np.max(np.abs(up2 - up[3:])) < 1e-13


def test_permuting_cached_rows_does_not_change_u():
    dims = SMALL
    W = rand_weights(dims, 10)
    h = rand_h(dims, 9, 10)
    pos = np.arange(9.0)
    c, kr = om.latent_rows(W, h, pos, dims)
    perm = np.random.default_rng(1).permutation(9)
    u0 = om.decode_unabsorbed(W, h, dims, cache_rows=(c, kr))
    u1 = om.decode_unabsorbed(W, h, dims, cache_rows=(c[perm], kr[perm]))
    assert np.max(np.abs(u0 - u1)) < 1e-13


# ---------------------------------------------------------------- rounding helpers

def test_round_bf16_f64_matches_library_conversion():
    """On fp32-exact inputs the library's bf16 conversion rounds once, so it is
    the reference; ties must go to the even significand."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(11)
    x32 = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ref32 = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(om.round_bf16_f64(x32.astype(np.float64)), ref32.astype(np.float64))
    assert np.array_equal(round_bf16(x32), ref32)
    assert np.array_equal(bf16_bits_to_f32(to_bf16_bits(x32)), ref32)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert om.round_bf16_f64(1.0 + 2.0 ** -8) == 1.0
    assert om.round_bf16_f64(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    # just above the tie rounds up (fp64 keeps bits an fp32 step would drop)
    assert om.round_bf16_f64(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7


def test_ragged_lengths_draw():
    L = ragged_lengths(0)
    assert L.sum() == 2_007_088 and L.max() == 126_832 and np.median(L) == 679
    assert L.min() >= 1 and (L == 1).sum() == 11


def test_hidden_subset_regenerates():
    from synth import hidden
    p = PRESETS["lite"]
    a = hidden(p, 3, 700)
    b = hidden(p, 3, 300, first=400)
    assert np.array_equal(a[400:], b)
    assert not np.array_equal(hidden(p, 4, 10), a[:10])


# ---------------------------------------------------------------- planted mistakes

_ORIG_ROPE = om.rope


def _rope_half_split(x, pos, base, theta=None):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    perm = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])
    inv = np.argsort(perm)
    xi = np.empty_like(x)
    xi[..., 0::2] = x[..., : d // 2]
    xi[..., 1::2] = x[..., d // 2:]
    y = _ORIG_ROPE(xi, pos, base, theta)
    out = np.empty_like(y)
    out[..., : d // 2] = y[..., 0::2]
    out[..., d // 2:] = y[..., 1::2]
    return out


MUTANTS = {
    "rope_direction": ("rope", lambda x, pos, base, theta=None: _ORIG_ROPE(x, -np.asarray(pos, dtype=np.float64), base, theta)),
    "rope_half_split": ("rope", _rope_half_split),
    "rope_frequency": ("rope", lambda x, pos, base, theta=None: _ORIG_ROPE(x, pos, base * 2, theta)),
    "scale_dh_only": ("attend", lambda q, k, v, scale: _ORIG_ATTEND(q, k, v, scale * math.sqrt((4 + 4) / 4))),
    "no_rope_key": ("keys_values", lambda W, c, kr, dims: _ORIG_KV(W, c, kr * 0, dims)),
    "uk_row_order": ("keys_values", lambda W, c, kr, dims: _ORIG_KV(
        dict(W, W_UK=np.asarray(W["W_UK"]).reshape(dims.n_h, dims.d_h, dims.d_c)[:, ::-1, :].reshape(-1, dims.d_c)), c, kr, dims)),
    "softmax_unnormalised": ("softmax", lambda s, axis=-1: np.exp(np.asarray(s) - np.max(s, axis=axis, keepdims=True))),
}
_ORIG_ATTEND = om.attend
_ORIG_KV = om.keys_values


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(om, attr, fn)
    dims = SMALL
    W = rand_weights(dims, 13)
    h = rand_h(dims, 4, 13)
    ref = np.array(bf.mla_token_output(W, h.tolist(), 3, dims))
    u = om.decode_unabsorbed(W, h, dims)
    assert np.max(np.abs(u - ref)) > 1e-6, f"mutant {name} went unnoticed"


def test_prefill_row_subset_matches_full():
    dims = SMALL
    W = rand_weights(dims, 14)
    h = rand_h(dims, 6, 14)
    full = om.prefill_unabsorbed(W, h, dims)
    part = om.prefill_unabsorbed(W, h, dims, rows=[5, 0, 3])
    assert np.array_equal(part, full[[5, 0, 3]])
