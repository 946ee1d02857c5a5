"""Pins of the low-bit latent-cache oracle (oracle/lowbit.py).

The element formats are checked against the constants published for the OCP
8-bit (E5M2, E4M3) and 6-bit (E3M2, E2M3) floats, against a brute-force
nearest-value search written independently of the encoder, and against
invariants (monotone code order, exact round trips, the half-spacing error
bound, the per-row scale rule).  Planted mistakes at the end check that
these pins catch the plausible slips in such an encoder.
"""
import math

import numpy as np
import pytest

from oracle import lowbit as lb
from oracle import mla as om
from tests.test_oracle_pins import SMALL, rand_h, rand_weights

# Published constants: (largest finite, smallest normal, largest subnormal,
# smallest subnormal, count of non-negative finite values including zero)
PUBLISHED = {
    "e5m2": (57344.0, 2.0 ** -14, 0.75 * 2.0 ** -14, 2.0 ** -16, 124),
    "e4m3": (448.0, 2.0 ** -6, 0.875 * 2.0 ** -6, 2.0 ** -9, 127),
    "e3m2": (28.0, 0.25, 0.1875, 0.0625, 32),
    "e2m3": (7.5, 1.0, 0.875, 0.125, 32),
}
FMTS = sorted(PUBLISHED)


def _positive_finite(fmt):
    E, M, _ = lb.FORMATS[fmt]
    v = lb.code_values(fmt)[: 1 << (E + M)]
    return v[np.isfinite(v)]


@pytest.mark.parametrize("fmt", FMTS)
def test_published_constants(fmt):
    top, min_norm, max_sub, min_sub, count = PUBLISHED[fmt]
    E, M, bias = lb.FORMATS[fmt]
    v = _positive_finite(fmt)
    assert lb.max_finite(fmt) == top
    assert v.size == count
    assert v[0] == 0.0 and v[1] == min_sub
    # the subnormals are the codes with exponent field 0
    assert v[(1 << M) - 1] == max_sub and v[1 << M] == min_norm


@pytest.mark.parametrize("fmt", FMTS)
def test_codes_are_monotone_and_symmetric(fmt):
    E, M, _ = lb.FORMATS[fmt]
    vals = lb.code_values(fmt)
    half = 1 << (E + M)
    pos = vals[:half]
    fin = np.isfinite(pos)
    assert np.all(np.diff(pos[fin]) > 0)
    neg = vals[half:]
    assert np.array_equal(np.isfinite(neg), fin)
    assert np.array_equal(neg[fin], -pos[fin])


@pytest.mark.parametrize("fmt", FMTS)
def test_every_finite_code_round_trips(fmt):
    vals = lb.code_values(fmt)
    codes = np.nonzero(np.isfinite(vals))[0]
    x = vals[codes].copy()
    x[codes == (1 << (sum(lb.FORMATS[fmt][:2])))] = -0.0   # the negative-zero code carries a sign
    assert np.array_equal(lb.encode(x, fmt).astype(np.int64), codes)


def _brute_nearest(x, fmt):
    """Nearest finite code by scanning every code; ties to the code whose last bit is 0."""
    vals = lb.code_values(fmt)
    out = []
    for xi in x:
        best, best_d = None, math.inf
        for c, v in enumerate(vals):
            if not math.isfinite(v) or (v == 0 and math.copysign(1, v) != math.copysign(1, xi)):
                continue
            d = abs(xi - v)
            if d < best_d or (d == best_d and (c & 1) == 0):
                best, best_d = c, d
        out.append(best)
    return np.array(out)


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_matches_brute_force(fmt):
    rng = np.random.default_rng(FMTS.index(fmt))
    top = lb.max_finite(fmt)
    pos = _positive_finite(fmt)
    mids = (pos[1:] + pos[:-1]) / 2                       # exact ties
    x = np.concatenate([
        rng.uniform(-top, top, 400),
        np.exp2(rng.uniform(math.log2(pos[1]) - 2, math.log2(top), 400)) * rng.choice([-1, 1], 400),
        mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf),
    ])
    x = x[x != 0]
    assert np.array_equal(lb.encode(x, fmt).astype(np.int64), _brute_nearest(x, fmt))


@pytest.mark.parametrize("fmt", FMTS)
def test_magnitudes_above_the_top_take_it(fmt):
    top = lb.max_finite(fmt)
    got = lb.decode(lb.encode(np.array([top * 1.01, top * 1e6, -top * 3]), fmt), fmt)
    assert np.array_equal(got, [top, top, -top])


@pytest.mark.parametrize("fmt", FMTS)
def test_row_scale_rule(fmt):
    top = lb.max_finite(fmt)
    rng = np.random.default_rng(7)
    amax = np.concatenate([np.exp2(rng.uniform(-40, 40, 500)), top * np.exp2(np.arange(-20, 21.0)),
                           np.exp2(np.arange(-30, 31.0))])
    k = lb.row_scale_exp(amax, fmt)
    y = np.ldexp(amax, -k)
    assert np.all(y <= top) and np.all(y > top / 2)        # the smallest power of two that fits
    assert lb.row_scale_exp(np.array([0.0]), fmt)[0] == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_error_is_half_a_spacing(fmt):
    E, M, bias = lb.FORMATS[fmt]
    rng = np.random.default_rng(11)
    x = rng.standard_normal((64, 96)) * np.exp2(rng.uniform(-20, 20, (64, 1)))
    codes, k = lb.quantize_rows(x, fmt)
    got = lb.dequantize_rows(codes, k, fmt)
    y = np.ldexp(x, -k[:, None])
    e = np.maximum(np.floor(np.log2(np.maximum(np.abs(y), 1e-300))), 1 - bias)
    assert np.all(np.abs(y - np.ldexp(got, -k[:, None])) <= np.exp2(e - M) / 2)
    # the row maximum keeps the format's full precision: it is a normal value
    assert np.all(np.max(np.abs(np.ldexp(got, -k[:, None])), axis=1) >= 2.0 ** (1 - bias))


@pytest.mark.parametrize("fmt", FMTS)
def test_rows_on_the_grid_are_stored_exactly(fmt):
    rng = np.random.default_rng(5)
    vals = lb.code_values(fmt)
    ok = np.nonzero(np.isfinite(vals))[0]
    codes = rng.choice(ok, (8, 40))
    codes[:, 0] = np.argmax(np.where(np.isfinite(vals), vals, -np.inf))   # each row holds the top value
    k = rng.integers(-10, 10, 8)
    x = lb.dequantize_rows(codes, k, fmt)
    c2, k2 = lb.quantize_rows(x, fmt)
    assert np.array_equal(lb.dequantize_rows(c2, k2, fmt), x)


def test_store_rows_keeps_k_r_in_bf16_by_default():
    rng = np.random.default_rng(3)
    c, r = rng.standard_normal((5, 12)), rng.standard_normal((5, 4))
    cs, rs = lb.store_rows(c, r, "e4m3")
    assert np.array_equal(rs, om.round_bf16_f64(r))
    cs2, rs2 = lb.store_rows(c, r, "e4m3", "e4m3")
    assert np.array_equal(cs2, cs) and not np.array_equal(rs2, rs)


def test_decode_error_halves_per_mantissa_bit():
    """With a per-row scale the element's mantissa width sets the error of the
    decode: over a dozen draws the 3-bit-mantissa formats (e4m3, e2m3) land
    about twice as close to the exact decode as the 2-bit ones (e5m2, e3m2),
    as halving the grid spacing predicts."""
    dims = SMALL
    errs = {f: [] for f in FMTS}
    for seed in range(30, 42):
        W = rand_weights(dims, seed)
        h = rand_h(dims, 9, seed)
        ref = om.decode_unabsorbed(W, h, dims)
        for f in FMTS:
            errs[f].append(np.mean(np.abs(lb.decode_lowbit(W, h, dims, f) - ref)) / np.max(np.abs(ref)))
    med = {f: float(np.median(v)) for f, v in errs.items()}
    assert med["e4m3"] < 0.7 * med["e3m2"] and med["e2m3"] < 0.7 * med["e5m2"]
    assert med["e4m3"] > 0.3 * med["e3m2"]


# ---------------------------------------------------------------- planted mistakes

def _enc_ties_away(x, fmt):
    E, M, bias = lb.FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), 1 - bias)
    q = np.floor(a / np.exp2(e - M) + 0.5) * np.exp2(e - M)
    return _ORIG_ENCODE(np.copysign(np.minimum(q, lb.max_finite(fmt)), x), fmt)


def _enc_truncate(x, fmt):
    E, M, bias = lb.FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), 1 - bias)
    q = np.floor(a / np.exp2(e - M)) * np.exp2(e - M)
    return _ORIG_ENCODE(np.copysign(np.minimum(q, lb.max_finite(fmt)), x), fmt)


def _enc_flush_subnormals(x, fmt):
    E, M, bias = lb.FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    return _ORIG_ENCODE(np.where(np.abs(x) < 2.0 ** (1 - bias), 0.0 * x, x), fmt)


_ORIG_ENCODE = lb.encode
_ORIG_SCALE = lb.row_scale_exp

MUTANTS = {
    "ties_away_from_zero": ("encode", _enc_ties_away, "test_encode_matches_brute_force"),
    "truncation": ("encode", _enc_truncate, "test_encode_matches_brute_force"),
    "subnormals_flushed": ("encode", _enc_flush_subnormals, "test_encode_matches_brute_force"),
    "scale_one_too_large": ("row_scale_exp", lambda a, f: _ORIG_SCALE(a, f) + 1, "test_row_scale_rule"),
    "scale_from_floor": ("row_scale_exp", lambda a, f: np.floor(np.log2(np.maximum(np.asarray(a, float), 1e-300)
                                                                      / lb.max_finite(f))).astype(np.int64) * (np.asarray(a) > 0),
                         "test_row_scale_rule"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn, pin = MUTANTS[name]
    monkeypatch.setattr(lb, attr, fn)
    with pytest.raises(AssertionError):
        for fmt in FMTS:
            globals()[pin](fmt)


@pytest.mark.parametrize("preset,L", [("tiny", 40), ("v2", 90)])
def test_absorbed_lowbit_equals_unabsorbed_lowbit(preset, L):
    """The absorbed form over low-bit rows equals the un-absorbed one (the
    absorption identity of App. C holds for whatever rows are cached), so the
    long GPU parity cases may use the cheaper form."""
    import synth
    p = synth.preset(preset)
    W = synth.weights(p)
    h = synth.hidden(p, 1, L + 1)
    for fmt in ("e4m3", "e5m2"):
        a = lb.decode_lowbit(W, h, p.dims, fmt, absorbed=True)
        b = lb.decode_lowbit(W, h, p.dims, fmt)
        assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))
