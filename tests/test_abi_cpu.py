"""CPU checks of the C ABI: the library loads without a GPU, exports every entry
point declared in include/mla.h, and rejects bad arguments on the host before
anything is enqueued."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def m():
    from mla_latent_kv_47_b200 import build
    build.build()
    import mla_latent_kv_47_b200 as mod
    return mod


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(m):
    names = declared_functions()
    assert len(names) >= 7
    for n in names:
        assert hasattr(m.lib, n), n
    assert set(m.EXPORTS) == set(names)


def test_status_strings(m):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert m.status_string(code) and m.status_string(code) != "unknown status"
    assert m.status_string(-99) == "unknown status"


def test_workspace_sizes(m):
    import synth
    for name, p in synth.PRESETS.items():
        dims = m.make_dims(p.dims)
        n = m.workspace_bytes(dims, p.batch, p.prefill_T or 1)
        assert n > 0
        for which in range(5):
            off = m.workspace_offset(dims, p.batch, which)
            assert 0 < off < n and off % 256 == 0
        assert m.workspace_offset(dims, p.batch, 7) == 2 ** 64 - 1
    bad = m.make_dims(synth.PRESETS["v2"].dims)
    bad.d_R = 63
    assert m.workspace_bytes(bad, 4, 4) == 0
    bad = m.make_dims(synth.PRESETS["v2"].dims)
    bad.dtype = 7
    assert m.workspace_bytes(bad, 4, 4) == 0


def test_decode_workspace_grows_with_batch(m):
    import synth
    dims = m.make_dims(synth.PRESETS["v2"].dims)
    assert m.workspace_bytes(dims, 128, 1) > m.workspace_bytes(dims, 64, 1)
    # prefill region is sized by the key tokens
    assert m.workspace_bytes(dims, 1, 16384) > m.workspace_bytes(dims, 1, 1024)


def _call_decode(m, dims, weights, h, B, cache, seqlen, u, ws, nbytes):
    return m.lib.mla_decode(ctypes.byref(dims) if dims is not None else None,
                            ctypes.byref(weights) if weights is not None else None, h, B,
                            ctypes.byref(cache) if cache is not None else None, seqlen, u, ws, nbytes, None)


def test_host_argument_checks_without_gpu(m):
    """Fake (never dereferenced) device addresses: every case fails a host check."""
    import synth
    dims = m.make_dims(synth.PRESETS["v2"].dims)
    A = 1 << 20  # 16-byte aligned fake address
    W = m.Weights(*[A] * 8)
    C = m.Cache(A, A, None, 1000)
    assert _call_decode(m, None, W, A, 4, C, A, A, A, 1 << 40) == -1
    assert _call_decode(m, dims, None, A, 4, C, A, A, A, 1 << 40) == -1
    assert _call_decode(m, dims, W, A, 0, C, A, A, A, 1 << 40) == -1
    assert _call_decode(m, dims, W, A + 2, 4, C, A, A, A, 1 << 40) == -3
    W_bad = m.Weights(*[A] * 8)
    W_bad.W_UK = A + 8
    assert _call_decode(m, dims, W_bad, A, 4, C, A, A, A, 1 << 40) == -3
    assert _call_decode(m, dims, W, A, 4, m.Cache(A + 4, A, None, 1000), A, A, A, 1 << 40) == -3
    assert _call_decode(m, dims, W, A, 4, m.Cache(A, A, None, 0), A, A, A, 1 << 40) == -1   # n_rows required
    assert _call_decode(m, dims, W, A, 4, C, A, A, None, 1 << 40) == -4
    assert _call_decode(m, dims, W, A, 4, C, A, A, A, 1024) == -4
    assert _call_decode(m, dims, W, A, 4, C, A, A, A + 16, 1 << 40) == -3   # workspace wants 256-byte alignment
    odd = m.make_dims(synth.PRESETS["v2"].dims)
    odd.d_R = 63
    assert _call_decode(m, odd, W, A, 4, C, A, A, A, 1 << 40) == -2
    noq = m.make_dims(synth.PRESETS["v2"].dims)
    W_noq = m.Weights(*[A] * 8)
    W_noq.W_DQ = None
    assert _call_decode(m, noq, W_noq, A, 4, C, A, A, A, 1 << 40) == -1   # d_cq > 0 needs W_DQ


def test_prefill_and_append_argument_checks(m):
    import synth
    dims = m.make_dims(synth.PRESETS["v2"].dims)
    A = 1 << 20
    W = m.Weights(*[A] * 8)
    C = m.Cache(A, A, None, 1000)
    lib = m.lib
    assert lib.mla_prefill(ctypes.byref(dims), ctypes.byref(W), A, 0, 0, ctypes.byref(C), 0, A, A, 1 << 40, None) == -1
    assert lib.mla_prefill(ctypes.byref(dims), ctypes.byref(W), A, 8, -1, ctypes.byref(C), 0, A, A, 1 << 40, None) == -1
    assert lib.mla_prefill(ctypes.byref(dims), ctypes.byref(W), A, 8, 0, ctypes.byref(C), -2, A, A, 1 << 40, None) == -1
    assert lib.mla_cache_append(ctypes.byref(dims), ctypes.byref(W), A, 0, A, A, ctypes.byref(C), A, 1 << 40, None) == 0
    assert lib.mla_cache_append(ctypes.byref(dims), ctypes.byref(W), A, -1, A, A, ctypes.byref(C), A, 1 << 40, None) == -1
    assert lib.mla_cache_append(ctypes.byref(dims), ctypes.byref(W), A, 4, None, A, ctypes.byref(C), A, 1 << 40, None) == -1
    assert lib.mla_get_device_status(None, None, None) == -4


def test_oracle_is_not_reachable_from_the_product():
    """The product package never imports the oracle (it is test infrastructure)."""
    pkg = os.path.join(ROOT, "mla_latent_kv_47_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f


def test_bf16_shapes_outside_the_tensor_core_kernels_are_rejected(m):
    """bf16 storage runs on the tensor-core kernels alone: a bf16 layer of
    another head shape is refused on the host (nothing enqueued, the fake
    device addresses are never touched) instead of running on other kernels."""
    import synth
    A = 1 << 20
    W = m.Weights(*[A] * 8)
    C = m.Cache(A, A, None, 1000)
    base = synth.PRESETS["v2"].dims
    for field, value in (("d_h", 64), ("d_c", 256), ("n_h", 256), ("d_model", 5120 + 32), ("d_cq", 1536 + 32)):
        dims = m.make_dims(base)
        setattr(dims, field, value)
        assert _call_decode(m, dims, W, A, 4, C, A, A, A, 1 << 40) == -2, field
        assert m.lib.mla_prefill(ctypes.byref(dims), ctypes.byref(W), A, 8, 0, ctypes.byref(C), 0, A, A,
                                 1 << 40, None) == -2, field
        assert m.lib.mla_cache_append(ctypes.byref(dims), ctypes.byref(W), A, 4, A, A, ctypes.byref(C), A,
                                      1 << 40, None) == -2, field
        assert m.workspace_bytes(dims, 4, 4) == 0, field
    # the same head shapes in fp32 storage stay on the CUDA-core kernels
    small = m.make_dims(synth.PRESETS["tiny"].dims)
    assert m.workspace_bytes(small, 1, 64) > 0


def test_yarn_arguments_are_checked(m):
    """YaRN is off at yarn_s = 0; otherwise s >= 1, beta > alpha >= 0 and
    L0 > 0 are required (checked on the host, nothing enqueued)."""
    import synth
    A = 1 << 20
    W = m.Weights(*[A] * 8)
    C = m.Cache(A, A, None, 1000)
    ok = m.make_dims(synth.PRESETS["v2"].dims)
    assert m.workspace_bytes(ok, 4, 4) > 0
    for y in ((0.5, 1.0, 32.0, 4096.0), (40.0, 32.0, 1.0, 4096.0), (40.0, 1.0, 32.0, 0.0),
              (40.0, -1.0, 32.0, 4096.0), (float("nan"), 1.0, 32.0, 4096.0)):
        d = m.make_dims(synth.PRESETS["v2"].dims)
        d.yarn_s, d.yarn_alpha, d.yarn_beta, d.yarn_L0 = y
        assert _call_decode(m, d, W, A, 4, C, A, A, A, 1 << 40) == -1, y
    d = m.make_dims(synth.PRESETS["v2"].dims)
    d.yarn_s, d.yarn_alpha, d.yarn_beta, d.yarn_L0 = 40.0, 1.0, 32.0, 4096.0
    assert m.workspace_bytes(d, 4, 4) > 0


def test_paged_cache_arguments_are_checked(m):
    """A block table needs block_size a positive multiple of 64 and
    max_blocks > 0; without one, seq_start is required."""
    import synth
    A = 1 << 20
    W = m.Weights(*[A] * 8, None, None)
    dims = m.make_dims(synth.PRESETS["v2"].dims)
    assert _call_decode(m, dims, W, A, 4, m.Cache(A, None, None, 1000, None, 0, 0), A, A, A, 1 << 40) == -1
    for bs, mb in ((0, 4), (96, 4), (64, 0), (-64, 4)):
        assert _call_decode(m, dims, W, A, 4, m.Cache(A, None, None, 1000, A, bs, mb), A, A, A, 1 << 40) == -1, (bs, mb)
    assert _call_decode(m, dims, W, A, 4, m.Cache(A, None, None, 1000, A + 4, 64, 4), A, A, A, 1 << 40) == -3


def test_rmsnorm_gain_arguments_are_checked(m):
    """g_q needs query compression; gains must be 16-byte aligned."""
    import synth
    A = 1 << 20
    C = m.Cache(A, A, None, 1000, None, 0, 0)
    lite = m.make_dims(synth.PRESETS["lite"].dims)
    assert _call_decode(m, lite, m.Weights(*[A] * 8, None, A), A, 4, C, A, A, A, 1 << 40) == -1
    v2 = m.make_dims(synth.PRESETS["v2"].dims)
    assert _call_decode(m, v2, m.Weights(*[A] * 8, A + 2, None), A, 4, C, A, A, A, 1 << 40) == -3


def test_e4m3_cache_arguments_are_checked(m):
    """The E4M3 cache format needs bf16 storage; mla_prefill does not take it;
    an unknown format is refused."""
    import dataclasses
    import synth
    A = 1 << 20
    W = m.Weights(*[A] * 8, None, None)
    C = m.Cache(A, A, None, 1000, None, 0, 0)
    e4 = m.make_dims(dataclasses.replace(synth.PRESETS["v2"].dims, cache="e4m3"))
    assert e4.cache_format == m.CACHE_E4M3 and m.cache_row_bytes(e4) == 656
    assert m.workspace_bytes(e4, 4, 4) > 0
    assert m.lib.mla_prefill(ctypes.byref(e4), ctypes.byref(W), A, 8, 0, ctypes.byref(C), 0, A, A, 1 << 40, None) == -2
    tiny = m.make_dims(synth.PRESETS["tiny"].dims)
    tiny.cache_format = m.CACHE_E4M3
    assert m.workspace_bytes(tiny, 1, 4) == 0
    bad = m.make_dims(synth.PRESETS["v2"].dims)
    bad.cache_format = 5
    assert _call_decode(m, bad, W, A, 4, C, A, A, A, 1 << 40) == -2


def test_wait_timeout_check_needs_a_workspace(m):
    assert m.lib.mla_check_wait_timeout(None, None) == -4
    assert m.lib.mla_check_wait_timeout((1 << 20) + 16, None) == -3


def test_structs_keep_their_tensors_alive(m, monkeypatch):
    """make_weights / make_cache hand the library raw device pointers; the
    structs they return hold the tensors, so a caller who drops its own
    references (e.g. builds the weight dict inline) leaves no dangling pointer."""
    import gc
    import weakref

    import torch

    monkeypatch.setattr(m, "_ptr", lambda t: None if t is None else 4096)  # no device here
    w_t = torch.zeros(4)
    ref_w = weakref.ref(w_t)
    w = m.make_weights({"W_O": w_t})
    base = torch.zeros(2, 3)
    ss = torch.zeros(1, dtype=torch.int64)
    ref_b, ref_s = weakref.ref(base), weakref.ref(ss)
    c = m.make_cache(base, seq_start=ss)
    del w_t, base, ss
    gc.collect()
    assert ref_w() is not None and ref_b() is not None and ref_s() is not None
    del w, c
    gc.collect()
    assert ref_w() is None and ref_b() is None and ref_s() is None
