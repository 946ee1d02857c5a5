"""mla_decode_static: the decode entry point that allocates nothing.

Some callers cannot allocate device memory when they call the library (an
engine plugin handed only its input and output buffers, a latency-critical
path where cudaMalloc may synchronise the device), so they cannot pass a
workspace.  This variant keeps its scratch in a static device array inside the
library.  Here it is called through the C ABI twice in a row (the second call
finds the first call's leftovers in the shared array) and each result is
checked against mla_decode, which uses a caller-owned workspace: bit for bit
(both run the same kernels with the same plans) and within the tolerance of
the other decode tests.  The batch limit of the array is exercised at its
edge.  The file is named so that pytest collects it last.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import synth  # noqa: E402
from tests import gpu_util as gu  # noqa: E402


def _setup(m, preset, L):
    from mla_latent_kv_47_b200.cache import LatentCache
    p = synth.preset(preset)
    d = p.dims
    dims = m.make_dims(d)
    _, Wd = gu.device_weights(p)
    wts = m.make_weights(Wd)
    cache = LatentCache(dims, [x + 1 for x in L])
    ws = m.alloc_workspace(dims, len(L), 1)
    gu.fill_cache(m, dims, Wd, cache, ws, {}, L, p, gen_seed=7)
    tdt = torch.float32 if d.dtype == "fp32" else torch.bfloat16
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    h = torch.randn((len(L), d.d_model), generator=g, device="cuda").to(tdt)
    seqlen = torch.tensor(L, dtype=torch.int32, device="cuda")
    return dims, wts, Wd, cache, ws, h, seqlen


def _run_both(m, dims, wts, cache, ws, h, seqlen, B):
    """u from mla_decode (caller's workspace), then two mla_decode_static calls
    in a row; returns the three outputs."""
    d_model = dims.d_model
    u_ref = torch.empty((B, d_model), dtype=torch.float32, device="cuda")
    m.decode(dims, wts, h, cache.handle, seqlen, u_ref, ws)
    assert m.device_status(ws) == (0, 0)
    outs = []
    for _ in range(2):  # two calls in a row share (and reuse) the static scratch
        u = torch.full((B, d_model), float("nan"), dtype=torch.float32, device="cuda")
        m.decode_static(dims, wts, h, cache.handle, seqlen, u)
        torch.cuda.synchronize()
        outs.append(u)
    return u_ref, outs


@pytest.mark.parametrize("preset,L", [("v2", [0, 63, 64, 700, 3000]), ("lite", [5, 1000, 4096]), ("tiny", [64])])
def test_static_decode_matches_workspace_decode(preset, L):
    """Both entry points run the same kernels in the same order with the same
    split-K and split-KV plans, so the results are equal bit for bit; a
    leftover from the previous call in the shared array would show here."""
    import mla_latent_kv_47_b200 as m
    dims, wts, Wd, cache, ws, h, seqlen = _setup(m, preset, L)  # Wd keeps the weights alive
    u_ref, outs = _run_both(m, dims, wts, cache, ws, h, seqlen, len(L))
    ref = u_ref.cpu().numpy().astype(np.float64)
    for u in outs:
        assert torch.equal(u, u_ref)
        gu.assert_gate(gu.gate(u.cpu().numpy().astype(np.float64), ref))


def _static_code(m, dims, wts, cache, h, seqlen, u, B):
    import ctypes
    return m.lib.mla_decode_static(ctypes.byref(dims), ctypes.byref(wts), h.data_ptr(), B,
                                   ctypes.byref(cache.handle), seqlen.data_ptr(), u.data_ptr(), None)


def test_static_decode_at_the_headline_batch_and_at_its_limit():
    """DeepSeek-V2 dims at batch 64 and at the largest batch the static array
    holds on this GPU (found by asking: a batch beyond the array is refused on
    the host with MLA_ERR_WORKSPACE before anything is enqueued), both equal
    to mla_decode bit for bit; one sequence more is refused."""
    import mla_latent_kv_47_b200 as m
    n_max = 512
    L = [(7 * b) % 97 for b in range(n_max)]
    dims, wts, Wd, cache, ws, h, seqlen = _setup(m, "v2", L)
    u = torch.empty((n_max, dims.d_model), dtype=torch.float32, device="cuda")
    assert _static_code(m, dims, wts, cache, h, seqlen, u, n_max) == -4
    lo, hi = 64, n_max          # lo fits (checked below), hi does not
    assert _static_code(m, dims, wts, cache, h, seqlen, u, lo) == 0
    while hi - lo > 1:
        mid = (lo + hi) // 2
        code = _static_code(m, dims, wts, cache, h, seqlen, u, mid)
        assert code in (0, -4), code
        lo, hi = (mid, hi) if code == 0 else (lo, mid)
    torch.cuda.synchronize()
    assert lo >= 64
    for B in (64, lo):
        u_ref, outs = _run_both(m, dims, wts, cache, ws, h[:B], seqlen[:B], B)
        for out in outs:
            assert torch.equal(out, u_ref), B
    assert _static_code(m, dims, wts, cache, h, seqlen, u, lo + 1) == -4
    torch.cuda.synchronize()
