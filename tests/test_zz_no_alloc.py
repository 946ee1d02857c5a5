"""mla_decode_static: the decode entry point that allocates nothing.

Some callers cannot allocate device memory when they call the library (an
engine plugin handed only its input and output buffers, a latency-critical
path where cudaMalloc may synchronise the device), so they cannot pass a
workspace.  This variant keeps its scratch in a static device array inside the
library.  Here it is called through the C ABI twice in a row (the second call
finds the first call's leftovers in the shared array) and each result is
checked against mla_decode, which uses a caller-owned workspace, with the
tolerance of the other decode tests.  The file is named so that pytest
collects it last.
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


@pytest.mark.parametrize("preset,L", [("v2", [0, 63, 64, 700, 3000]), ("lite", [5, 1000, 4096]), ("tiny", [64])])
def test_static_decode_matches_workspace_decode(preset, L):
    import mla_latent_kv_47_b200 as m
    dims, wts, Wd, cache, ws, h, seqlen = _setup(m, preset, L)  # Wd keeps the weights alive
    d_model = dims.d_model
    u_ref = torch.empty((len(L), d_model), dtype=torch.float32, device="cuda")
    m.decode(dims, wts, h, cache.handle, seqlen, u_ref, ws)
    assert m.device_status(ws) == (0, 0)
    ref = u_ref.cpu().numpy().astype(np.float64)
    for _ in range(2):  # two calls in a row share (and reuse) the static scratch
        u = torch.full((len(L), d_model), float("nan"), dtype=torch.float32, device="cuda")
        m.decode_static(dims, wts, h, cache.handle, seqlen, u)
        torch.cuda.synchronize()
        got = u.cpu().numpy().astype(np.float64)
        stats = gu.gate(got, ref)
        gu.assert_gate(stats)


def test_static_decode_rejects_a_batch_beyond_its_scratch():
    import ctypes
    import mla_latent_kv_47_b200 as m
    dims, wts, Wd, cache, ws, h, seqlen = _setup(m, "v2", [10, 20])
    u = torch.empty((2, dims.d_model), dtype=torch.float32, device="cuda")
    # a batch of 4096 needs far more than the static array: refused before any launch
    code = m.lib.mla_decode_static(ctypes.byref(dims), ctypes.byref(wts), h.data_ptr(), 4096,
                                   ctypes.byref(cache.handle), seqlen.data_ptr(), u.data_ptr(), None)
    assert code == -4
    torch.cuda.synchronize()
