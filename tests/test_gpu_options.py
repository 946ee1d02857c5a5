"""GPU parity of the layer's options in combination: the E4M3 cache over a
paged layout, the RMSNorm on c^KV before the E4M3 encoding, and YaRN, RMSNorm
and the E4M3 cache all on at once (decode against the fp64 oracle run with
the same options over the same stored rows)."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import synth  # noqa: E402
from oracle import lowbit as lb  # noqa: E402
from tests import gpu_util as gu  # noqa: E402
from tests.test_gpu_decode import run_decode  # noqa: E402
from tests.test_gpu_rmsnorm import weights_with_gains  # noqa: E402

V2_E4M3 = dataclasses.replace(synth.V2, cache="e4m3")
V2_ALL = dataclasses.replace(synth.V2, cache="e4m3", yarn=(40.0, 1.0, 32.0, 4096.0))


@pytest.fixture(scope="module")
def m():
    import mla_latent_kv_47_b200 as mod
    return mod


def test_e4m3_paged_equals_e4m3_contiguous(m):
    """The same E4M3 rows through a scattered block table and through a
    contiguous cache give the same bits; both match the low-bit oracle."""
    from mla_latent_kv_47_b200.cache import LatentCache, PagedLatentCache
    p = synth.preset("v2")
    dims = m.make_dims(V2_E4M3)
    Wh, Wd = gu.device_weights(p)
    wts = m.make_weights(Wd)
    L = [0, 63, 64, 130, 1000]
    B = len(L)
    caps = [x + 2 for x in L]
    n_pages = sum((c + 63) // 64 for c in caps) + 3
    paged = PagedLatentCache(dims, caps, block_size=64, poison=True, spare_pages=3,
                             page_order=np.random.default_rng(4).permutation(n_pages))
    flat = LatentCache(dims, [x + 1 for x in L])
    ws = m.alloc_workspace(dims, B, 2048)
    hs = {b: synth.hidden(p, b, L[b] + 1) for b in range(B)}
    gu.fill_cache(m, dims, Wd, paged, ws, hs, L, p, chunk=2048)
    gu.fill_cache(m, dims, Wd, flat, ws, hs, L, p, chunk=2048)
    h_new = gu.to_dev(np.stack([hs[b][L[b]] for b in range(B)]), "bf16")
    seqlen = torch.tensor(L, dtype=torch.int32, device="cuda")
    u_p = torch.full((B, p.dims.d_model), float("nan"), dtype=torch.float32, device="cuda")
    u_f = torch.full((B, p.dims.d_model), float("nan"), dtype=torch.float32, device="cuda")
    m.decode(dims, wts, h_new, paged.handle, seqlen, u_p, ws)
    assert m.device_status(ws) == (0, 0)
    m.decode(dims, wts, h_new, flat.handle, seqlen, u_f, ws)
    assert m.device_status(ws) == (0, 0)
    assert torch.equal(u_p, u_f)
    data = paged.data.cpu().numpy()
    written = np.zeros(paged.total_rows, dtype=bool)
    for b in range(B):
        for q in range(L[b] + 1):
            written[paged.row_of(b, q)] = True
    assert np.all(data[~written] == 0x7F)
    u = u_p.cpu().numpy().astype(np.float64)
    for b in range(B):
        gu.assert_gate(gu.gate(u[b], lb.decode_lowbit(Wh, hs[b], V2_E4M3, "e4m3")))


def test_rmsnorm_then_e4m3(m):
    """c^KV is normalised and then encoded (the cache-row check covers the
    normalised rows' codes and scales; u against the oracle over the same
    stored rows)."""
    p = synth.preset("v2")
    L = [0, 65, 700, 3000]
    st = run_decode(m, "v2", checked=list(range(len(L))), lengths=L, dims=V2_E4M3, weights=weights_with_gains(p),
                    chunk=4096)
    for s in st.values():
        gu.assert_gate(s)


def test_all_options_together(m):
    """YaRN (positions past 4K), RMSNorm on c^KV and c^Q, and the E4M3 cache."""
    p = synth.preset("v2")
    L = [4095, 5000, 9000]
    st = run_decode(m, "v2", checked=[0, 1, 2], lengths=L, dims=V2_ALL, weights=weights_with_gains(p), chunk=4096,
                    oracle=lambda n: "unabsorbed" if n < 8192 else "absorbed")
    for s in st.values():
        gu.assert_gate(s)
    print("all options", st)


def test_static_decode_over_an_e4m3_cache(m):
    """mla_decode_static runs the E4M3 attention variant on its static
    scratch and gives mla_decode's bits."""
    from mla_latent_kv_47_b200.cache import LatentCache
    p = synth.preset("v2")
    dims = m.make_dims(V2_E4M3)
    _, Wd = gu.device_weights(p)
    wts = m.make_weights(Wd)
    L = [5, 300, 2000]
    cache = LatentCache(dims, [x + 1 for x in L])
    ws = m.alloc_workspace(dims, len(L), 2048)
    gu.fill_cache(m, dims, Wd, cache, ws, {}, L, p, chunk=2048)
    h = torch.randn((len(L), p.dims.d_model), device="cuda").to(torch.bfloat16)
    seqlen = torch.tensor(L, dtype=torch.int32, device="cuda")
    u_ref = torch.empty((len(L), p.dims.d_model), dtype=torch.float32, device="cuda")
    m.decode(dims, wts, h, cache.handle, seqlen, u_ref, ws)
    assert m.device_status(ws) == (0, 0)
    for _ in range(2):
        u = torch.full_like(u_ref, float("nan"))
        m.decode_static(dims, wts, h, cache.handle, seqlen, u)
        torch.cuda.synchronize()
        assert torch.equal(u, u_ref)
