"""GPU parity of the paged latent cache (a pool of pages with a block table,
the layout of PagedAttention, cited among the pages' references; the vLLM
serving path of "딥시크 V2" (downcodes.com) §8 runs on it).

A sequence's pages are scattered through the pool (a seeded permutation,
with spare pages left poisoned).  Checked: exactly the rows the block table
names are written (every other byte keeps its NaN poison), decode and prefill
match the fp64 oracle, and decode over the paged cache equals, bit for bit,
decode over a contiguous cache holding the same rows (the attention reads
the same rows in the same order, only from other addresses).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import synth  # noqa: E402
from oracle import mla as om  # noqa: E402
from tests import gpu_util as gu  # noqa: E402


@pytest.fixture(scope="module")
def m():
    import mla_latent_kv_47_b200 as mod
    return mod


def _paged(m, dims, L, block_size, seed=3, spare=5, pad=1):
    from mla_latent_kv_47_b200.cache import PagedLatentCache
    caps = [x + 1 + pad for x in L]
    n_pages = sum((c + block_size - 1) // block_size for c in caps) + spare
    order = np.random.default_rng(seed).permutation(n_pages)
    return PagedLatentCache(dims, caps, block_size=block_size, poison=True, spare_pages=spare, page_order=order)


def _written_mask(cache, L):
    w = np.zeros(cache.total_rows, dtype=bool)
    for b, n in enumerate(L):
        for p in range(n + 1):
            w[cache.row_of(b, p)] = True
    return w


@pytest.mark.parametrize("preset,L,bs", [("v2", [0, 1, 63, 64, 65, 200, 1000, 130], 64),
                                         ("v2", [5, 300, 2049], 128),
                                         ("lite", [100, 4096], 64),
                                         ("tiny", [64, 3], 64)])
def test_paged_decode_matches_oracle_and_contiguous(m, preset, L, bs):
    from mla_latent_kv_47_b200.cache import LatentCache
    p = synth.preset(preset)
    d = p.dims
    dims = m.make_dims(d)
    Wh, Wd = gu.device_weights(p)
    wts = m.make_weights(Wd)
    B = len(L)
    paged = _paged(m, dims, L, bs)
    flat = LatentCache(dims, [x + 1 for x in L])
    ws = m.alloc_workspace(dims, B, 1)
    hs = {b: synth.hidden(p, b, L[b] + 1) for b in range(B)}
    gu.fill_cache(m, dims, Wd, paged, ws, hs, L, p)
    gu.fill_cache(m, dims, Wd, flat, ws, hs, L, p)
    h_new = gu.to_dev(np.stack([hs[b][L[b]] for b in range(B)]), d.dtype)
    seqlen = torch.tensor(L, dtype=torch.int32, device="cuda")
    u_p = torch.full((B, d.d_model), float("nan"), dtype=torch.float32, device="cuda")
    u_f = torch.full((B, d.d_model), float("nan"), dtype=torch.float32, device="cuda")
    m.decode(dims, wts, h_new, paged.handle, seqlen, u_p, ws)
    assert m.device_status(ws) == (0, 0)
    m.decode(dims, wts, h_new, flat.handle, seqlen, u_f, ws)
    assert m.device_status(ws) == (0, 0)
    assert torch.equal(u_p, u_f), "paged and contiguous layouts must give the same bits"
    # layout: exactly the rows the block table names for positions 0..L_b
    written = _written_mask(paged, L)
    if d.dtype == "bf16":
        bits = paged.data.view(torch.int16).cpu().numpy().astype(np.uint16)
        pois = np.uint16(0x7FC1)
    else:
        bits = paged.data.view(torch.int32).cpu().numpy().astype(np.uint32)
        pois = np.uint32(0x7FC00001)
    assert np.all(bits[~written] == pois), "a row outside the block table's rows changed"
    assert not np.any(np.all(bits[written] == pois, axis=1))
    flat_bits = flat.data.view(torch.int16 if d.dtype == "bf16" else torch.int32).cpu().numpy()
    for b in range(B):
        s0 = int(flat.seq_start[b].item())
        rows = [paged.row_of(b, q) for q in range(L[b] + 1)]
        assert np.array_equal(bits[rows].view(flat_bits.dtype), flat_bits[s0:s0 + L[b] + 1]), b
    u = u_p.cpu().numpy().astype(np.float64)
    for b in range(B):
        st = gu.gate(u[b], om.decode_unabsorbed(Wh, hs[b], d))
        if d.dtype == "fp32":
            gu.assert_gate(st, 1e-4, 1e-4)
        else:
            gu.assert_gate(st)


def test_paged_prefill_after_prefix(m):
    """Prefill of 130 tokens after a 200-token prefix, both through the block
    table (pages of 64 rows scattered in the pool)."""
    p = synth.preset("v2")
    d = p.dims
    dims = m.make_dims(d)
    Wh, Wd = gu.device_weights(p)
    start, T = 200, 130
    S = start + T
    cache = _paged(m, dims, [0, S - 1], 64, seed=9)
    ws = m.alloc_workspace(dims, 1, S)
    h_all = synth.hidden(p, 1, S)
    gu.fill_cache(m, dims, Wd, cache, ws, {1: h_all}, [0, start], p)
    u = torch.full((T, d.d_model), float("nan"), dtype=torch.float32, device="cuda")
    m.prefill(dims, m.make_weights(Wd), gu.to_dev(h_all[start:], d.dtype), start, cache.handle, 1, u, ws)
    assert m.device_status(ws) == (0, 0)
    rows = [0, 1, 63, 64, 127, 129]
    ref = om.prefill_unabsorbed(Wh, h_all[start:], d, start_pos=start, h_prefix=h_all[:start], rows=rows)
    gu.assert_gate(gu.gate(u.cpu().numpy().astype(np.float64)[rows], ref))
    bits = cache.data.view(torch.int16).cpu().numpy().astype(np.uint16)
    written = np.zeros(cache.total_rows, dtype=bool)
    for q in range(S):
        written[cache.row_of(1, q)] = True
    assert np.all(bits[~written] == np.uint16(0x7FC1))


def test_position_past_the_block_table_is_reported(m):
    """A token at a position the block table has no page for is not written
    and raises FAULT_CAPACITY (no capacity array given)."""
    from mla_latent_kv_47_b200.cache import PagedLatentCache
    p = synth.preset("v2")
    d = p.dims
    dims = m.make_dims(d)
    _, Wd = gu.device_weights(p)
    cache = PagedLatentCache(dims, [64, 64], block_size=64, poison=True)
    cache.handle.capacity = None
    ws = m.alloc_workspace(dims, 2, 1)
    h = torch.randn((2, d.d_model), device="cuda").to(torch.bfloat16)
    seqlen = torch.tensor([10, 64], dtype=torch.int32, device="cuda")   # sequence 1 has no page for position 64
    u = torch.empty((2, d.d_model), dtype=torch.float32, device="cuda")
    m.decode(dims, m.make_weights(Wd), h, cache.handle, seqlen, u, ws)
    code, detail = m.device_status(ws)
    assert code == -6 and detail & m.FAULT_CAPACITY
