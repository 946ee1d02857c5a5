"""GPU parity of the decode path (mla_cache_append + mla_decode) against the fp64 oracle.

Cache layout and sequence-length indexing are checked bit-exactly: every
cache row outside the rows written for (sequence, position) keeps its NaN
poison pattern, and no poisoned row reaches u.  Row values must be within
half a bf16 ulp of the exact row plus the fp32 accumulation noise bound
(tests/gpu_util.cache_value_check).  Outputs u must pass the gate
max|d| <= 1e-2 max|ref| and mean|d| <= 2e-3 max|ref| (bf16 storage), or a
1e-4 bound on both for fp32 storage.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import synth  # noqa: E402
from oracle import lowbit as lb  # noqa: E402
from oracle import mla as om  # noqa: E402
from tests import gpu_util as gu  # noqa: E402


@pytest.fixture(scope="module")
def m():
    import mla_latent_kv_47_b200 as mod
    return mod


def run_decode(m, preset, checked, lengths=None, pad=2, oracle="unabsorbed", dirty_workspace=False, h_scale=None,
               dims=None, weights=None, chunk=None):
    """Fills a poisoned cache through mla_cache_append, runs one mla_decode and
    checks layout, cache rows and u.  `dims` replaces the preset's dims (same
    shapes, e.g. with YaRN on); `weights` (host, device) replaces its weights.
    `oracle` names the fp64 form u is compared with, per sequence when it is a
    callable of the sequence's length.  `chunk`: tokens per mla_cache_append
    call, with a workspace sized for them (the latent RMSNorm needs it)."""
    from mla_latent_kv_47_b200.cache import LatentCache
    p = synth.preset(preset) if isinstance(preset, str) else preset
    d = p.dims if dims is None else dims
    dims = m.make_dims(d)
    L = list(lengths if lengths is not None else p.seqlen)
    B = len(L)
    Wh, Wd = gu.device_weights(p) if weights is None else weights
    cache = LatentCache(dims, [x + 1 + pad for x in L], poison=True, gap=1)
    ws = m.alloc_workspace(dims, B, chunk or 1)
    if dirty_workspace:
        ws.fill_(0xFF)      # NaN floats, -1 counters: nothing may be read before it is written
        ws[:256].zero_()    # except the status word, zeroed once by contract
    seqs_h = {b: synth.hidden(p, b, L[b] + 1) for b in checked}
    if h_scale is not None:   # per-token scale of the checked sequences (powers of two keep bf16 values exact)
        seqs_h = {b: h * h_scale(np.arange(h.shape[0]))[:, None].astype(h.dtype) for b, h in seqs_h.items()}
    gu.fill_cache(m, dims, Wd, cache, ws, seqs_h, L, p, chunk=chunk or 32768)
    tdt = torch.float32 if d.dtype == "fp32" else torch.bfloat16
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    h_new = torch.randn((B, d.d_model), generator=g, device="cuda").to(tdt)
    for b in checked:
        h_new[b] = gu.to_dev(seqs_h[b][L[b]:L[b] + 1], d.dtype)[0]
    seqlen = torch.tensor(L, dtype=torch.int32, device="cuda")
    u = torch.full((B, d.d_model), float("nan"), dtype=torch.float32, device="cuda")
    m.decode(dims, m.make_weights(Wd), h_new, cache.handle, seqlen, u, ws)
    code, detail = m.device_status(ws)
    assert (code, detail) == (0, 0)
    u_h = u.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(u_h)), "a poisoned or unwritten row reached u"
    # ---- layout: exactly rows seq_start[b] + [0, L_b] were written
    written = np.zeros(cache.total_rows, dtype=bool)
    ss = cache.seq_start.cpu().numpy()
    for b in range(B):
        written[ss[b]:ss[b] + L[b] + 1] = True
    data = cache.data.cpu()
    e4m3 = getattr(d, "cache", "dtype") == "e4m3"
    if e4m3:
        bits = data.numpy()
        pois = np.uint8(0x7F)
    elif d.dtype == "bf16":
        bits = data.view(torch.int16).numpy().astype(np.uint16)
        pois = np.uint16(0x7FC1)
    else:
        bits = data.view(torch.int32).numpy().astype(np.uint32)
        pois = np.uint32(0x7FC00001)
    assert np.all(bits[~written] == pois), "a row outside the written range changed"
    assert not np.any(np.all(bits[written] == pois, axis=1)), "a row that should be written is still poison"
    # ---- values
    stats = {}
    for b in checked:
        hb = seqs_h[b]
        got = bits[ss[b]:ss[b] + L[b] + 1]
        if e4m3:
            ratio = gu.e4m3_row_check(got, Wh, hb, np.arange(L[b] + 1.0), d)
            assert ratio <= 1.0, f"seq {b}: E4M3 cache row error at {ratio:.3g} of its bound"
        elif d.dtype == "bf16":
            ratio = gu.cache_value_check(got, Wh, hb, np.arange(L[b] + 1.0), d)
            assert ratio <= 1.0, f"seq {b}: cache row error at {ratio:.3g} of its bound"
        else:
            c_kv, k_r = om.latent_rows(Wh, hb, np.arange(L[b] + 1.0), d)
            rows_ref = np.concatenate([c_kv, k_r], axis=1)
            gotf = got.view(np.float32).astype(np.float64)
            assert np.max(np.abs(gotf - rows_ref)) <= 1e-5 * np.max(np.abs(rows_ref))
        form = oracle(L[b]) if callable(oracle) else oracle
        if e4m3:   # the oracle over the same low-bit rows (codes and scales of the exact latents)
            u_ref = lb.decode_lowbit(Wh, hb, d, "e4m3", absorbed=(form == "absorbed"))
        else:
            u_ref = (om.decode_unabsorbed if form == "unabsorbed" else om.decode_absorbed)(Wh, hb, d)
        stats[b] = gu.gate(u_h[b], u_ref)
    return stats


def test_tiny_fp32_decode(m):
    st = run_decode(m, "tiny", checked=[0])
    for s in st.values():
        gu.assert_gate(s, 1e-4, 1e-4)


def test_lite_decode_all_sequences(m):
    st = run_decode(m, "lite", checked=list(range(32)))
    for b, s in st.items():
        gu.assert_gate(s)
    print("lite gate", max(s["max_rel"] for s in st.values()), max(s["mean_rel"] for s in st.values()),
          max(s["sum_rel"] for s in st.values()))


@pytest.mark.parametrize("n_h", [8, 32])
def test_other_head_counts(m, n_h):
    """V2-Lite dims with 8 heads (the few-head attention kernel, its Q rows
    past n_h zero; the combine split over 4 CTAs) and 32 heads (the 2-CTA
    kernel with 96 empty head rows; the combine split over 2), on ragged
    short lengths, every sequence checked."""
    import dataclasses
    d = dataclasses.replace(synth.V2_LITE, n_h=n_h)
    L = (0, 1, 63, 65, 300, 1000)
    p = synth.Preset(f"lite_h{n_h}", 2, d, len(L), L)
    st = run_decode(m, p, checked=list(range(len(L))))
    for s in st.values():
        gu.assert_gate(s)


def test_v2_decode_sampled(m):
    st = run_decode(m, "v2", checked=[0, 31, 63])
    for s in st.values():
        gu.assert_gate(s)
    print("v2 gate", st)


def test_v2_dims_ragged_small(m):
    """V2 dims with short ragged lengths: empty caches (L=0), single tiles,
    ragged tails and a long sequence, all checked."""
    L = [0, 1, 63, 64, 65, 127, 128, 129, 700, 2049, 5, 0, 300, 1000, 64 * 7 + 3, 1]
    st = run_decode(m, "v2", checked=list(range(len(L))), lengths=L)
    for s in st.values():
        gu.assert_gate(s)


def test_ragged_preset_sampled(m):
    p = synth.preset("ragged")
    L = np.array(p.seqlen)
    order = np.argsort(L, kind="stable")
    picks = sorted({int(order[0]), int(order[-1]), int(order[len(L) // 2])} |
                   set(int(x) for x in np.random.default_rng(0).choice(len(L), 5, replace=False)))
    st = run_decode(m, "ragged", checked=picks, oracle="absorbed")
    for s in st.values():
        gu.assert_gate(s)
    print("ragged gate", st)


@pytest.mark.parametrize("preset,L", [("tiny", [64]), ("v2", [3, 70]), ("lite", [0, 1, 4096])])
def test_decode_with_dirty_workspace(m, preset, L):
    """Small batches leave most attention workers without tiles; a workspace
    full of 0xFF bytes must still give the oracle's result."""
    st = run_decode(m, preset, checked=list(range(len(L))), lengths=L, dirty_workspace=True)
    for s in st.values():
        if preset == "tiny":
            gu.assert_gate(s, 1e-4, 1e-4)
        else:
            gu.assert_gate(s)


def test_scores_above_the_piece_reference(m):
    """Cached tokens scaled by 1 and 4 in alternate 64-token tiles (the query
    row unscaled) put the max score of a scaled tile ~11.5 log2 units above an
    unscaled tile's (~15 against ~3.5).  The attention kernel forms P against
    the max of a piece's first tile, so inside most pieces P rises to ~2^11
    (never rescaled; the reference cancels in O / l), which unscaled inputs
    never reach.  The lengths give ~2.8 tiles per worker, so pieces span
    several tiles.  With scores this large the bf16 operands alone (Q_lat,
    cache rows, P) cost up to 0.72% max / 0.15% mean of max|u| (fp64
    emulation of those roundings), inside the gate; larger scales push that
    bound past it."""
    L = [8192, 4000, 777]

    def scale(pos):
        s = np.array([1.0, 4.0])[(pos // 64) % 2]
        s[-1] = 1.0   # the new token, whose query scores the rest
        return s

    st = run_decode(m, "v2", checked=[0, 1, 2], lengths=L, h_scale=scale)
    for s in st.values():
        gu.assert_gate(s)
    print("rescale gate", st)


def test_single_token_closed_form(m):
    """L_b = 0: the softmax is exactly 1, so u = W_O blockdiag(W_UV) c^KV (fp64 closed form)."""
    p = synth.preset("lite")
    st = run_decode(m, "lite", checked=[0, 1, 2], lengths=[0, 0, 0])
    for s in st.values():
        gu.assert_gate(s)


def test_capacity_overflow_is_reported(m):
    from mla_latent_kv_47_b200.cache import LatentCache
    p = synth.preset("tiny")
    d = p.dims
    dims = m.make_dims(d)
    Wh, Wd = gu.device_weights(p)
    cache = LatentCache(dims, [4, 4], poison=True)
    ws = m.alloc_workspace(dims, 2, 1)
    h = torch.randn((2, d.d_model), device="cuda")
    seqlen = torch.tensor([3, 4], dtype=torch.int32, device="cuda")   # seq 1 is full
    u = torch.empty((2, d.d_model), device="cuda")
    m.decode(dims, m.make_weights(Wd), h, cache.handle, seqlen, u, ws)
    code, detail = m.device_status(ws)
    assert code == -6 and detail & m.FAULT_CAPACITY
    assert m.device_status(ws) == (0, 0)   # reading clears the word
    bits = cache.data.view(torch.int32).cpu().numpy()
    assert np.all(bits[4:8] == 0x7FC00001)   # nothing written past sequence 1's capacity


def test_host_errors_enqueue_nothing(m):
    p = synth.preset("tiny")
    dims = m.make_dims(p.dims)
    Wh, Wd = gu.device_weights(p)
    from mla_latent_kv_47_b200.cache import LatentCache
    cache = LatentCache(dims, [8])
    ws = m.alloc_workspace(dims, 1, 1)
    h = torch.randn((1, p.dims.d_model), device="cuda")
    seqlen = torch.tensor([2], dtype=torch.int32, device="cuda")
    u = torch.empty((1, p.dims.d_model), device="cuda")
    with pytest.raises(m.MLAError) as e:
        m.decode(dims, m.make_weights(Wd), h, cache.handle, seqlen, u, ws[:1024])
    assert e.value.code == -4
    bad = m.make_dims(p.dims)
    bad.d_R = 7
    with pytest.raises(m.MLAError) as e:
        m.decode(bad, m.make_weights(Wd), h, cache.handle, seqlen, u, ws)
    assert e.value.code == -2
    W2 = dict(Wd)
    W2["W_O"] = None
    with pytest.raises(m.MLAError) as e:
        m.decode(dims, m.make_weights(W2), h, cache.handle, seqlen, u, ws)
    assert e.value.code == -1


@pytest.mark.parametrize("preset", ["v2", "lite"])
def test_decode_intermediates(m, preset):
    """Q_lat = [W_UK_i^T q^C_i ; q^R_i] * log2(e)/sqrt(d_h+d_R) and the normalised
    latent output O_lat, read back from the workspace, against the oracle's
    absorbed-form intermediates (localises a failure to one step)."""
    import math
    from mla_latent_kv_47_b200.cache import LatentCache
    p = synth.preset(preset)
    d = p.dims
    dims = m.make_dims(d)
    L = [3, 200, 64, 129]
    B = len(L)
    Wh, Wd = gu.device_weights(p)
    cache = LatentCache(dims, [x + 1 for x in L], poison=True)
    ws = m.alloc_workspace(dims, B, 1)
    hs = {b: synth.hidden(p, b, L[b] + 1) for b in range(B)}
    gu.fill_cache(m, dims, Wd, cache, ws, hs, L, p)
    h_new = gu.to_dev(np.stack([hs[b][L[b]] for b in range(B)]), d.dtype)
    u = torch.empty((B, d.d_model), dtype=torch.float32, device="cuda")
    m.decode(dims, m.make_weights(Wd), h_new, cache.handle, torch.tensor(L, dtype=torch.int32, device="cuda"), u, ws)
    assert m.device_status(ws) == (0, 0)
    row = d.d_c + d.d_R
    off_q = m.workspace_offset(dims, B, m.WS_QLAT)
    off_o = m.workspace_offset(dims, B, m.WS_OLAT)
    qlat = ws[off_q:off_q + B * d.n_h * row * 2].view(torch.bfloat16).float().cpu().numpy().reshape(B, d.n_h, row)
    olat = ws[off_o:off_o + B * d.n_h * d.d_c * 2].view(torch.bfloat16).float().cpu().numpy().reshape(B, d.n_h, d.d_c)
    scale = math.log2(math.e) / math.sqrt(d.d_h + d.d_R)
    for b in range(B):
        _, parts = om.decode_absorbed(Wh, hs[b], d, return_parts=True)
        qref = parts["q_lat"] * scale
        for name, got, ref in (("q_abs", qlat[b, :, :d.d_c], qref[:, :d.d_c]),
                               ("q_rope", qlat[b, :, d.d_c:], qref[:, d.d_c:]),
                               ("o_lat", olat[b], parts["o_lat"])):
            s = gu.gate(got, ref)
            assert s["max_rel"] <= 1e-2 and s["mean_rel"] <= 2e-3, (name, b, s)


def test_score_jump_past_the_kernel_range_is_reported(m):
    """Inside a run of tiles the attention kernel forms P against the max of
    the run's first tile, so P may exceed 1; its range is P <= 2^96.  Cached tokens 192..255 of sequence 0 scaled by 64
    put that tile's scores ~200 log2 units above the earlier tiles' (its piece
    starts at tile 0: 8 sequences of 4096 tokens give ~7 tiles per attention
    worker), past the range, so the call reports FAULT_RANGE through the
    status word instead of returning a silently wrong u; the status is
    cleared by reading it."""
    from mla_latent_kv_47_b200.cache import LatentCache
    p = synth.preset("v2")
    d = p.dims
    dims = m.make_dims(d)
    L = [4096] * 8
    Wh, Wd = gu.device_weights(p)
    cache = LatentCache(dims, [x + 1 for x in L])
    ws = m.alloc_workspace(dims, len(L), 1)
    h0 = synth.hidden(p, 0, L[0] + 1)
    h0[192:256] *= 64.0
    gu.fill_cache(m, dims, Wd, cache, ws, {0: h0}, L, p)
    h_new = gu.to_dev(np.stack([h0[L[0]]] + [synth.hidden(p, b, 1, first=L[b])[0] for b in range(1, 8)]), "bf16")
    u = torch.empty((len(L), d.d_model), dtype=torch.float32, device="cuda")
    m.decode(dims, m.make_weights(Wd), h_new, cache.handle, torch.tensor(L, dtype=torch.int32, device="cuda"), u, ws)
    code, detail = m.device_status(ws)
    assert code == -6 and detail & m.FAULT_RANGE, (code, detail)
    assert m.device_status(ws) == (0, 0)


def test_bounded_wait_gives_up_and_the_context_stays_usable(m):
    """A pipeline wait that nothing satisfies gives up after its time limit,
    reports FAULT_WAIT_TIMEOUT through the status word, and leaves the GPU
    context usable: a decode right after it passes the gate."""
    p = synth.preset("tiny")
    dims = m.make_dims(p.dims)
    ws = m.alloc_workspace(dims, 1, 1)
    m.check_wait_timeout(ws)
    code, detail = m.device_status(ws)
    assert code == -6 and detail == m.FAULT_WAIT_TIMEOUT, (code, detail)
    st = run_decode(m, "tiny", checked=[0])
    for s in st.values():
        gu.assert_gate(s, 1e-4, 1e-4)
