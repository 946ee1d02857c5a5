"""GPU parity of the causal prefill path (mla_prefill) against the fp64 oracle."""
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


def run_prefill(m, preset, T, start_pos=0, rows=None, seq=1, n_seq=3, pad=3, dims=None, weights=None):
    from mla_latent_kv_47_b200.cache import LatentCache
    p = synth.preset(preset)
    d = p.dims if dims is None else dims
    dims = m.make_dims(d)
    Wh, Wd = gu.device_weights(p) if weights is None else weights
    S = start_pos + T
    cache = LatentCache(dims, [S + pad] * n_seq, poison=True, gap=1)
    ws = m.alloc_workspace(dims, 1, S)
    h_all = synth.hidden(p, seq, S)
    if start_pos:
        gu.fill_cache(m, dims, Wd, cache, ws, {seq: h_all}, [0] * seq + [start_pos], p)
    u = torch.full((T, d.d_model), float("nan"), dtype=torch.float32, device="cuda")
    m.prefill(dims, m.make_weights(Wd), gu.to_dev(h_all[start_pos:], d.dtype), start_pos, cache.handle, seq, u, ws)
    assert m.device_status(ws) == (0, 0)
    u_h = u.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(u_h))
    # layout: only rows [0, S) of sequence `seq` are written
    written = np.zeros(cache.total_rows, dtype=bool)
    s0 = int(cache.seq_start[seq].item())
    written[s0:s0 + S] = True
    data = cache.data.cpu()
    if d.dtype == "bf16":
        bits = data.view(torch.int16).numpy().astype(np.uint16)
        assert np.all(bits[~written] == np.uint16(0x7FC1))
        ratio = gu.cache_value_check(bits[s0:s0 + S], Wh, h_all, np.arange(float(S)), d)
        assert ratio <= 1.0, f"cache row error at {ratio:.3g} of its bound"
    else:
        bits = data.view(torch.int32).numpy().astype(np.uint32)
        assert np.all(bits[~written] == np.uint32(0x7FC00001))
    rows = list(range(T)) if rows is None else rows
    u_ref = om.prefill_unabsorbed(Wh, h_all[start_pos:], d, start_pos=start_pos,
                                  h_prefix=h_all[:start_pos] if start_pos else None, rows=rows)
    return gu.gate(u_h[rows], u_ref)


def test_tiny_fp32_prefill(m):
    gu.assert_gate(run_prefill(m, "tiny", 40), 1e-4, 1e-4)


def test_tiny_fp32_prefill_after_prefix(m):
    gu.assert_gate(run_prefill(m, "tiny", 25, start_pos=17), 1e-4, 1e-4)


def test_v2_dims_prefill_small(m):
    """300 tokens: several 128-token tiles and a ragged tail, every row checked."""
    s = run_prefill(m, "v2", 300)
    gu.assert_gate(s)
    print("v2 prefill small", s)


def test_v2_dims_prefill_after_prefix(m):
    s = run_prefill(m, "v2", 130, start_pos=200, rows=[0, 1, 63, 64, 127, 128, 129])
    gu.assert_gate(s)


def test_prefill_preset_sampled(m):
    """The full 16384-token prefill; the oracle checks a fixed set of rows."""
    T = synth.preset("prefill").prefill_T
    rows = sorted({0, 1, 127, 128, 129, 4095, 8191, 12345, T - 2, T - 1} |
                  set(int(x) for x in np.random.default_rng(5).choice(T, 6, replace=False)))
    s = run_prefill(m, "prefill", T, rows=rows, n_seq=1, seq=0)
    gu.assert_gate(s)
    print("prefill gate", s)
