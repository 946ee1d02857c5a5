"""GPU parity of the E4M3 latent cache (the low-bit cache of "DeepSeek-V2
summary" (7shi.hateblo.jp) §3.2.3 and the FP8 KV cache of the serving example
in "딥시크 V2" (downcodes.com) §8; the format is the reading recorded with
oracle/lowbit.py: E4M3 codes of c^KV with one power-of-two scale per row, k^R
kept in bf16).

The encoder is checked bit for bit: the codes and scale exponents written by
mla_cache_append are those oracle/lowbit.quantize_rows computes from the same
fp32 c^KV (read back from the workspace), so the decision of every code is
taken in the same precision on both sides.  Decode over the E4M3 cache is
checked against the oracle run over the same stored rows (decode_lowbit),
within the bf16 gate; the format's own error against the exact decode is
printed beside it.
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import synth  # noqa: E402
from oracle import lowbit as lb  # noqa: E402
from oracle import mla as om  # noqa: E402
from tests import gpu_util as gu  # noqa: E402
from tests.test_gpu_decode import run_decode  # noqa: E402

V2_E4M3 = dataclasses.replace(synth.V2, cache="e4m3")


@pytest.fixture(scope="module")
def m():
    import mla_latent_kv_47_b200 as mod
    return mod


def test_e4m3_append_writes_the_oracle_codes(m):
    from mla_latent_kv_47_b200.cache import LatentCache
    p = synth.preset("v2")
    dims = m.make_dims(V2_E4M3)
    Wh, Wd = gu.device_weights(p)
    T = 300
    cache = LatentCache(dims, [T + 5, 40], poison=True, gap=3)
    ws = m.alloc_workspace(dims, 2, T)
    h = synth.hidden(p, 0, T)
    m.cache_append(dims, m.make_weights(Wd), gu.to_dev(h, "bf16"), torch.zeros(T, dtype=torch.int32, device="cuda"),
                   torch.arange(T, dtype=torch.int32, device="cuda"), cache.handle, ws)
    assert m.device_status(ws) == (0, 0)
    off = m.workspace_offset_tokens(dims, T, m.WS_CKV_RAW)
    raw = ws[off:off + T * 512 * 4].view(torch.float32).cpu().numpy().reshape(T, 512).astype(np.float64)
    # the fp32 c^KV is the down-projection (sanity: against the exact product)
    exact = np.asarray(h, np.float64) @ np.asarray(Wh["W_DKV"], np.float64).T
    assert np.max(np.abs(raw - exact)) <= 1e-4 * np.max(np.abs(exact))
    codes_ref, k_ref = lb.quantize_rows(raw, "e4m3")
    data = cache.data.cpu().numpy()
    rows = data[:T]
    got = rows[:, :512]
    zero_either_sign = ((got & 0x7F) == 0) & ((codes_ref & 0x7F) == 0)
    assert np.all((got == codes_ref) | zero_either_sign), "codes differ from the oracle encoder"
    assert np.array_equal(rows[:, 640].view(np.int8).astype(np.int64), k_ref), "scale exponents differ"
    assert np.all(rows[:, 641:656] == 0)
    assert gu.e4m3_row_check(rows, Wh, h, np.arange(float(T)), V2_E4M3) <= 1.0
    assert np.all(data[T:] == 0x7F), "a row outside the written range changed"


def test_e4m3_decode_matches_the_lowbit_oracle(m):
    L = [0, 1, 63, 64, 65, 700, 8192]
    st = run_decode(m, "v2", checked=list(range(len(L))), lengths=L, dims=V2_E4M3, chunk=4096)
    for s in st.values():
        gu.assert_gate(s)
    print("e4m3 decode vs decode_lowbit", st)


def test_e4m3_decode_ragged_picks(m):
    p = synth.preset("ragged")
    L = np.array(p.seqlen)
    order = np.argsort(L, kind="stable")
    picks = sorted({int(order[0]), int(order[-1]), int(order[len(L) // 2])})
    st = run_decode(m, "ragged", checked=picks, dims=dataclasses.replace(p.dims, cache="e4m3"), chunk=4096,
                    oracle=lambda n: "unabsorbed" if n < 8192 else "absorbed")
    for s in st.values():
        gu.assert_gate(s)
    print("e4m3 ragged vs decode_lowbit", st)


def test_e4m3_format_error_is_reported():
    """CPU side, for the record: the format's own error against the exact
    decode at DeepSeek-V2 dims (the GPU matches decode_lowbit, which has it)."""
    p = synth.preset("v2")
    W = synth.weights(p)
    h = synth.hidden(p, 0, 2001)
    a = lb.decode_lowbit(W, h, p.dims, "e4m3", absorbed=True)
    b = om.decode_absorbed(W, h, p.dims)
    s = gu.gate(a, b)
    print("E4M3 cache vs exact decode", s)
    assert s["max_rel"] < 0.1
