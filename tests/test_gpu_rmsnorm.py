"""GPU parity of the RMSNorm on the compressed latents ("DeepSeek-V2 summary"
(7shi.hateblo.jp) §3.1.2: RMSNorm layers after c^KV and c^Q) against the fp64
oracle run with the same gains.

The gains g_kv [d_c] and g_q [d_cq] are drawn in [0.5, 1.5) and rounded to
bf16.  The cache rows written through mla_cache_append and mla_decode hold
the normalised c^KV (checked against the exact rows within the cache-row
bound), and decode and prefill outputs pass the bf16 gate.  The CPU suite
pins the oracle's norm (tests/test_oracle_rmsnorm.py) and shows that with
these gains the result moves by far more than the gate, so passing here
means the norm really runs.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import synth  # noqa: E402
from tests import gpu_util as gu  # noqa: E402
from tests.test_gpu_decode import run_decode  # noqa: E402
from tests.test_gpu_prefill import run_prefill  # noqa: E402


@pytest.fixture(scope="module")
def m():
    import mla_latent_kv_47_b200 as mod
    return mod


def weights_with_gains(p, seed=17, q=True):
    Wh = synth.weights(p)
    rng = np.random.default_rng(seed)
    Wh["g_kv"] = synth.round_bf16((0.5 + rng.random(p.dims.d_c)).astype(np.float32))
    if q and p.dims.d_cq:
        Wh["g_q"] = synth.round_bf16((0.5 + rng.random(p.dims.d_cq)).astype(np.float32))
    return Wh, {k: gu.to_dev(v, p.dims.dtype) for k, v in Wh.items()}


def test_rmsnorm_decode_v2(m):
    p = synth.preset("v2")
    L = [0, 1, 63, 64, 65, 700, 2049]
    st = run_decode(m, "v2", checked=list(range(len(L))), lengths=L, weights=weights_with_gains(p), chunk=4096)
    for s in st.values():
        gu.assert_gate(s)
    print("rmsnorm v2", st)


def test_rmsnorm_decode_lite_kv_only(m):
    """V2-Lite has no query compression, so only c^KV is normalised."""
    p = synth.preset("lite")
    L = [5, 1000, 4096]
    st = run_decode(m, "lite", checked=[0, 1, 2], lengths=L, weights=weights_with_gains(p), chunk=4096)
    for s in st.values():
        gu.assert_gate(s)


def test_rmsnorm_tiny_fp32(m):
    p = synth.preset("tiny")
    st = run_decode(m, "tiny", checked=[0], weights=weights_with_gains(p), chunk=4096)
    for s in st.values():
        gu.assert_gate(s, 1e-4, 1e-4)


def test_rmsnorm_prefill_v2(m):
    p = synth.preset("v2")
    s = run_prefill(m, "v2", 300, weights=weights_with_gains(p))
    gu.assert_gate(s)


def test_rmsnorm_prefill_after_prefix(m):
    p = synth.preset("v2")
    s = run_prefill(m, "v2", 130, start_pos=200, rows=[0, 1, 64, 129], weights=weights_with_gains(p))
    gu.assert_gate(s)
