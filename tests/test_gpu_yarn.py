"""GPU parity of YaRN-scaled RoPE and its attention factor ("DeepSeek-V2
summary" (7shi.hateblo.jp) §3.1.4: s = 40, alpha = 1, beta = 32 on top of a 4K
pre-training length, scores times t with sqrt(t) = 0.0707 ln s + 1) against
the fp64 oracle run with the same `yarn` dims.

Positions go past the 4K pre-training length, up to the longest sequence of
the ragged preset (126,832 cached tokens).  The CPU suite checks that at
such positions the YaRN result differs from plain RoPE by several times the
gate (tests/test_oracle_yarn.py), so a GPU result inside the gate cannot be
plain RoPE.
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import synth  # noqa: E402
from oracle import mla as om  # noqa: E402
from tests import gpu_util as gu  # noqa: E402
from tests.test_gpu_decode import run_decode  # noqa: E402
from tests.test_gpu_prefill import run_prefill  # noqa: E402

YARN = (40.0, 1.0, 32.0, 4096.0)
V2_YARN = dataclasses.replace(synth.V2, yarn=YARN)


@pytest.fixture(scope="module")
def m():
    import mla_latent_kv_47_b200 as mod
    return mod


def _oracle_form(n):
    # the absorbed form is pinned to the un-absorbed one at these dims; it is
    # used for the long sequences, where the un-absorbed k/v cost dominates
    return "unabsorbed" if n < 8192 else "absorbed"


def test_yarn_decode_beyond_the_pretraining_length(m):
    L = [4095, 4096, 6000, 20000, 0, 64]
    st = run_decode(m, "v2", checked=list(range(len(L))), lengths=L, dims=V2_YARN, oracle=_oracle_form)
    for s in st.values():
        gu.assert_gate(s)
    print("yarn decode", st)


def test_yarn_decode_longest_ragged_sequence(m):
    p = synth.preset("ragged")
    L = list(p.seqlen)
    longest = int(np.argmax(L))
    st = run_decode(m, "ragged", checked=[longest, int(np.argsort(L)[len(L) // 2])], dims=V2_YARN,
                    oracle=_oracle_form)
    for s in st.values():
        gu.assert_gate(s)
    print("yarn ragged", st)


def test_yarn_prefill_after_a_long_prefix(m):
    s = run_prefill(m, "v2", 200, start_pos=4500, rows=[0, 1, 127, 128, 199], dims=V2_YARN)
    gu.assert_gate(s)
