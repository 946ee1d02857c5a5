"""fp64 CPU oracle for the MLA latent-KV hot path (test infrastructure only).

Only tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The CUDA library never does, and it shares no
code with it.
"""
from .mla import *  # noqa: F401,F403
from . import mla  # noqa: F401
