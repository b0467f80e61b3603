"""CPU oracle for the XAttention prefill path (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this package. The CUDA library never reaches it.
"""
from .xattn_oracle import *  # noqa: F401,F403
from .xattn_oracle import __all__  # noqa: F401
