"""fp64 CPU oracle of the activation-sparse gated FFN forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` do.  It shares no code with the CUDA path.
"""
from .ffn import *  # noqa: F401,F403
