"""Test infrastructure: the fp64 CPU oracle of the batch-invariant MoE layer.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  It does not import, and is not
imported by, the CUDA library.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import MAC_COUNTER  # noqa: F401
