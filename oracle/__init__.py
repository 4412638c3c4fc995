"""Float64 CPU oracle of the decode-time MoE layer (test infrastructure only).

Only ``tests/``, the smoke check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py``
may import this package; the library and its binding never do.
"""
from .moe_ref import *  # noqa: F401,F403
from . import moe_ref  # noqa: F401
