"""CPU oracle of the sparse MoE FFN layer forward (test infrastructure only).

Imported only by the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py``; the library never imports it.
"""
from .moe_oracle import *  # noqa: F401,F403
from . import moe_oracle  # noqa: F401
