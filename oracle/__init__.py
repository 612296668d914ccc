"""Test infrastructure: the fp64 CPU oracle of the MoE layer forward pass.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use this
package.  The CUDA library never imports it.
"""
from .moe_ref import *  # noqa: F401,F403
from .moe_ref import __all__  # noqa: F401
