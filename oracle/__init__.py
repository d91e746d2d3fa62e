"""CPU oracle of the MoE-layer forward -- test infrastructure only.

Imported only by the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
and reference arms of ``bench.py``; the CUDA library and its Python binding
never import it.  See ``moe_oracle.py`` for the sources each step follows.
"""
from .moe_oracle import *  # noqa: F401,F403
