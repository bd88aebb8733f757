"""CPU oracle of the speculative MoE decode step -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it.  It shares no code with the CUDA library.
"""
from .decoder import *  # noqa: F401,F403
