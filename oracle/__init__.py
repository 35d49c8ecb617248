"""CPU oracle of the Sparse-First sparse step -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check in __graft_entry__ and the CPU-baseline leg of bench.py may import
this package. The product path never does; it shares no code with the CUDA library.
"""
from .oracle import *  # noqa: F401,F403
