"""CPU oracle of the SVDQuant W4A4 linear layer (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this package.  It shares no code with the CUDA library.
"""
from . import svdq_oracle  # noqa: F401
