"""fp64 CPU oracle for block-sparse attention (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg import this package.
It shares no code with the CUDA path, and the product path never routes through it.
"""
from . import attention, metadata  # noqa: F401
