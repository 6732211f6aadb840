"""Float64 CPU oracle for the cascade-pruned attention path (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import this package.
The CUDA library never imports, links or runs anything here.
"""
from . import spatten_ref  # noqa: F401
