"""fp64 CPU oracle for the NABLA hot path (test infrastructure only).

Only tests/, the package smoke check in __graft_entry__.smoke() and the
benchmark's CPU-baseline leg may import this package.  The CUDA library and
its Python binding never do: the product path fails loudly when its CUDA
extension is missing instead of falling back to anything here.
"""
from .nabla_oracle import *  # noqa: F401,F403
from . import nabla_oracle  # noqa: F401
