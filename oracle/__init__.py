"""fp64 CPU oracle of the SparsePR per-call attention operator.

Test infrastructure only: imported by tests/, by the package's smoke check and by the
benchmark's CPU-baseline leg, never by the product path.  Shares no code with the CUDA path.
"""
from .sparsepr_oracle import *  # noqa: F401,F403
