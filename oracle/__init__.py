"""CPU oracle for the OWQ mixed-precision weight-only matmul (fp64, numpy).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the CPU-baseline
leg of bench.py.  The CUDA library and its Python binding never import it.
"""
from .owq_oracle import *  # noqa: F401,F403
from .owq_oracle import __all__  # noqa: F401
