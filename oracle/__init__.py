"""CPU oracle for the ResidualQuant hot path (test infrastructure only).

Importable only from tests/, __graft_entry__.smoke() and bench.py's CPU
baseline / reference arm.  Shares no code with the CUDA library.
"""
from .rq_oracle import *  # noqa: F401,F403
