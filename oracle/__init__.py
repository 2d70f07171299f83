"""CPU oracle for the retriever path -- test infrastructure, not product code.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
leg may import it.  It shares nothing with the CUDA library.
"""
from .retriever import *  # noqa: F401,F403
