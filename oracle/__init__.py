"""CPU oracle for the TokenGate pruned-prefill path.

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by
the CPU-baseline leg of bench.py.  The product path (learned_token_pruning_b200)
never imports it and has no CPU fallback.
"""
from .tokengate_oracle import *  # noqa: F401,F403
