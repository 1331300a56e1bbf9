"""CPU oracle for the MoE layer (test infrastructure; see moe_oracle.py, and ref.py for
the plain C++ restatement of the forward path that the CPU tests check it against).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and reference legs
import this package. The product path (grouped_ffn_moe_b200) never imports it.
"""
from .moe_oracle import *  # noqa: F401,F403
