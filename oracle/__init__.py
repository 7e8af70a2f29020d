"""CPU oracle of the DSA forward path: test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
leg import this package. The library (sparse_attention_long_tcgen05_b200)
never imports it and has no CPU fallback.
"""
from .dsa_oracle import *  # noqa: F401,F403
