"""DeepSeek Sparse Attention (DSA) forward path for one B200 (sm_100a).

The compute lives in ``libdsa.so`` (hand-written CUDA, C ABI declared in
include/dsa.h). ``sparse_attention_long_tcgen05_b200.dsa`` is the thin ctypes
binding; it loads the library on first use and raises if it is missing.
There is no CPU fallback.
"""
