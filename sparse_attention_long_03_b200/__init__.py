"""B200-native DeepSeek Sparse Attention (DSA) hot path.

The compute path is ``libdsa.so`` (hand-written sm_100a CUDA behind a C ABI);
``sparse_attention_long_03_b200.dsa`` is its thin Python binding.  Nothing here
falls back to the CPU: if the library is missing, the binding raises.
"""

__all__ = ["workloads", "dsa"]
