"""B200-native DeepSeek-Sparse-Attention hot path (indexer -> top-2048 -> absorbed sparse MLA).

The compute lives in ``libdsa.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in include/dsa.h).  ``sparse_attention_16_b200.ops`` is a thin ctypes
binding with the same names; it loads the library on first use and raises if
it is missing: there is no CPU fallback.
"""

__all__ = ["accounting", "workloads"]
