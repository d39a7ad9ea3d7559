"""Shared-index top-k sparse KV attention for block-diffusion LLMs, on B200 (sm_100a).

The compute lives in ``libdsa.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/dsa.h``).  ``block_sparse_attention_27_b200.dsa`` is the thin
ctypes binding with the same names; it is imported lazily so that the input
generator (``workloads``) can be used without a GPU.
"""

__all__ = ["workloads"]
