"""HiLS-Attention hot path for NVIDIA B200 (sm_100a).

The compute lives in hand-written CUDA kernels behind the C ABI declared in include/hils.h
(libhils.so, built in-tree by `chunk_wise_hierarchical_summary_b200.build`). The Python
binding `chunk_wise_hierarchical_summary_b200.hils` only marshals torch tensors into that ABI;
it raises if the library is missing and never falls back to another implementation.
"""
__all__ = ["workloads"]
