"""B200-native hierarchically pruned attention (HiP): mask + block-sparse attention.

The hot path lives in libhip_sparse.so (CUDA, sm_100a) behind the C ABI in
include/hip_sparse.h; ``binding`` marshals torch tensors into it. Importing
this package does not load the library; the first call through ``binding``
does, and raises if it is missing.
"""

__all__ = ["binding", "workloads", "build"]
