"""fp8_block_scaled_group_b200 — W8A8 FP8 block-scaled linear for B200 (sm_100a).

The compute lives in libfp8q.so (hand-written CUDA behind the C ABI in
include/fp8q.h); `api` marshals torch tensors into it. `inputs` holds the
seeded synthetic workloads.
"""
__all__ = ["api", "inputs"]
