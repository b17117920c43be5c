"""Sparse MoE FFN block forward on B200 (sm_100a).

The CUDA library sits behind a C ABI (include/moe.h); `sparse_moe_ffn_gemv_b200.moe`
is its thin Python binding. Importing this package does not load the library;
`inputs` (shapes and seeded synthetic inputs) needs no GPU.
"""
__all__ = ["inputs", "moe"]
