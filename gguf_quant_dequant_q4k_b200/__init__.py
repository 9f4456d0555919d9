"""GGUF Q4_K GEMV (plain and fused gate/up SwiGLU), dequantisation and embedding
lookup on one NVIDIA B200 (sm_100a).

The computation runs in libq4k_b200.so (hand-written CUDA, C ABI in
include/q4k.h); this package is its ctypes binding (`capi`), which takes torch
tensors or raw device addresses. Importing it fails loudly if the library is
not built: there is no CPU path.
"""
from .capi import (  # noqa: F401
    EXPORTS, Q4K_BLOCK_BYTES, Q4K_GEMM_K_MULTIPLE, Q4K_ERR_ALIGN, Q4K_ERR_CUDA, Q4K_ERR_NULL, Q4K_ERR_OVERLAP,
    Q4K_ERR_RANGE, Q4K_ERR_SHAPE, Q4K_ERR_UNSUPPORTED_M, Q4K_FAULT_COPY_TIMEOUT,
    Q4K_FAULT_TOKEN_RANGE, Q4K_GEMV_X_READY, Q4K_KERNEL_I8, Q4K_KERNEL_STREAM, Q4K_KERNEL_TC, Q4K_KERNEL_WARP_ROWS,
    Q4K_MAX_M, Q4K_OK, Q4K_QK,
    LIB_PATH, Q4KError, q4k_dequant_f32, q4k_dequant_f32_status, q4k_device_fault_flags,
    q4k_embed_gather_f32, q4k_embed_gather_f32_status, q4k_embed_lookup_f32,
    q4k_embed_lookup_f32_status, q4k_gemv, q4k_gemv_plan_for, q4k_gemv_status,
    q4k_gemv_swiglu, q4k_gemv_swiglu_plan_for, q4k_gemv_swiglu_status,
    q4k_last_cuda_error, q4k_selftest_wait_timeout, q4k_status_string, q4k_weight_bytes,
    q4k_dequant_f16, q4k_dequant_f16_status, q4k_f32_to_f16, q4k_f32_to_f16_status,
    q4k_gemm_f16, q4k_gemm_f16_status, q4k_prefill_f16, q4k_prefill_f16_status,
    q4k_prefill_f16_noalloc, q4k_prefill_f16_noalloc_status, Q4K_ERR_CAPACITY,
    Q4K_PREFILL_NOALLOC_MAX_ELEMS,
)
