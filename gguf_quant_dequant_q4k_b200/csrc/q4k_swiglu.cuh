// q4k_swiglu.cuh -- the SwiGLU epilogue of the fused gate/up GEMV:
// silu(g) * u with silu(g) = g / (1 + exp(-g)) ("realizar 0.8.5" kernel cache
// page: `FusedGateUpSwigluHwDp4aQ4KGemv { k: hidden_dim, n: intermediate_dim }`,
// gate and up projections of the same x followed by SwiGLU).
#pragma once

namespace q4k {

// expf is CUDA's accurate exponential (not the fast intrinsic); for g below
// about -88 it overflows to +inf and the quotient is -0, the limit of silu.
__device__ __forceinline__ float silu_mul(float g, float u) {
    return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
}

}  // namespace q4k
