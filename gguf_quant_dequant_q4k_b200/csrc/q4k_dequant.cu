// q4k_dequant.cu -- Q4_K superblocks -> row-major f32 (q4k_dequant_f32).
//
// The load-time "mirror" pass of "memra-engine 0.83.1, src/f16_ffi.rs"
// (`memra_q4_K_dequant_f16`, called from `build_q4k_f16_raw` with (w, dst,
// out_f, nsb_row, stream)), with an f32 target so every value is exact to one
// rounding and the result is bit-reproducible.
//
// Work mapping: a warp owns one superblock per step (the 144 bytes in, 1 KiB
// out). Lane L writes the 8 consecutive weights 8L..8L+7, which are 8
// consecutive bytes of Q, all in the low or all in the high nibbles of one
// 64-weight group, and all in one sub-block; so each lane does one 8-byte load
// of Q, one broadcast 16-byte load of the header and two 16-byte stores; the
// warp's stores cover 1 KiB contiguously. The kernel is HBM-bound on the
// 4 bytes/weight it writes (0.5625 read + 4 written per weight).
#include "q4k_internal.h"
#include "q4k_superblock.cuh"

namespace q4k {

namespace {

constexpr int kDequantThreads = 256;

__global__ void __launch_bounds__(kDequantThreads)
q4k_dequant_f32_kernel(const uint8_t* __restrict__ w, float* __restrict__ out,
                       long long total_sb) {
    const int lane = threadIdx.x & 31;
    const long long warp0 = (static_cast<long long>(blockIdx.x) * kDequantThreads + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * kDequantThreads) >> 5;
    const int g = lane >> 3;               // 64-weight group 0..3
    const int r = (lane & 7) * 8;          // first weight of this lane within the group
    const int high = r >= 32;              // weights 32..63 of the group: high nibbles
    const int l0 = r & 31;                 // byte offset within the group's 32 bytes
    const int j = 2 * g + high;            // sub-block
    for (long long s = warp0; s < total_sb; s += nwarps) {
        const uint8_t* sb = w + s * kBlockBytes;
        const Header hd = decode_header(ldg_nc_v4(sb));
        const uint2 qb = ldg_nc_v2(sb + kQsOffset + 32 * g + l0);
        float dsc, dm;
        subblock_coeffs(hd, j, dsc, dm);
        const int shift = high ? 4 : 0;
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t word = (e < 4) ? qb.x : qb.y;
            const uint32_t q = (word >> (8 * (e & 3) + shift)) & 15u;
            v[e] = weight_value(dsc, dm, q);
        }
        float4* dst = reinterpret_cast<float4*>(out + s * kQK + 8 * lane);
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
}

}  // namespace

int launch_dequant(const void* w, float* out, int n, int k, int num_sms, cudaStream_t stream) {
    const long long total_sb = static_cast<long long>(n) * (k / kQK);
    const long long warps_needed = total_sb;
    long long blocks = (warps_needed * 32 + kDequantThreads - 1) / kDequantThreads;
    const long long cap = static_cast<long long>(num_sms) * 8;  // 8 CTAs x 8 warps per SM
    if (blocks > cap) blocks = cap;
    q4k_dequant_f32_kernel<<<static_cast<unsigned>(blocks), kDequantThreads, 0, stream>>>(
        static_cast<const uint8_t*>(w), out, total_sb);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

}  // namespace q4k
