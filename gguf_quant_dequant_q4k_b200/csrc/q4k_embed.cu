// q4k_embed.cu -- Q4_K embedding lookup and row gather (q4k_embed_lookup_f32,
// q4k_embed_gather_f32).
//
// The lookup of "turbospark-runtime 0.1.0, src/real_forward_dispatch.rs"
// (`encode_embed_lookup_q4_k(..., token, hidden, embed_scale)`, after
// `validate_q4_k_embedding`): one row of the table, dequantised, times
// embed_scale. The table checks run on the host before launch (q4k_api.cu);
// the gather reads its tokens from device memory and checks each one here.
//
// Work mapping: as in the dequant kernel, a warp owns one superblock of one
// output row per step and lane L writes weights 8L..8L+7 (one 8-byte quant
// load, a broadcast 16-byte header load, two 16-byte stores), so a warp writes
// 1 KiB contiguously. Each value is fl32(w * embed_scale) with w the f32
// weight d*sc*q - dmin*m (one rounding, exact products), so results are
// bit-reproducible.
#include "q4k_internal.h"
#include "q4k_superblock.cuh"

namespace q4k {

namespace {

// Set by the gather for a token outside the table; read and cleared by
// q4k_device_fault_flags().
__device__ unsigned int g_embed_fault_flags = 0;

constexpr int kEmbedThreads = 256;

// out[i*hidden + t] = row tokens[i] (or `token` when tokens is null) times scale.
__global__ void __launch_bounds__(kEmbedThreads)
q4k_embed_kernel(const uint8_t* __restrict__ table, long long rows, int nsb,
                 const int* __restrict__ tokens, unsigned token, int n_tokens, float scale,
                 float* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const long long warp0 = (static_cast<long long>(blockIdx.x) * kEmbedThreads + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * kEmbedThreads) >> 5;
    const long long total = static_cast<long long>(n_tokens) * nsb;
    const int g = lane >> 3;               // 64-weight group 0..3
    const int r = (lane & 7) * 8;          // first weight of this lane within the group
    const int high = r >= 32;              // weights 32..63 of the group: high nibbles
    const int l0 = r & 31;                 // byte offset within the group's 32 bytes
    const int j = 2 * g + high;            // sub-block
    for (long long s = warp0; s < total; s += nwarps) {
        const long long i = s / nsb;       // output row
        const int b = static_cast<int>(s - i * nsb);
        long long row = tokens != nullptr ? static_cast<long long>(__ldg(tokens + i)) : token;
        float4* dst = reinterpret_cast<float4*>(out + (i * nsb + b) * kQK + 8 * lane);
        if (row < 0 || row >= rows) {
            dst[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            dst[1] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane == 0) atomicOr(&g_embed_fault_flags, Q4K_FAULT_TOKEN_RANGE);
            continue;
        }
        const uint8_t* sb = table + (row * nsb + b) * kBlockBytes;
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
            v[e] = __fmul_rn(weight_value(dsc, dm, q), scale);
        }
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
}

}  // namespace

int launch_embed(const void* table, long long rows, int hidden, const int* tokens, unsigned token,
                 int n_tokens, float scale, float* out, int num_sms, cudaStream_t stream) {
    const int nsb = hidden / kQK;
    const long long warps_needed = static_cast<long long>(n_tokens) * nsb;
    long long blocks = (warps_needed * 32 + kEmbedThreads - 1) / kEmbedThreads;
    const long long cap = static_cast<long long>(num_sms) * 8;   // 8 CTAs x 8 warps per SM
    if (blocks > cap) blocks = cap;
    if (blocks < 1) return Q4K_OK;
    q4k_embed_kernel<<<static_cast<unsigned>(blocks), kEmbedThreads, 0, stream>>>(
        static_cast<const uint8_t*>(table), rows, nsb, tokens, token, n_tokens, scale, out);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

int read_embed_fault_flags(unsigned* flags) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_embed_fault_flags, sizeof(v));
    if (e != cudaSuccess) return cuda_failure(e);
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_embed_fault_flags, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_failure(e);
    *flags = v;
    return Q4K_OK;
}

}  // namespace q4k
