// q4k_superblock.cuh -- device-side decoding of one GGUF Q4_K superblock.
//
// A superblock holds 256 weights in 144 bytes ("memra-engine 0.83.1,
// src/f16_ffi.rs": `memra_q4_K_dequant_f16` takes "GGUF Q4_K 144B superblocks";
// `build_q8_f16` checks row_bytes == (in_f/256)*144). The field layout is GGUF's
// block_q4_K, which the pages do not print:
//   bytes 0..1 d (binary16), 2..3 dmin (binary16), 4..15 twelve bytes S holding
//   eight 6-bit scales sc_j and eight 6-bit mins m_j, 16..143 128 bytes Q of
//   4-bit quants; byte Q[32g+l] holds weight 64g+l (low nibble) and weight
//   64g+32+l (high nibble); weight t is in sub-block j = t/32 and its value is
//   d*sc_j*q_t - dmin*m_j.
//
// Everything here works on registers: a 16-byte header word (d, dmin, S) and
// 16-byte slices of Q.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace q4k {

constexpr int kQK = 256;          // weights per superblock
constexpr int kBlockBytes = 144;  // bytes per superblock
constexpr int kQsOffset = 16;     // byte offset of the 128 quant bytes

// d and dmin as f32 (exact: binary16 values are a subset of f32) and the
// 16 six-bit fields, one per byte, in four words:
//   sc_lo bytes = sc_0..3, sc_hi bytes = sc_4..7, m_lo = m_0..3, m_hi = m_4..7.
struct Header {
    float d, dmin;
    uint32_t sc_lo, sc_hi, m_lo, m_hi;
};

// `h` = bytes 0..15 of the superblock as four little-endian words:
// h.x = d | dmin << 16, h.y = S[0..3], h.z = S[4..7], h.w = S[8..11].
// Packing (GGUF get_scale_min_k4):
//   j < 4 : sc_j = S[j] & 63,                      m_j = S[j+4] & 63
//   j >= 4: sc_j = (S[j+4] & 15) | (S[j-4] >> 6) << 4,
//           m_j  = (S[j+4] >> 4) | (S[j]   >> 6) << 4
// done four fields at a time with byte-parallel masks.
__device__ __forceinline__ Header decode_header(uint4 h) {
    Header r;
    r.d = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x & 0xFFFFu)));
    r.dmin = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x >> 16)));
    r.sc_lo = h.y & 0x3F3F3F3Fu;
    r.m_lo = h.z & 0x3F3F3F3Fu;
    r.sc_hi = (h.w & 0x0F0F0F0Fu) | ((h.y >> 2) & 0x30303030u);
    r.m_hi = ((h.w >> 4) & 0x0F0F0F0Fu) | ((h.z >> 2) & 0x30303030u);
    return r;
}

__device__ __forceinline__ uint32_t byte_of(uint32_t word, int i) {
    return (word >> (8 * i)) & 0xFFu;
}

// Small non-negative integer (< 2^23) to f32, exactly, without the I2F pipe:
// 0x4B000000 is 2^23, so its bit pattern ORed with v is the float 2^23 + v.
__device__ __forceinline__ float small_u32_to_f32(uint32_t v) {
    return __uint_as_float(0x4B000000u | v) - 8388608.0f;
}

// (d*sc_j, dmin*m_j) of sub-block j (0..7). Both products are exact in f32.
__device__ __forceinline__ void subblock_coeffs(const Header& hd, int j, float& dsc, float& dm) {
    const uint32_t scw = (j < 4) ? hd.sc_lo : hd.sc_hi;
    const uint32_t mw = (j < 4) ? hd.m_lo : hd.m_hi;
    dsc = hd.d * small_u32_to_f32(byte_of(scw, j & 3));
    dm = hd.dmin * small_u32_to_f32(byte_of(mw, j & 3));
}

// Weight value d*sc*q - dmin*m rounded once (the product dsc*q is exact, so
// the fused and unfused forms agree bit for bit).
__device__ __forceinline__ float weight_value(float dsc, float dm, uint32_t q) {
    return fmaf(dsc, small_u32_to_f32(q), -dm);
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

}  // namespace q4k
