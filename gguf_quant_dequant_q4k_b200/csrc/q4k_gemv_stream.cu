// q4k_gemv_stream.cu -- the streaming Q4_K GEMV (plain, or fused gate/up
// SwiGLU) for m = 1, 2 and K <= 30720 (m = 1) or 15360 (m = 2).
//
// What it computes: y[i][r] = sum_k W[r][k] x[i][k] with W in Q4_K, as the
// pages' `Q4KGemv` / `TiledQ4KGemv` / `ChunkedTiledQ4KGemv` / `MwvQ4KGemv`
// family ("realizar 0.8.5, src/cuda/executor/q4k_gemv_cached.rs") and
// `BatchedQ4KGemv` ("realizar 0.8.5, src/cuda/executor/uses.rs"). The pages'
// designs stage x in shared memory per CTA (K*4 bytes, capped at 48 KB by
// `MAX_TILED_K`) and give each CTA 4 output rows; this kernel is laid out for
// B200 instead:
//
// * Work split. One persistent CTA per SM owns a balanced, contiguous range of
//   whole rows (counts differ by at most one). The CTA's compute warps form T
//   "teams"; the CTA's superblocks (rows x K/256, contiguous in memory) are
//   cut into T equal contiguous pieces at superblock granularity, one per
//   team, so every team streams the same number of bytes. A row cut between
//   two teams is finished from the teams' partial sums in shared memory, in
//   team order (deterministic; no atomics, no global workspace).
// * x-stationary. A team has ceil(K/1024) warps: team lane l owns the 16-byte
//   quant slice c = l%8 of superblock position b = l/8 of every row, i.e. 32
//   fixed weights of K (16 low nibbles of sub-block 2g and 16 high nibbles of
//   sub-block 2g+1, g = c/2). Its 32 x values per vector live in registers for
//   the whole kernel, so x costs no shared-memory bandwidth per row and there
//   is no K*4-byte shared-memory ceiling. For one vector on very tall
//   matrices, or K > 20480, a lane owns two adjacent slices (S = 2: 64
//   weights, ceil(K/2048) warps per team).
// * Streaming. Each team streams its byte range through a ring of `depth`
//   shared-memory stages with 1-D bulk async copies (cp.async.bulk, completing
//   on a "full" mbarrier; no multicast). A stage is up to 4 consecutive row
//   segments (one contiguous copy). Every weight byte is read from HBM once.
//   One producer warp per CTA (lane t serves team t) issues the copies, polls
//   each team's "done" mbarrier (one arrival per warp per stage), refills a
//   drained slot at once and then adds the warps' partials into y. Each team's
//   first stage is requested before griddepcontrol.wait, so under
//   programmatic dependent launch it overlaps the previous kernel's tail; the
//   rest of the ring follows once every compute warp has issued its x loads
//   (x is the dependent input, so it must not queue behind the ring).
// * Decode. Once per stage each warp decodes the headers of its superblocks
//   (d, dmin, 12 scale bytes; GGUF get_scale_min_k4 packing) into (A_j, B_j,
//   e_j) with A_j = 256*d*sc_j (exact), B_j = -fl(128*d*sc_j + dmin*m_j) and
//   e_j the exact rounding error of that sum (TwoSum). A weight with quant q is
//   formed as fma(A_j, f, B_j), f = 1/2 + q/256 built by one byte permute of
//   the masked nibble into the mantissa of 1/2 (exact): that is w + e_j
//   rounded once, w = d*sc_j*q - dmin*m_j. Each item then adds -e_j times the
//   sum of the lane's x over sub-block j (a per-lane constant, since x stays
//   in registers), so the error left per weight is the one rounding of w +
//   e_j, relative to |w| up to |e_j| <= 2^-24 (128*d*sc_j + dmin*m_j). Weights
//   and dot products use packed f32x2 FMAs.
// * Reduction. Per stage each lane holds one partial per row segment; a
//   4-segment transpose-reduce across the warp (5 shuffles) leaves one value
//   per segment, published to shared memory for the producer lane to add.
// * Fused gate/up SwiGLU (FUSED = true, q4k_gemv_swiglu): a CTA's rows of the
//   gate matrix followed by the same rows of the up matrix form one virtual
//   range that its teams cut as above (a stage crossing from gate into up rows
//   is two copies); row totals go to shared memory, and the CTA finishes with
//   y = silu(gate total) * (up total) for its rows ("realizar 0.8.5" kernel
//   cache page: `FusedGateUpSwigluHwDp4aQ4KGemv`).
//
// All waits are bounded: a wait that gives up raises a device fault flag
// (q4k_device_fault_flags) and the kernel skips its remaining work.
#include <cstdint>
#include <cuda_fp16.h>

#include "q4k_internal.h"
#include "q4k_sm100.cuh"
#include "q4k_stream.h"
#include "q4k_superblock.cuh"
#include "q4k_swiglu.cuh"

namespace q4k {

namespace {

// Set by a kernel whose bounded wait on a bulk copy gave up; read and cleared by
// q4k_device_fault_flags(). Never set in normal operation.
__device__ unsigned int g_fault_flags = 0;

constexpr int kSeg = kStreamSegRows;         // row segments per stage (a multiple of 4)
static_assert(kSeg % 4 == 0, "stages hold groups of four row segments");
constexpr unsigned kXIssuedBarrier = 1;      // named barrier: compute warps issued x loads
constexpr uint32_t kMagicOne = 0x3F000000u;  // 1/2: bytes 0..2 = 0x00, byte 3 = 0x3F
constexpr uint32_t kMagic2p23 = 0x4B000000u; // 2^23
// Coefficient buffer per warp: [segment][position][4 groups] float4s
// (A_2g, A_2g+1, B_2g, B_2g+1), then [segment][position][4 groups] float2s
// (-e_2g, -e_2g+1): B's rounding errors.
__host__ __device__ constexpr int coef_main_bytes_per_warp(int slices) {
    return kSeg * pos_per_warp(slices) * 4 * 16;
}
__host__ __device__ constexpr int coef_bytes_per_warp(int slices) {
    return kSeg * pos_per_warp(slices) * 4 * (16 + 8);
}

// f = 1/2 + q/256 for the nibble q held in byte SEL of `masked` (bytes 0..15):
// the byte becomes bits 16..23 of 0x3F000000 (1/2), i.e. mantissa bits 16..19.
template <int SEL>
__device__ __forceinline__ float nib_to_f(uint32_t masked) {
    return __uint_as_float(__byte_perm(masked, kMagicOne, 0x7054 | (SEL << 8)));
}

// 2^23 + (byte SEL of w), exactly.
template <int SEL>
__device__ __forceinline__ float byte_2p23(uint32_t w) {
    return __uint_as_float(__byte_perm(w, kMagic2p23, 0x7650 | SEL));
}

struct TeamRange {
    long long s0, s1;   // superblock range [s0, s1) in flat (row*nsb + b) units
    long long row0;     // first row touched
    int nseg;           // rows touched
    int nstages;
};
static_assert(sizeof(TeamRange) == kTeamRangeBytes, "team range table entry");

// Superblock range of cluster-global team `gteam` (= cta_rank * teams + team)
// of the calling CTA's cluster. The cluster owns a contiguous range of whole
// rows; its C * teams teams cut it into equal contiguous pieces. Boundaries are
// computed cluster-relative in 32 bits (a cluster's rows*nsb is far below
// 2^31 for any matrix whose N*K/256 fits the int arguments); only the cluster
// origin is 64-bit.
// FUSED (fused gate/up SwiGLU, cluster = 1): the CTA's rows of the gate
// matrix followed by the same rows of the up matrix form one virtual range of
// 2 * rows rows, indexed from 0 (CTA-relative); its teams cut that range.
template <bool FUSED>
__device__ __forceinline__ TeamRange team_range(const StreamParams& p, int gteam) {
    const int q = static_cast<int>(blockIdx.x) / p.cluster;
    const int crows = p.rows_base + (q < p.rows_extra ? 1 : 0);
    const int rows = FUSED ? 2 * crows : crows;
    const long long row_begin = FUSED ? 0 :
        static_cast<long long>(q) * p.rows_base + (q < p.rows_extra ? q : p.rows_extra);
    const int L = rows * p.nsb;
    const unsigned nt = static_cast<unsigned>(p.cluster * p.teams);
    int b, e;
    if (static_cast<unsigned>(L) <= 0xFFFFFFFFu / nt) {   // products fit 32 bits
        b = static_cast<int>(static_cast<unsigned>(L) * gteam / nt);
        e = static_cast<int>(static_cast<unsigned>(L) * (gteam + 1) / nt);
    } else {
        b = static_cast<int>((static_cast<unsigned long long>(L) * gteam) / nt);
        e = static_cast<int>((static_cast<unsigned long long>(L) * (gteam + 1)) / nt);
    }
    TeamRange r;
    r.s0 = row_begin * p.nsb + b;
    r.s1 = row_begin * p.nsb + e;
    if (e > b) {
        const int rb = b / p.nsb;                 // cluster-relative first row
        r.row0 = row_begin + rb;
        r.nseg = (e - 1) / p.nsb - rb + 1;
        r.nstages = (r.nseg + kSeg - 1) / kSeg;
    } else {
        r.row0 = 0;
        r.nseg = 0;
        r.nstages = 0;
    }
    return r;
}

// First row and row count of the calling CTA's share (cluster = 1).
__device__ __forceinline__ void cta_rows(const StreamParams& p, long long& row0, int& rows) {
    const int q = static_cast<int>(blockIdx.x);
    rows = p.rows_base + (q < p.rows_extra ? 1 : 0);
    row0 = static_cast<long long>(q) * p.rows_base + (q < p.rows_extra ? q : p.rows_extra);
}

__device__ __forceinline__ long long seg_begin(const TeamRange& r, int i, int nsb) {
    const long long b = (r.row0 + i) * nsb;
    return b > r.s0 ? b : r.s0;
}

__device__ __forceinline__ long long seg_end(const TeamRange& r, int i, int nsb) {
    const long long e = (r.row0 + i + 1) * nsb;
    return e < r.s1 ? e : r.s1;
}


__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
    return __fadd2_rn(a, make_float2(-b.x, -b.y));
}

// (A_2g, A_2g+1, B_2g, B_2g+1) for the two 64-weight groups g = 2*half and
// 2*half+1 of one superblock header h (bytes 0..15), with A_j = 256*d*sc_j and
// B_j = -fl(128*d*sc_j + dmin*m_j), so that A_j*(1/2 + q/256) + B_j =
// d*sc_j*q - dmin*m_j + e_j, where e_j = 128*d*sc_j + dmin*m_j - fl(...) is
// the rounding error of B_j. A_j and both products are exact, and e_j is
// recovered exactly (TwoSum); `err` receives (-e_4h, -e_4h+1, -e_4h+2,
// -e_4h+3). The weight the fma rounds is then w + e_j, rounded once; the
// caller removes e_j's contribution as -e_j * (sum of the lane's x over
// sub-block j), so the error left per weight is that one rounding of
// w + e_j (|e_j| is at most half an ulp of 128*d*sc_j + dmin*m_j).
__device__ __forceinline__ void decode_half(uint4 h, float d, float dmin, int half, float4& out0,
                                            float4& out1, float4& err) {
    // six-bit fields of sub-blocks 4*half .. +3 (GGUF get_scale_min_k4 packing)
    const uint32_t sc = half ? ((h.w & 0x0F0F0F0Fu) | ((h.y >> 2) & 0x30303030u))
                             : (h.y & 0x3F3F3F3Fu);
    const uint32_t mm = half ? (((h.w >> 4) & 0x0F0F0F0Fu) | ((h.z >> 2) & 0x30303030u))
                             : (h.z & 0x3F3F3F3Fu);
    const float d128 = d * 128.0f;
    // (2^23 + v) * s - 2^23 * s == v * s exactly for the 6-bit v and these s.
    const float2 sa = make_float2(d128, d128);
    const float2 sb2 = make_float2(-8388608.0f * d128, -8388608.0f * d128);
    const float2 ma = make_float2(dmin, dmin);
    const float2 mb = make_float2(-8388608.0f * dmin, -8388608.0f * dmin);
    const float2 a01 = ffma2(sa, make_float2(byte_2p23<0>(sc), byte_2p23<1>(sc)), sb2);  // 128 d sc
    const float2 a23 = ffma2(sa, make_float2(byte_2p23<2>(sc), byte_2p23<3>(sc)), sb2);
    const float2 m01 = ffma2(ma, make_float2(byte_2p23<0>(mm), byte_2p23<1>(mm)), mb);  // dmin m
    const float2 m23 = ffma2(ma, make_float2(byte_2p23<2>(mm), byte_2p23<3>(mm)), mb);
    const float2 A01 = __fadd2_rn(a01, a01), A23 = __fadd2_rn(a23, a23);
    const float2 s01 = __fadd2_rn(a01, m01), s23 = __fadd2_rn(a23, m23);
    // TwoSum: e = (a + m) - s exactly, without assuming |a| >= |m|.
    const float2 v01 = fsub2(s01, a01), v23 = fsub2(s23, a23);
    const float2 e01 = __fadd2_rn(fsub2(a01, fsub2(s01, v01)), fsub2(m01, v01));
    const float2 e23 = __fadd2_rn(fsub2(a23, fsub2(s23, v23)), fsub2(m23, v23));
    out0 = make_float4(A01.x, A01.y, -s01.x, -s01.y);
    out1 = make_float4(A23.x, A23.y, -s23.x, -s23.y);
    err = make_float4(-e01.x, -e01.y, -e23.x, -e23.y);
}

// kWords consecutive 32-bit words of quant bytes from shared memory (one
// 8- or 16-byte load per 16 bytes).
template <int kWords>
__device__ __forceinline__ void load_words(const uint8_t* smem, uint32_t addr, uint32_t (&w)[kWords]) {
    if (kWords == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(smem + addr);
        w[0] = v.x;
        w[1 % kWords] = v.y;
    } else {
#pragma unroll
        for (int j = 0; j < kWords / 4; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(smem + addr + 16 * j);
            w[(4 * j + 0) % kWords] = v.x;
            w[(4 * j + 1) % kWords] = v.y;
            w[(4 * j + 2) % kWords] = v.z;
            w[(4 * j + 3) % kWords] = v.w;
        }
    }
}

__device__ __forceinline__ void header_scales(uint4 h, float& d, float& dmin) {
    d = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x & 0xFFFFu)));
    dmin = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x >> 16)));
}

// One 32-bit word of quants (bytes e = 0..3; low nibble = weight of sub-block
// 2g, high nibble = weight of sub-block 2g+1) against x pairs xp[i][e0 + e]:
// the two nibbles of a byte form one f32x2 lane pair with coefficients
// a = (A_2g, A_2g+1), b = (B_2g, B_2g+1). Accumulates into acc[i], one chain
// per vector (measured faster on B200 than four split chains: fewer
// instructions, and the other warps hide the chain's latency); `first`
// initialises the chain.
template <int M, int NX>
__device__ __forceinline__ void dot_word(uint32_t w, float2 a, float2 b, const float2 (&xp)[M][NX],
                                         int e0, bool first, float2 (&acc)[M]) {
    const uint32_t lo = w & 0x0F0F0F0Fu;
    const uint32_t hi = __umulhi(w, 1u << 28) & 0x0F0F0F0Fu;   // (w >> 4) on the FMA pipe
    float2 w0 = ffma2(a, make_float2(nib_to_f<0>(lo), nib_to_f<0>(hi)), b);
    float2 w1 = ffma2(a, make_float2(nib_to_f<1>(lo), nib_to_f<1>(hi)), b);
    float2 w2 = ffma2(a, make_float2(nib_to_f<2>(lo), nib_to_f<2>(hi)), b);
    float2 w3 = ffma2(a, make_float2(nib_to_f<3>(lo), nib_to_f<3>(hi)), b);
#pragma unroll
    for (int i = 0; i < M; ++i) {
        acc[i] = first ? __fmul2_rn(w0, xp[i][e0 + 0]) : ffma2(w0, xp[i][e0 + 0], acc[i]);
        acc[i] = ffma2(w1, xp[i][e0 + 1], acc[i]);
        acc[i] = ffma2(w2, xp[i][e0 + 2], acc[i]);
        acc[i] = ffma2(w3, xp[i][e0 + 3], acc[i]);
    }
}

// 4 values per lane -> each lane holds the warp sum of value index
// ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1).
__device__ __forceinline__ float transpose_reduce4(float s0, float s1, float s2, float s3,
                                                   int lane) {
    const bool up = (lane & 16) != 0;
    float a0 = up ? s2 : s0, a1 = up ? s3 : s1;
    const float b0 = up ? s0 : s2, b1 = up ? s1 : s3;
    a0 += __shfl_xor_sync(0xFFFFFFFFu, b0, 16);
    a1 += __shfl_xor_sync(0xFFFFFFFFu, b1, 16);
    const bool up8 = (lane & 8) != 0;
    float k = up8 ? a1 : a0;
    const float snd = up8 ? a0 : a1;
    k += __shfl_xor_sync(0xFFFFFFFFu, snd, 8);
    k += __shfl_xor_sync(0xFFFFFFFFu, k, 4);
    k += __shfl_xor_sync(0xFFFFFFFFu, k, 2);
    k += __shfl_xor_sync(0xFFFFFFFFu, k, 1);
    return k;
}


__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ int cta_rank(const StreamParams& p) {
    return static_cast<int>(blockIdx.x) % p.cluster;
}

// Cluster-wide barrier with release/acquire semantics for shared memory.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A float at the same shared-memory address in CTA `rank` of the cluster.
__device__ __forceinline__ float ld_dsmem(const float* local, int rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(remote)
                 : "r"(smem_addr(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Per-team view of the kernel's shared memory and work range.
struct Team {
    TeamRange tr;
    int head0;          // row-relative index of the team's first superblock
    int team_len;       // superblocks in the team's range
    const uint8_t* w;   // W at the team's first superblock
    uint8_t* ring;      // depth slots of stage_bytes
    float* red;         // [depth][2 phases][team_warps][M][kSeg] warp partials
    uint64_t* full;     // [depth] stage landed (1 arrival + bytes)
    uint64_t* done;     // [depth] stage consumed (team_warps arrivals)
    long long cta_row0; // fused: the CTA's first row and row count
    int cta_rows;
};

template <int M, bool FUSED>
__device__ __forceinline__ Team make_team(const StreamParams& p, uint8_t* smem, int team) {
    Team t;
    if (FUSED) {
        cta_rows(p, t.cta_row0, t.cta_rows);
    } else {
        t.cta_row0 = 0;
        t.cta_rows = 0;
    }
    t.tr = reinterpret_cast<const TeamRange*>(smem + p.off_tr)[cta_rank(p) * p.teams + team];
    t.head0 = static_cast<int>(t.tr.s0 - t.tr.row0 * p.nsb);
    t.team_len = static_cast<int>(t.tr.s1 - t.tr.s0);
    t.w = FUSED ? p.w : p.w + t.tr.s0 * kBlockBytes;
    t.ring = smem + static_cast<size_t>(team) * p.depth * p.stage_bytes;
    t.red = reinterpret_cast<float*>(smem + p.off_red) +
            static_cast<size_t>(team) * p.depth * 2 * p.team_warps * kSeg * M;
    t.full = reinterpret_cast<uint64_t*>(smem + p.off_bar) + static_cast<size_t>(team) * 2 * p.depth;
    t.done = t.full + p.depth;
    return t;
}

// Stage with first row start rb (team-relative) -> one bulk copy into `slot`;
// FUSED: two copies where the stage crosses from gate rows into up rows.
template <bool FUSED>
__device__ __forceinline__ void issue_stage(const Team& T, const StreamParams& p, int rb, int slot) {
    const int span = kSeg * p.nsb;
    const int b_rel = rb > 0 ? rb : 0;
    const int e_rel = (rb + span) < T.team_len ? (rb + span) : T.team_len;
    const uint32_t bytes = static_cast<uint32_t>(e_rel - b_rel) * kBlockBytes;
    mbar_arrive_expect_tx(&T.full[slot], bytes);
    uint8_t* dst = T.ring + static_cast<size_t>(slot) * p.stage_bytes;
    if (!FUSED) {
        if (p.nsb_row == p.nsb && p.sb_off == 0) {   // contiguous rows: one copy
            bulk_copy_g2s(dst, T.w + static_cast<size_t>(b_rel) * kBlockBytes, bytes, &T.full[slot]);
            return;
        }
        // a K-chunk of longer rows: one copy per row segment, from row r's
        // superblocks sb_off + col of its nsb_row
        long long vs = T.tr.s0 + b_rel;
        const long long ve = T.tr.s0 + e_rel;
        while (vs < ve) {
            const long long r = vs / p.nsb;
            const long long c = vs - r * p.nsb;
            const long long e = ve < (r + 1) * p.nsb ? ve : (r + 1) * p.nsb;
            const uint32_t nb = static_cast<uint32_t>(e - vs) * kBlockBytes;
            bulk_copy_g2s(dst, p.w + static_cast<size_t>(r * p.nsb_row + p.sb_off + c) * kBlockBytes,
                          nb, &T.full[slot]);
            dst += nb;
            vs = e;
        }
        return;
    }
    long long vs = T.tr.s0 + b_rel;                               // virtual, CTA-relative
    const long long ve = T.tr.s0 + e_rel;
    const long long bound = static_cast<long long>(T.cta_rows) * p.nsb;   // gate | up
    const long long base = T.cta_row0 * p.nsb;
    if (vs < bound) {
        const long long e1 = ve < bound ? ve : bound;
        const uint32_t nb = static_cast<uint32_t>(e1 - vs) * kBlockBytes;
        bulk_copy_g2s(dst, p.w + static_cast<size_t>(base + vs) * kBlockBytes, nb, &T.full[slot]);
        dst += nb;
        vs = e1;
    }
    if (vs < ve)
        bulk_copy_g2s(dst, p.w_up + static_cast<size_t>(base + vs - bound) * kBlockBytes,
                      static_cast<uint32_t>(ve - vs) * kBlockBytes, &T.full[slot]);
}

// Where a finished row total goes: y, or (FUSED) the CTA's row-total buffer,
// gate rows at 0..rows-1 and up rows at rows..2*rows-1 (virtual row index).
template <bool FUSED>
__device__ __forceinline__ float& row_out_ref(const StreamParams& p, uint8_t* smem, int i,
                                              long long row) {
    if (FUSED)
        return reinterpret_cast<float*>(smem + p.off_rows)[static_cast<size_t>(i) * 2 * p.rows_cap + row];
    return p.y[static_cast<size_t>(i) * p.n + row];
}

// Finishes row `row` of vector i: y = tot, or y += tot for a later K-chunk.
template <bool FUSED>
__device__ __forceinline__ void store_row(const StreamParams& p, uint8_t* smem, int i, long long row,
                                          float tot) {
    float& r = row_out_ref<FUSED>(p, smem, i, row);
    r = p.accumulate ? r + tot : tot;
}

// M vectors, S 16-byte quant slices (S*32 weights) per lane per row.
template <int M, int S, bool FUSED>
__global__ void __maxnreg__(stream_max_regs(M, S))
q4k_gemv_stream_kernel(const StreamParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ volatile int abort_flag;
    constexpr int kLanesPerSb = lanes_per_sb(S);   // lanes covering one superblock of a row
    constexpr int kPos = pos_per_warp(S);          // superblock positions per warp
    constexpr int kNX = lane_bytes(S);             // x pairs per lane per vector
    constexpr int kWords = kNX / 4;                // 32-bit quant words per lane and row
    const int nsb = p.nsb;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int compute_warps = p.teams * p.team_warps;
    float* part = reinterpret_cast<float*>(smem + p.off_part);   // [teams][2][M]

    if (threadIdx.x == 0) abort_flag = 0;
    {
        // barriers [team][full, done][depth]: one per thread
        const int nbar = 2 * p.teams * p.depth;
        const int i = static_cast<int>(threadIdx.x);
        if (i < nbar) {
            uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
            mbar_init(&bars[i], ((i / p.depth) & 1) ? p.team_warps : 1);
            fence_mbar_init();
        }
        if (i < p.teams * 2 * M) part[i] = 0.f;
        // superblock ranges of every team of the cluster (64-bit divisions once)
        if (i < p.cluster * p.teams)
            reinterpret_cast<TeamRange*>(smem + p.off_tr)[i] = team_range<FUSED>(p, i);
    }
    __syncthreads();

    if (warp == compute_warps) {
        // ------------------------------------------------------------ producer
        // Lane t < teams owns team t's ring: it issues the team's copies, and
        // as soon as every warp of the team has consumed a stage it adds the
        // warps' partials into y (or a cut row's partial) and refills the slot.
        const bool own = lane < p.teams;
        Team T;
        int nst = 0;
        if (own) {
            T = make_team<M, FUSED>(p, smem, lane);
            nst = T.tr.nstages;
            const int all = nst < p.depth ? nst : p.depth;
            const int pre = all < kStreamPreStages ? all : kStreamPreStages;
            for (int s = 0; s < pre; ++s) issue_stage<FUSED>(T, p, s * kSeg * nsb - T.head0, s);
        }
        pdl_launch_dependents();
        pdl_wait();
        // x first: wait until every compute warp has issued its x loads.
        named_barrier_sync(kXIssuedBarrier, blockDim.x);
        if (own) {
            const int all = nst < p.depth ? nst : p.depth;
            const int pre = all < kStreamPreStages ? all : kStreamPreStages;
            for (int s = pre; s < all; ++s) issue_stage<FUSED>(T, p, s * kSeg * nsb - T.head0, s);
        }
        int tf = 0, fslot = 0;
        uint32_t fphase = 0;
        int rbf = own ? -T.head0 : 0;
        unsigned idle = 0;
        const int red_slot = p.team_warps * kSeg * M;
        for (;;) {
            const bool active = own && tf < nst && !abort_flag;
            if (!__any_sync(0xFFFFFFFFu, active)) break;
            bool progressed = false;
            if (active && mbar_test_wait(&T.done[fslot], fphase)) {
                // Refill the drained slot at once: its quant bytes are consumed,
                // and its partial sums sit in the (slot, phase) half of the
                // team's buffer, which the refilled stage does not write.
                if (tf + p.depth < nst) issue_stage<FUSED>(T, p, rbf + p.depth * kSeg * nsb, fslot);
                const float* rbuf = T.red + static_cast<size_t>(fslot * 2 + fphase) * red_slot;
                // Sum the team's warp partials: warp wi's M*kSeg values are
                // consecutive ([wi][i][u]), so each warp's block is read as
                // float4s, the loads of several warps in flight before their
                // adds (warp order, as a serial sum would add them).
                constexpr int kVals = M * kSeg;
                float tot[kVals];
#pragma unroll
                for (int v = 0; v < kVals; ++v) tot[v] = 0.f;
#pragma unroll 4
                for (int wi = 0; wi < p.team_warps; ++wi) {
                    const float4* src = reinterpret_cast<const float4*>(rbuf + wi * kVals);
#pragma unroll
                    for (int v4 = 0; v4 < kVals / 4; ++v4) {
                        const float4 t = src[v4];
                        tot[4 * v4 + 0] += t.x;
                        tot[4 * v4 + 1] += t.y;
                        tot[4 * v4 + 2] += t.z;
                        tot[4 * v4 + 3] += t.w;
                    }
                }
#pragma unroll
                for (int u = 0; u < kSeg; ++u) {
                    if (tf * kSeg + u >= T.tr.nseg) break;
                    const int r0 = rbf + u * nsb;              // team-relative row start
                    const int b = (r0 > 0 ? r0 : 0) - r0;      // row-relative segment bounds
                    const int e = ((r0 + nsb) < T.team_len ? (r0 + nsb) : T.team_len) - r0;
                    const long long row = T.tr.row0 + tf * kSeg + u;
#pragma unroll
                    for (int i = 0; i < M; ++i) {
                        if (b == 0 && e == nsb)
                            store_row<FUSED>(p, smem, i, row, tot[i * kSeg + u]);
                        else
                            part[(lane * 2 + (b > 0 ? 0 : 1)) * M + i] = tot[i * kSeg + u];
                    }
                }
                ++tf;
                rbf += kSeg * nsb;
                if (++fslot == p.depth) {
                    fslot = 0;
                    fphase ^= 1u;
                }
                progressed = true;
                idle = 0;
            } else if (active && ++idle > kSpinLimit) {
                atomicOr(&g_fault_flags, kFaultCopyTimeout);
                abort_flag = 1;
            }
            if (!__any_sync(0xFFFFFFFFu, progressed)) __nanosleep(64);
        }
        // After a lost copy, give the copies still in flight a bounded chance
        // to land before the CTA's shared memory is released. Stages [0, tf)
        // were consumed; the ring holds the issued stages [tf, min(tf + depth,
        // nst)), stage s completing phase (s / depth) & 1 of full[s % depth].
        if (own && abort_flag) {
            const int last = tf + p.depth < nst ? tf + p.depth : nst;
            for (int s = tf; s < last; ++s)
                mbar_wait_bounded(&T.full[s % p.depth], static_cast<uint32_t>((s / p.depth) & 1),
                                  &g_fault_flags);
        }
    } else {
        // ------------------------------------------------------------ compute
        const int team = warp / p.team_warps;
        const int wit = warp % p.team_warps;
        const Team T = make_team<M, FUSED>(p, smem, team);
        pdl_launch_dependents();
        // x belongs to the dependency chain unless the caller says otherwise;
        // these warps write only shared memory (the producer, which stores
        // y, waits in any case)
        if (!p.x_ready) pdl_wait();

        // This lane's superblock position bl and its kNX quant bytes, from
        // byte qoff of the superblock's 128: group g = qoff / 32 (sub-blocks
        // 2g, 2g+1), bytes b0 .. b0 + kNX - 1 of the group's 32.
        const int lpos = lane / kLanesPerSb;
        const int qoff = (lane % kLanesPerSb) * kNX;
        const int g = qoff >> 5;
        const int b0 = qoff & 31;
        const int bl = wit * kPos + lpos;
        const bool valid = bl < nsb;
        // xp[i][e] = (x of the low nibble of byte e of the lane's quant bytes, x
        // of its high nibble): weights k0 + e and k0 + 32 + e.
        float2 xp[M][kNX];
        {
            // A lane past the last superblock position loads position 0's x
            // (its products are discarded), so the loads need no branch and
            // their latency overlaps the first stage's wait and decode. Plain
            // (coherent, L1-allocating) loads: measured on B200 the
            // non-coherent path made the K = 14336 call 10 % slower.
            const int k0 = (valid ? bl : 0) * kQK + 64 * g + b0;
#pragma unroll
            for (int i = 0; i < M; ++i) {
                const float4* xl = reinterpret_cast<const float4*>(
                    p.x + static_cast<size_t>(i) * p.x_stride + k0);
                const float4* xh = xl + 8;   // + 32 weights
#pragma unroll
                for (int v = 0; v < kNX / 4; ++v) {
                    const float4 a = xl[v], b = xh[v];
                    xp[i][4 * v + 0] = make_float2(a.x, b.x);
                    xp[i][4 * v + 1] = make_float2(a.y, b.y);
                    xp[i][4 * v + 2] = make_float2(a.z, b.z);
                    xp[i][4 * v + 3] = make_float2(a.w, b.w);
                }
            }
        }
        named_barrier_arrive(kXIssuedBarrier, blockDim.x);
        // Per vector, the sums of the lane's low-nibble x values (sub-block
        // 2g) and high-nibble x values (sub-block 2g+1).
        float2 sx[M];
#pragma unroll
        for (int i = 0; i < M; ++i) {
            sx[i] = xp[i][0];
#pragma unroll
            for (int e = 1; e < kNX; ++e) sx[i] = __fadd2_rn(sx[i], xp[i][e]);
        }

        // Shared-memory byte offsets (32-bit). The coefficient float4 of
        // (segment u, position pos, group g) sits at (u*kPos + pos)*4 +
        // (g ^ ((pos >> 1) & 3)): conflict-free for decode stores and item loads.
        const int span = kSeg * nsb;
        const uint32_t ring_off = static_cast<uint32_t>(T.ring - smem);
        const uint32_t lane_qoff = static_cast<uint32_t>(bl * kBlockBytes + kQsOffset + qoff);
        const uint32_t coef_off = static_cast<uint32_t>(p.off_coef) +
                                  static_cast<uint32_t>(warp) * static_cast<uint32_t>(coef_bytes_per_warp(S));
        const uint32_t lane_coef_off =
            coef_off + static_cast<uint32_t>((lpos * 4 + (g ^ ((lpos >> 1) & 3))) * 16);
        // Decode lanes: S = 2: lane -> (segment du, position dpos), whole header;
        // S = 1: lane -> (segment du, position dpos, half dhalf).
        const int du = lane >> 3;
        const int dpos = S == 2 ? (lane & 7) : ((lane >> 1) & 3);
        const int dhalf = S == 1 ? (lane & 1) : 0;
        const int dbl = wit * kPos + dpos;
        const uint32_t dec_base = coef_off + static_cast<uint32_t>((du * kPos + dpos) * 4 * 16);
        const int dswz = (dpos >> 1) & 3;
        // B's rounding errors: float2 (-e_2g, -e_2g+1) of (segment, position,
        // group) at err_off + ((u*kPos + pos)*4 + g)*8 (unswizzled: the item
        // loads of a warp read 16 consecutive float2s, decode stores 16-byte runs).
        const uint32_t err_off = coef_off + static_cast<uint32_t>(coef_main_bytes_per_warp(S));
        const uint32_t dec_err = err_off + static_cast<uint32_t>((du * kPos + dpos) * 4 * 8);
        const uint32_t lane_err_off = err_off + static_cast<uint32_t>((lpos * 4 + g) * 8);
        const int red_slot = p.team_warps * kSeg * M;

        int slot = 0;
        uint32_t phase = 0;
        int rb = -T.head0;   // team-relative index of stage s's first row start
        for (int s = 0; s < T.tr.nstages; ++s, rb += span) {
            const uint32_t st_off = ring_off + static_cast<uint32_t>(slot) * p.stage_bytes;
            const int b_rel = rb > 0 ? rb : 0;
            const int e_rel = (rb + span) < T.team_len ? (rb + span) : T.team_len;
            const int nsb_stage = e_rel - b_rel;
            const int head = b_rel - rb;   // row-relative index of the stage's first superblock

            if (!abort_flag && !mbar_wait_bounded(&T.full[slot], phase, &g_fault_flags))
                abort_flag = 1;

            // Decode this warp's superblock headers of the stage (segments
            // du, du + 4, ...).
#pragma unroll
            for (int dg = 0; dg < kSeg / 4; ++dg) {
                const int idx = (du + 4 * dg) * nsb + dbl - head;
                if (dbl < nsb && static_cast<unsigned>(idx) < static_cast<unsigned>(nsb_stage)) {
                    const uint4 hdr = *reinterpret_cast<const uint4*>(
                        smem + st_off + static_cast<uint32_t>(idx) * kBlockBytes);
                    float d, dmin;
                    header_scales(hdr, d, dmin);
                    const uint32_t cb = dec_base + static_cast<uint32_t>(dg * 4 * kPos * 4 * 16);
                    const uint32_t eb = dec_err + static_cast<uint32_t>(dg * 4 * kPos * 4 * 8);
#pragma unroll
                    for (int hh = 0; hh < S; ++hh) {
                        const int half = S == 2 ? hh : dhalf;
                        float4 c_a, c_b, c_e;
                        decode_half(hdr, d, dmin, half, c_a, c_b, c_e);
                        *reinterpret_cast<float4*>(smem + cb + ((2 * half) ^ dswz) * 16) = c_a;
                        *reinterpret_cast<float4*>(smem + cb + ((2 * half + 1) ^ dswz) * 16) = c_b;
                        *reinterpret_cast<float4*>(smem + eb + half * 16) = c_e;
                    }
                }
            }
            __syncwarp();

            // The stage's (up to) kSeg row segments. Segments past the team's
            // last row are skipped (a warp-uniform branch); inside a segment a
            // lane whose superblock is not in it computes on superblock 0 and
            // the result is discarded by a select. Item u + 1's operands are
            // loaded while item u computes.
            bool use[kSeg];
            uint32_t qaddr[kSeg];
#pragma unroll
            for (int u = 0; u < kSeg; ++u) {
                const int idx = u * nsb - head + bl;
                use[u] = valid && static_cast<unsigned>(idx) < static_cast<unsigned>(nsb_stage);
                qaddr[u] = st_off + (use[u] ? lane_qoff + static_cast<uint32_t>((u * nsb - head) * kBlockBytes)
                                            : static_cast<uint32_t>(kQsOffset + qoff));
            }
            const int nseg_s = T.tr.nseg - s * kSeg < kSeg ? T.tr.nseg - s * kSeg : kSeg;
            float part_sum[M][kSeg];
            uint32_t qn[kWords];
            load_words<kWords>(smem, qaddr[0], qn);
            float4 cfn = *reinterpret_cast<const float4*>(smem + lane_coef_off);
            // Item u: the lane's slice of segment u; loads item u + 1's operands
            // first if `next`.
            auto item = [&](const int u, const bool next) {
                uint32_t q[kWords];
#pragma unroll
                for (int j = 0; j < kWords; ++j) q[j] = qn[j];
                const float4 cf = cfn;
                // used after the item's dot products: loaded here, not a step ahead
                const float2 ne = *reinterpret_cast<const float2*>(smem + lane_err_off + u * kPos * 32);
                if (next) {
                    load_words<kWords>(smem, qaddr[u + 1], qn);
                    cfn = *reinterpret_cast<const float4*>(smem + lane_coef_off + (u + 1) * kPos * 64);
                }
                const float2 a = make_float2(cf.x, cf.y), b = make_float2(cf.z, cf.w);
                float2 acc[M];
#pragma unroll
                for (int j = 0; j < kWords; ++j)
                    dot_word<M, kNX>(q[j], a, b, xp, 4 * j, j == 0, acc);
#pragma unroll
                for (int i = 0; i < M; ++i) {
                    acc[i] = ffma2(ne, sx[i], acc[i]);   // remove B's rounding error
                    part_sum[i][u] = use[u] ? (acc[i].x + acc[i].y) : 0.f;
                }
            };
            if (nseg_s == kSeg) {
#pragma unroll
                for (int u = 0; u < kSeg; ++u) item(u, u + 1 < kSeg);
            } else {
#pragma unroll
                for (int u = 0; u < kSeg; ++u) {
                    if (u < nseg_s) {
                        item(u, u + 1 < nseg_s);
                    } else {
#pragma unroll
                        for (int i = 0; i < M; ++i) part_sum[i][u] = 0.f;
                    }
                }
            }
            float* rbuf = T.red + static_cast<size_t>(slot * 2 + phase) * red_slot;
#pragma unroll
            for (int i = 0; i < M; ++i) {
#pragma unroll
                for (int q = 0; q < kSeg / 4; ++q) {
                    const float r = transpose_reduce4(part_sum[i][4 * q], part_sum[i][4 * q + 1],
                                                      part_sum[i][4 * q + 2], part_sum[i][4 * q + 3],
                                                      lane);
                    if ((lane & 7) == 0) {
                        const int u = 4 * q + ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
                        rbuf[(wit * M + i) * kSeg + u] = r;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&T.done[slot]);
            if (++slot == p.depth) {
                slot = 0;
                phase ^= 1u;
            }
        }
    }
    // All teams' cut-row partials must be in shared memory before any team of
    // the cluster reads them.
    if (p.cluster > 1)
        cluster_sync();
    else
        __syncthreads();

    // Rows cut between teams (of this CTA or of other CTAs of the cluster): the
    // team holding a row's first superblock adds the partial sums of the
    // following teams that touch the row, in team order; a partial held by
    // another CTA of the cluster is read through distributed shared memory.
    if (warp == compute_warps && lane < p.teams) {
        const int rank = cta_rank(p);
        const int gteam = rank * p.teams + lane;
        const int nteams = p.cluster * p.teams;
        const TeamRange* table = reinterpret_cast<const TeamRange*>(smem + p.off_tr);
        const TeamRange tr = table[gteam];
        if (tr.nseg > 0) {
            const long long last = tr.row0 + tr.nseg - 1;
            const long long lb = seg_begin(tr, tr.nseg - 1, nsb) - last * nsb;
            const long long le = seg_end(tr, tr.nseg - 1, nsb) - last * nsb;
            if (lb == 0 && le < nsb) {
                float tot[M];
#pragma unroll
                for (int i = 0; i < M; ++i) tot[i] = part[(lane * 2 + 1) * M + i];
                for (int g2 = gteam + 1; g2 < nteams; ++g2) {
                    const TeamRange o = table[g2];
                    if (o.s0 >= (last + 1) * nsb) break;
                    if (o.s1 <= o.s0) continue;   // a team with an empty range
                    const int r2 = g2 / p.teams, t2 = g2 % p.teams;
#pragma unroll
                    for (int i = 0; i < M; ++i) {
                        const float* src = part + (t2 * 2 + 0) * M + i;
                        tot[i] += (r2 == rank) ? *src : ld_dsmem(src, r2);
                    }
                }
#pragma unroll
                for (int i = 0; i < M; ++i) store_row<FUSED>(p, smem, i, last, tot[i]);
            }
        }
    }
    // Keep this CTA's shared memory alive until the cluster has read it.
    if (p.cluster > 1) cluster_sync();
    if (FUSED) {
        // SwiGLU epilogue: y = silu(gate row total) * (up row total).
        __syncthreads();
        long long row0;
        int rows;
        cta_rows(p, row0, rows);
        const float* tot = reinterpret_cast<const float*>(smem + p.off_rows);
        for (int v = static_cast<int>(threadIdx.x); v < rows * M; v += static_cast<int>(blockDim.x)) {
            const int i = v / rows, r = v - i * rows;
            const float* ti = tot + static_cast<size_t>(i) * 2 * p.rows_cap;
            p.y[static_cast<size_t>(i) * p.n + row0 + r] = silu_mul(ti[r], ti[rows + r]);
        }
    }
}

}  // namespace

namespace {

// Clusters of c CTAs that can be resident at once.
int resident_clusters(int c, int num_sms, const int* max_clusters) {
    if (max_clusters != nullptr && max_clusters[c] > 0) return max_clusters[c];
    return num_sms / c;
}

}  // namespace

int stream_max_nsb(int m, int slices) {
    if (m < 1 || m > kStreamMaxM || slices < 1 || slices > 2) return 0;
    // the warps of one team (one CTA's compute warps) times positions per warp
    const int by_warps = (stream_max_threads(m, slices) / 32) * pos_per_warp(slices);
    const int cap = kStreamMaxNsb * slices;
    return by_warps < cap ? by_warps : cap;
}

int plan_stream(int m, int n, int k, int num_sms, int max_smem, const int* max_clusters,
                bool fused, StreamParams* sp, int* grid, int* block, int* smem_bytes) {
    const int nsb = k / kQK;
    if (m < 1 || m > kStreamMaxM || n < 1) return 0;
    // Compact CTAs: at most half of an SM's registers and shared memory, so
    // that a CTA of the next kernel on the stream can be resident beside it
    // (programmatic dependent launch then runs its prologue and first weight
    // copies while this one finishes), with up to kCompactCtasPerSm per SM.
    // (Not for very tall matrices: there the streaming rate decides, and the
    // classic CTA's extra warps pay; measured on B200, LM head 128256 x 4096:
    // 100.9 us classic, 118.6 us compact.)
    const bool tall = (n + num_sms - 1) / num_sms >= kWideMinRows;
    const bool compact_ok = kPlanMode != 0 && !(kPlanMode == 3 && tall);
    // quant slices per lane: two for one vector on very tall matrices, for one
    // vector when K is too long for one-slice teams (K > 20480: a team of
    // two-slice lanes covers K <= 30720 with 15 warps), and for a compact CTA
    // whose one-slice team would not fit its warps
    const int compact_warps1 = kCompactRegs / (stream_max_regs(m, 1) * 32) - 1;
    const bool compact_s1 = compact_ok && (nsb * 8 + 31) / 32 <= compact_warps1;
    const bool compact_s2 = compact_ok && m == 1 && !fused &&
                            (nsb * 4 + 31) / 32 <= kCompactRegs / (stream_max_regs(1, 2) * 32) - 1;
    const bool compact = compact_s1 || compact_s2;
    const bool wide = m == 1 && !fused &&
                      ((n + num_sms - 1) / num_sms >= kWideMinRows || nsb > kStreamMaxNsb ||
                       (compact && !compact_s1));
    const int sl = wide ? 2 : 1;
    if (nsb > stream_max_nsb(m, sl)) return 0;
    const int team_warps = (nsb * lanes_per_sb(sl) + 31) / 32;
    const int max_warps = compact ? kCompactRegs / (stream_max_regs(m, sl) * 32) - 1
                                  : stream_max_threads(m, sl) / 32;
    if (team_warps > max_warps) return 0;
    int teams = max_warps / team_warps;
    if (teams > kStreamMaxTeams) teams = kStreamMaxTeams;
    const int per_sm = compact ? kCompactCtasPerSm : 1;
    // Cluster size. Within a CTA the warps of a team already split K, so a
    // row of any supported K is processed by up to 20 warps at once; splitting
    // rows across the CTAs of a cluster (split-K) adds a cluster launch and two
    // cluster barriers (measured 2-6 us on B200 for clusters of 4-8) and paid
    // off only for a handful of very long rows (N = 1, K = 14336: 7.2 -> 6.7
    // us with clusters of 2). So: clusters of two CTAs for N < 8 and K >= 8192.
    int cluster = 1;
    const int resident1 = compact ? per_sm * num_sms : resident_clusters(1, num_sms, max_clusters);
    int clusters = n < resident1 ? n : resident1;
    if (!fused && n < kClusterMaxRows && nsb >= kClusterMinNsb &&
        resident_clusters(2, num_sms, max_clusters) >= n) {
        cluster = 2;
        clusters = n;
    }
    const int ctas = clusters * cluster;
    const int stage_bytes = ((kSeg * nsb * kBlockBytes) + 127) / 128 * 128;
    // fused: gate and up row totals of the CTA's rows, [m][2 * rows_cap] floats
    const int rows_cap = (n + clusters - 1) / clusters;
    const long long rows_bytes = fused ? (static_cast<long long>(m) * 2 * rows_cap * 4 + 15) / 16 * 16 : 0;
    if (rows_bytes > kStreamMaxRowsBytes) return 0;
    const int cap = compact ? kCompactSmem : kStreamSmemBudget;
    const int budget = (max_smem < cap ? max_smem : cap) - 1024 - static_cast<int>(rows_bytes);
    // bytes per team besides its ring: coefficient buffers of its warps, the
    // partial sums per slot and ring phase, its cut-row partials, its entries of the cluster's
    // team-range table and two barriers per slot
    auto fixed_team = [&](int depth) {
        return team_warps * coef_bytes_per_warp(sl) + depth * 2 * team_warps * kSeg * m * 4 +
               2 * m * 4 + cluster * kTeamRangeBytes + 2 * depth * 8 + 16;
    };
    // A team never needs more slots than it has stages: a team's range is
    // ceil(rows * nsb / teams) superblocks at most, touching at most
    // ceil(that / nsb) + 1 row segments.
    auto max_depth = [&](int t) {
        const long long len = (static_cast<long long>(rows_cap) * (fused ? 2 : 1) * nsb +
                               t * cluster - 1) / (t * cluster);
        const long long segs = (len + nsb - 1) / nsb + 1;
        const long long st = (segs + kSeg - 1) / kSeg;
        return static_cast<int>(st < 2 ? 2 : (st > kStreamMaxDepth ? kStreamMaxDepth : st));
    };
    int depth = max_depth(teams);
    while (depth >= 2 && teams * (depth * stage_bytes + fixed_team(depth)) > budget) {
        if (depth > 2) {
            --depth;
        } else if (teams > 1) {
            --teams;
            depth = max_depth(teams);
        } else {
            break;
        }
    }
    if (teams * (depth * stage_bytes + fixed_team(depth)) > budget) return 0;
    StreamParams q{};
    q.n = n;
    q.k = k;
    q.nsb = nsb;
    q.cluster = cluster;
    q.rows_base = n / clusters;
    q.rows_extra = n % clusters;
    q.teams = teams;
    q.team_warps = team_warps;
    q.depth = depth;
    q.stage_bytes = stage_bytes;
    q.slices = sl;
    q.nsb_row = nsb;
    q.sb_off = 0;
    q.x_stride = k;
    q.accumulate = 0;
    size_t off = static_cast<size_t>(teams) * depth * stage_bytes;
    q.off_coef = static_cast<int>(off);
    off += static_cast<size_t>(teams) * team_warps * coef_bytes_per_warp(sl);
    q.off_red = static_cast<int>(off);
    off += static_cast<size_t>(teams) * depth * 2 * team_warps * kSeg * m * 4;
    q.off_part = static_cast<int>(off);
    off += static_cast<size_t>(teams) * 2 * m * 4;
    off = (off + 15) / 16 * 16;
    q.off_tr = static_cast<int>(off);
    off += static_cast<size_t>(cluster) * teams * kTeamRangeBytes;
    q.off_bar = static_cast<int>(off);
    off += static_cast<size_t>(teams) * 2 * depth * 8;
    q.off_rows = static_cast<int>(off);
    q.rows_cap = fused ? rows_cap : 0;
    off += static_cast<size_t>(rows_bytes);
    *sp = q;
    *grid = ctas;
    *block = teams * team_warps * 32 + 32;   // + the producer warp
    *smem_bytes = static_cast<int>(off);
    return 1;
}

int launch_stream(const StreamParams& sp0, int grid, int block, int smem_bytes, const void* w,
                  const void* w_up, const float* x, float* y, int m, cudaStream_t stream) {
    StreamParams sp = sp0;
    sp.w = static_cast<const uint8_t*>(w);
    sp.w_up = static_cast<const uint8_t*>(w_up);
    sp.x = x;
    sp.y = y;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(sp.cluster);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = sp.cluster > 1 ? 2 : 1;
    cudaError_t e;
    if (w_up != nullptr) {
        e = (m == 1) ? cudaLaunchKernelEx(&cfg, q4k_gemv_stream_kernel<1, 1, true>, sp)
                     : cudaLaunchKernelEx(&cfg, q4k_gemv_stream_kernel<2, 1, true>, sp);
    } else if (m == 1) {
        e = sp.slices == 2 ? cudaLaunchKernelEx(&cfg, q4k_gemv_stream_kernel<1, 2, false>, sp)
                           : cudaLaunchKernelEx(&cfg, q4k_gemv_stream_kernel<1, 1, false>, sp);
    } else {
        e = cudaLaunchKernelEx(&cfg, q4k_gemv_stream_kernel<2, 1, false>, sp);
    }
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

int stream_set_attributes() {
    cudaError_t e = cudaFuncSetAttribute(q4k_gemv_stream_kernel<1, 1, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kStreamSmemBudget);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemv_stream_kernel<1, 2, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmemBudget);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemv_stream_kernel<2, 1, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmemBudget);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemv_stream_kernel<1, 1, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmemBudget);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemv_stream_kernel<2, 1, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmemBudget);
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

}  // namespace q4k

namespace q4k {

int stream_cluster_occupancy(int m, int* max_clusters) {
    for (int c = 0; c <= kStreamMaxCluster; ++c) max_clusters[c] = 0;
    for (int c = 1; c <= kStreamMaxCluster; c *= 2) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(c);
        cfg.blockDim = dim3(stream_max_threads(m, 1) + 32);
        cfg.dynamicSmemBytes = kStreamSmemBudget;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(c);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int count = 0;
        const cudaError_t e = (m == 1)
            ? cudaOccupancyMaxActiveClusters(&count, q4k_gemv_stream_kernel<1, 1, false>, &cfg)
            : cudaOccupancyMaxActiveClusters(&count, q4k_gemv_stream_kernel<2, 1, false>, &cfg);
        if (e != cudaSuccess) {
            cudaGetLastError();   // the query is advisory; clear the error
            count = 0;
        }
        max_clusters[c] = count;
    }
    return Q4K_OK;
}

namespace {

// One thread waits, bounded, on an mbarrier phase that nothing completes: the
// wait gives up after kSpinLimit tries and raises kFaultCopyTimeout, exactly as
// a kernel's wait on a lost bulk copy would, then the kernel returns.
__global__ void q4k_wait_timeout_selftest_kernel() {
    __shared__ __align__(8) uint64_t bar;
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait_bounded(&bar, 0u, &g_fault_flags);
}

}  // namespace

int selftest_wait_timeout(cudaStream_t stream) {
    q4k_wait_timeout_selftest_kernel<<<1, 1, 0, stream>>>();
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

int read_fault_flags(unsigned* flags) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_fault_flags, sizeof(v));
    if (e != cudaSuccess) return cuda_failure(e);
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_fault_flags, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_failure(e);
    *flags = v;
    return Q4K_OK;
}

}  // namespace q4k
