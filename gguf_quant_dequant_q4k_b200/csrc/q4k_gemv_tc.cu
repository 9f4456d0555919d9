// q4k_gemv_tc.cu -- y = W x for Q4_K W and 3..64 f32 vectors on the tcgen05
// tensor cores, each superblock of W decoded once for all vectors of a launch
// (`BatchedQ4KGemv`: dequantise once, multiply by M input vectors, and the
// m = 16 / 32 `MultiWarpBatchedQ4KGemv` branch of `batched_q4k_gemv_into`,
// "realizar 0.8.5, src/cuda/executor/uses.rs"). A batch of m vectors makes the
// product a contraction with m columns; decoding a weight costs the same for
// any m, and the per-vector multiply-adds that grow with m run on the tensor
// cores. The sum is formed exactly in integers; only the final combination
// and the output rounding are inexact:
//
// * Weights. Inside superblock b of a row, weight t is d*sc_j*q_t - dmin*m_j
//   (sub-block j = t/32). A_t = sc_j*q_t is an integer <= 945 and is exact in
//   binary16: (1024 + q) is built from the nibble by one bit operation, and one
//   half2 fma forms (1024 + q)*sc - 1024*sc = sc*q exactly, two weights at a
//   time. The decoded A of a superblock (128 rows x 256 K) goes to tensor
//   memory with tcgen05.st, where the MMA reads it as its A operand.
// * Vectors. A separate kernel writes each vector's 256-element block b as
//   X = round(x * 2^(33 - E)), E the exponent of the block's largest |x|
//   (|X| < 2^33; x is exact where |x| >= 2^(E - 10), else off by at most
//   2^(E - 34)), split into five balanced base-128 digits X = sum_l 128^l
//   X_l, X_l in [-64, 63], each exact in binary16. Row (l, i) of the MMA's B
//   operand holds digit l of vector i.
// * Products. D[row][(l, i)] = sum over the superblock's 256 K of A * X_l:
//   every partial sum is an integer below 945 * 64 * 256 < 2^24, so the f32
//   accumulation is exact. The epilogue forms
//   S1 = sum_l 128^l D_l (exact in f64, < 2^53) and
//   M = sum_j m_j * S0_j (S0_j: the sum of X over sub-block j, from the
//   vector kernel; exact in f64), and adds 2^(E - 33) * (d*S1 - dmin*M) to the
//   row's f64 total. y is that total rounded to f32 once.
//   So y = sum_t w_t x~_t (w exact, x~ the rounded x) up to the f64 roundings
//   (relative 2^-52 of |d*S1| + |dmin*M| per superblock) and the last f32
//   rounding: |y - sum w x| <= 2^-24 (|y| + sum |w x|) + sum_t |w_t| 2^(E_t - 34)
//   with w the once-rounded f32 weights. Non-finite x makes that vector's y NaN.
// * Pipeline. A persistent CTA owns 128-row tiles (the MMA's M). A producer
//   thread streams each superblock column of the tile (128 rows x 144 bytes,
//   one 2-D TMA box) and the vectors' digit image of that superblock (one bulk
//   copy) through rings of stages; four decode warps (one per TMEM lane
//   quarter) write A into one of two or three TMEM buffers; one elected lane
//   of the MMA warp issues 16 MMAs (K = 16) into one of two accumulators;
//   eight epilogue warps (two per lane quarter, half the vectors each) read
//   the accumulator (tcgen05.ld) and combine it in f64.
//
// All waits are bounded: one that gives up raises Q4K_FAULT_COPY_TIMEOUT and
// the CTA lets its copies and MMAs complete (bounded) before it releases shared
// and tensor memory.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "q4k_gemv_tc.h"
#include "q4k_internal.h"
#include "q4k_sm100.cuh"
#include "q4k_superblock.cuh"
#include "q4k_tcgen05.cuh"

namespace q4k {

// Raised (Q4K_FAULT_COPY_TIMEOUT) by a CTA whose bounded wait gave up; read
// and cleared by q4k_device_fault_flags(). Never set in normal operation.
__device__ unsigned int g_tc_fault_flags = 0;

namespace {

// Warp roles. 15 warps leave 128 registers per thread (four warps per
// sub-partition); the f64 epilogue needs them (eight warps, half the vectors
// each), the decode does not (four warps, one per TMEM lane quarter).
constexpr int kTcDecodeWarps = 4;      // warps 0-3: decode into TMEM
constexpr int kTcEpiWarps = 8;         // warps 4-11: epilogue
constexpr int kTcWProducerWarp = 12;   // weight copies
constexpr int kTcXProducerWarp = 13;   // digit image and metadata copies
constexpr int kTcMmaWarp = 14;
constexpr int kTcThreads = 32 * (kTcDecodeWarps + kTcEpiWarps + 3);
constexpr unsigned kTcEpiBarrier = 1;  // named barrier of the epilogue warps
constexpr int kTcRawBytes = kTcRows * kBlockBytes;   // one superblock column of a tile
constexpr int kTcAcols = 128;          // TMEM columns of one superblock of A (256 fp16)
constexpr int kTcTmemCols = 512;
constexpr int kTcMaxABufs = 3;
constexpr int kTcMmaK = 16;
constexpr int kTcMetaStages = 16;
constexpr uint32_t kHalfMagic = 0x64006400u;   // binary16 1024 in both halves

__host__ __device__ constexpr int tc_b_bytes_mp(int mp) { return tc_n_mp(mp) * kQK * 2; }
__host__ __device__ constexpr int tc_meta_bytes_mp(int mp) { return mp * kTcMetaDoubles * 8; }
// Three rings: weights (held until decoded; 4 stages for up to 8 vectors, 3
// for 16), digit images (held until the MMAs that read them complete; as many
// stages as the rest of the budget holds, at most 6) and block metadata
// (held until the epilogue; kTcMetaStages small stages, so that it never
// holds back the image copies).
__host__ __device__ constexpr int tc_wstages_mp(int mp) { return mp <= 8 ? 4 : 3; }
__host__ __device__ constexpr int tc_bstages_mp(int mp) {
    return (kTcSmemBudget - tc_wstages_mp(mp) * kTcRawBytes - kTcMetaStages * tc_meta_bytes_mp(mp)) /
                       tc_b_bytes_mp(mp) < 6
               ? (kTcSmemBudget - tc_wstages_mp(mp) * kTcRawBytes - kTcMetaStages * tc_meta_bytes_mp(mp)) /
                     tc_b_bytes_mp(mp)
               : 6;
}
// Decoded-A buffers in TMEM (128 columns each) and the two accumulators after
// them, kTcTmemCols in all: three A buffers (and accumulators of up to 64
// columns) for up to 8 vectors, two (and 128) for 16.
__host__ __device__ constexpr int tc_abufs_mp(int mp) { return mp <= 8 ? 3 : 2; }
__host__ __device__ constexpr int tc_dstride_mp(int mp) {
    return (kTcTmemCols - tc_abufs_mp(mp) * kTcAcols) / 2;
}
// Barriers: full / empty per stage of the three rings, A full / free per
// buffer, D full / free, MMA done; then the TMEM slot.
constexpr int tc_smem_bytes_mp(int mp) {
    return 1024 + tc_bstages_mp(mp) * tc_b_bytes_mp(mp) + kTcMetaStages * tc_meta_bytes_mp(mp) +
           tc_wstages_mp(mp) * kTcRawBytes +
           (2 * (tc_bstages_mp(mp) + kTcMetaStages + tc_wstages_mp(mp)) + 2 * kTcMaxABufs + 5) * 8 + 16;
}
static_assert(tc_bstages_mp(8) >= 3 && tc_bstages_mp(16) >= 3, "digit image ring too shallow");
static_assert(tc_smem_bytes_mp(8) <= kB200SmemOptin && tc_smem_bytes_mp(16) <= kB200SmemOptin,
              "stage ring exceeds shared memory");
static_assert(tc_n_mp(8) <= tc_dstride_mp(8) && tc_n_mp(16) <= tc_dstride_mp(16),
              "two accumulators must fit beside the A buffers");

// Byte offset of element (row n, MMA K position p) of one superblock's digit
// image: four 64-element atoms along K, each N rows x 128 bytes in the 128-byte
// swizzled K-major layout (8-row groups 1024 bytes apart; 16-byte chunk c of
// row n stored at chunk c ^ (n % 8)).
__host__ __device__ constexpr int tc_image_offset(int n, int p, int n_mma) {
    return (p >> 6) * (n_mma * 128) + (n >> 3) * 1024 + (n & 7) * 128 +
           ((((p & 63) >> 3) ^ (n & 7)) << 4) + (p & 7) * 2;
}

// MMA K position of weight t (0..255) of a superblock. The decode turns quant
// word u (bytes 4u..4u+3 of the 128, group g = u/8) into four TMEM columns
// 4u + c, each a pair of weights: c = 0: low nibbles of bytes 4u, 4u+2; c = 1:
// their high nibbles; c = 2, 3: the same for bytes 4u+1, 4u+3. Column c holds
// K positions 2c (bits 0..15) and 2c + 1.
__host__ __device__ constexpr int tc_k_position(int t) {
    // t = 64g + 32*high + e: byte 32g + e; u = 8g + e/4; byte-in-word e % 4
    return 2 * (4 * (8 * (t >> 6) + ((t & 31) >> 2)) + ((t & 1) << 1) + ((t >> 5) & 1)) +
           ((t >> 1) & 1);
}

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity) {
    return mbar_wait_bounded(bar, parity, &g_tc_fault_flags);
}

// Digits of the vectors' blocks: up to one CTA of four warps per SM (small
// enough to be resident beside a GEMV CTA, whose programmatic launch may
// already hold the rest of the SM), each warp taking (superblock b, vector i)
// pairs in turn: it scales the block to X = round(x * 2^(33 - E)) (into its
// shared-memory slice, in MMA K order), writes the block's metadata
// (2^(E-33), S0_0..7, 0), then the vector's five digit rows l*mp + i of the
// image as 16-byte chunks and the zero row 5*mp + i where that is below
// n_mma. Warp 0 of block 0 also zeroes the GEMV's per-tile piece counters.
constexpr int kTcDigitsWarps = 4;
constexpr int kTcDigitsThreads = 32 * kTcDigitsWarps;

// (At most 32 registers a thread: 4096 for the CTA, what a GEMV CTA leaves free.)
__global__ void __launch_bounds__(kTcDigitsThreads, 16)
q4k_tc_digits_kernel(const float* __restrict__ x, int k, int m, int mp, int n_mma,
                     uint8_t* __restrict__ image, double* __restrict__ meta,
                     unsigned* __restrict__ done, int tiles) {
    __shared__ long long xs_all[kTcDigitsWarps][kQK];   // X at MMA K position p
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long* xs = xs_all[warp];
    pdl_launch_dependents();
    pdl_wait();   // x is produced by the preceding work on the stream
    if (blockIdx.x == 0 && warp == 0)   // counters of the GEMV's tiles cut between CTAs
        for (int t = lane; t < tiles; t += 32) done[t] = 0u;
    const int nsb = k / kQK;
    const int pairs = nsb * mp;
    for (int q = blockIdx.x * kTcDigitsWarps + warp; q < pairs; q += gridDim.x * kTcDigitsWarps) {
        const int b = q / mp, i = q % mp;
        float v[8];
        if (i < m) {
            const float4* src = reinterpret_cast<const float4*>(
                x + static_cast<size_t>(i) * k + static_cast<size_t>(b) * kQK + 8 * lane);
            const float4 a = src[0], c = src[1];
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
        bool finite = true;
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            finite = finite && isfinite(v[e]);
            amax = fmaxf(amax, fabsf(v[e]));
        }
        finite = __all_sync(0xFFFFFFFFu, finite);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
        int ex = 0;
        if (finite && amax > 0.f) frexpf(amax, &ex);   // amax in [2^(ex-1), 2^ex)
        const bool scaled = finite && amax > 0.f;
        // 2^(33 - ex) and 2^(ex - 33) from their exponent fields (ex >= -148)
        const double up = scaled ? __longlong_as_double(static_cast<long long>(1023 + 33 - ex) << 52) : 0.0;
        long long sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int t = 8 * lane + e;
            // exact scaling, one rounding (a non-finite block has X = 0)
            const long long X = scaled ? __double2ll_rn(static_cast<double>(v[e]) * up) : 0;
            sum += X;
            xs[tc_k_position(t)] = X;
        }
        // S0 of sub-block j = lanes 4j..4j+3
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
        double* md = meta + (static_cast<size_t>(b) * mp + i) * kTcMetaDoubles;
        if ((lane & 3) == 0) md[1 + (lane >> 2)] = static_cast<double>(sum);
        if (lane == 0) {
            md[0] = finite ? (scaled ? __longlong_as_double(static_cast<long long>(1023 + ex - 33) << 52) : 0.0)
                           : __longlong_as_double(0x7FF8000000000000LL);
            md[9] = 0.0;
        }
        __syncwarp();
        // Row l*mp + i, chunk `lane` (K positions 8*lane .. + 7): digit l of
        // each value, peeled off the remainder kept in xs (balanced base 128).
        uint8_t* img = image + static_cast<size_t>(b) * (n_mma * kQK * 2);
        long long* xr = xs + 8 * lane;
#pragma unroll 1
        for (int l = 0; l < kTcLimbs; ++l) {
            uint32_t h[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const long long X = xr[e];
                const int dg = static_cast<int>(((X + 64) & 127) - 64);
                xr[e] = (X - dg) >> 7;
                h[e >> 1] |= static_cast<uint32_t>(__half_as_ushort(__int2half_rn(dg))) << (16 * (e & 1));
            }
            *reinterpret_cast<uint4*>(img + tc_image_offset(l * mp + i, 8 * lane, n_mma)) =
                make_uint4(h[0], h[1], h[2], h[3]);
        }
        if (kTcLimbs * mp + i < n_mma)   // the zero row 5*mp + i
            *reinterpret_cast<uint4*>(img + tc_image_offset(kTcLimbs * mp + i, 8 * lane, n_mma)) =
                make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();   // xs is rewritten by the warp's next pair
    }
}

struct TcParams {
    const uint8_t* image;   // [nsb][n_mma rows x 256] digit images
    const double* meta;     // [nsb][mp][10]
    double* part;           // cut tiles: [CTA][2][mp][128] partial row totals
    unsigned* done;         // cut tiles: [tiles] pieces finished (zeroed by the digits kernel)
    float* y;               // [m][n]
    const uint8_t* w;       // the Q4_K matrix (superblock headers for the epilogue)
    int n, nsb, m, tiles;
};

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t b) { return *reinterpret_cast<__half2*>(&b); }

// (a & b) | c in one instruction.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// half2 (s, s) from the 6-bit field in byte `sel` of w, exactly.
__device__ __forceinline__ __half2 scale_pair(uint32_t w, int sel) {
    const uint32_t v = (w >> (8 * sel)) & 0xFFu;
    return __hsub2(bits_h2((v | (v << 16)) | kHalfMagic), __float2half2_rn(1024.f));
}

// sc*q for the nibbles at bits 0..3 and 16..19 of (w & 0x000F000F).
__device__ __forceinline__ uint32_t sc_times_q(uint32_t w, __half2 sc, __half2 nsc) {
    return h2_bits(__hfma2(bits_h2(and_or(w, 0x000F000Fu, kHalfMagic)), sc, nsc));
}

// Small non-negative integer (< 2^31) to f64 exactly, on the FP64 pipe:
// the bits of 2^52 ORed with v are the double 2^52 + v.
__device__ __forceinline__ double small_u32_to_f64(uint32_t v) {
    return __longlong_as_double(0x4330000000000000LL | v) - 4503599627370496.0;
}

// The work is the flat sequence of items f = tile * nsb + b (superblock
// column b of 128-row tile `tile`), cut into gridDim.x equal contiguous
// ranges: CTA c owns [item_begin(c), item_begin(c + 1)). A tile cut between
// CTAs is finished by the last of them to publish its piece.
__device__ __forceinline__ long long item_begin(long long items, int c, int ctas) {
    return items * c / ctas;
}

// The CTA whose range holds item f.
__device__ __forceinline__ int item_owner(long long items, long long f, int ctas) {
    return static_cast<int>(((f + 1) * ctas - 1) / items);
}

// A CTA's range holds at most two pieces of tiles cut between CTAs: a piece
// of the tile its range starts in (slot 0) and a piece of a later tile (slot
// 1). tc_store_piece writes a piece's row totals (plain stores, no ordering);
// tc_finish_pieces, called once after the CTA's last item by all epilogue
// threads together (named barriers), makes them visible, counts them in, and
// finishes each tile whose last piece this CTA wrote: adds the pieces of the
// CTAs holding part of the tile, in CTA order, and stores y.
template <int MP>
__device__ __forceinline__ void tc_store_piece(const TcParams& p, int slot, const double (&yt)[MP / 2],
                                               int wg, int row) {
    double* base = p.part + (static_cast<size_t>(blockIdx.x) * 2 + slot) * MP * kTcRows;
#pragma unroll
    for (int v = 0; v < MP / 2; ++v) base[(wg * (MP / 2) + v) * kTcRows + row] = yt[v];
}

template <int MP>
__device__ __forceinline__ void tc_finish_pieces(const TcParams& p, long long items, bool has0, int t0,
                                                 bool has1, int t1, int wg, int ew, int lane, int row,
                                                 int* last_flags, bool aborted) {
    constexpr int kHalfV = MP / 2;
    __threadfence();
    named_barrier_sync(kTcEpiBarrier, kTcEpiWarps * 32);
    if (ew == 0 && lane < 2) {
        const bool has = lane == 0 ? has0 : has1;
        const int t = lane == 0 ? t0 : t1;
        bool last = false;
        if (has && !aborted) {
            const long long tf0 = static_cast<long long>(t) * p.nsb;
            const int pieces = item_owner(items, tf0 + p.nsb - 1, gridDim.x) - item_owner(items, tf0, gridDim.x);
            last = atomicAdd(&p.done[t], 1u) == static_cast<unsigned>(pieces);
        }
        last_flags[lane] = last ? 1 : 0;
    }
    named_barrier_sync(kTcEpiBarrier, kTcEpiWarps * 32);
#pragma unroll 1
    for (int q = 0; q < 2; ++q) {
        if (!last_flags[q]) continue;
        __threadfence();
        const int t = q == 0 ? t0 : t1;
        const long long tf0 = static_cast<long long>(t) * p.nsb;
        const int c_first = item_owner(items, tf0, gridDim.x);
        const int c_last = item_owner(items, tf0 + p.nsb - 1, gridDim.x);
        // Every CTA after c_first starts inside tile t (its piece is slot 0);
        // c_first's piece is slot 0 only if its range starts at the tile.
        const int first_slot = item_begin(items, c_first, gridDim.x) < tf0 ? 1 : 0;
        const int grow = t * kTcRows + row;
        double tot[kHalfV];
#pragma unroll
        for (int v = 0; v < kHalfV; ++v) tot[v] = 0.0;
        // four pieces per round: their loads are independent and in flight together
        for (int c0 = c_first; c0 <= c_last; c0 += 4) {
            double val[4][kHalfV];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + j;
                const int cs = c == c_first ? first_slot : 0;
                const double* src =
                    p.part + ((static_cast<size_t>(c) * 2 + cs) * MP + wg * kHalfV) * kTcRows + row;
#pragma unroll
                for (int v = 0; v < kHalfV; ++v) val[j][v] = c <= c_last ? __ldcg(src + v * kTcRows) : 0.0;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)   // pieces added in CTA order
#pragma unroll
                for (int v = 0; v < kHalfV; ++v) tot[v] += val[j][v];
        }
#pragma unroll
        for (int v = 0; v < kHalfV; ++v) {
            const int i = wg * kHalfV + v;
            if (grow < p.n && i < p.m) p.y[static_cast<size_t>(i) * p.n + grow] = static_cast<float>(tot[v]);
        }
    }
}

template <int MP>
__global__ void __launch_bounds__(kTcThreads, 1)
q4k_gemv_tc_kernel(const __grid_constant__ CUtensorMap map_w, const TcParams p) {
    constexpr int N = tc_n_mp(MP);
    constexpr int SW = tc_wstages_mp(MP);
    constexpr int SB = tc_bstages_mp(MP);
    constexpr int SM = kTcMetaStages;
    constexpr int kB = tc_b_bytes_mp(MP);
    constexpr int kMeta = tc_meta_bytes_mp(MP);
    constexpr int kHalfV = MP / 2;            // vectors per epilogue warpgroup
    constexpr int kAB = tc_abufs_mp(MP);
    constexpr int kDcol0 = kAB * kTcAcols;    // accumulator d at kDcol0 + d * kDstride
    constexpr int kDstride = tc_dstride_mp(MP);
    constexpr uint32_t kIdesc = mma_f16_idesc(kTcRows, N);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned (the swizzled digit images need it), as an offset from
    // smem_raw so that accesses stay shared-memory accesses
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t* bring = smem;                              // [SB][kB] digit images (swizzled)
    uint8_t* metaring = bring + SB * kB;                // [SM][MP][10] f64
    uint8_t* wring = metaring + SM * kMeta;             // [SW][128 rows][144] superblocks
    uint64_t* wfull = reinterpret_cast<uint64_t*>(wring + SW * kTcRawBytes);
    uint64_t* wempty = wfull + SW;
    uint64_t* bfull = wempty + SW;
    uint64_t* bempty = bfull + SB;
    uint64_t* mfull = bempty + SB;
    uint64_t* mempty = mfull + SM;
    uint64_t* afull = mempty + SM;              // [kAB] decoded A in TMEM buffer
    uint64_t* afree = afull + kTcMaxABufs;      // [kAB] MMAs done reading the buffer
    uint64_t* dfull = afree + kTcMaxABufs;      // [2] accumulator complete
    uint64_t* dfree = dfull + 2;                // [2] accumulator read
    uint64_t* mma_done = dfree + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    __shared__ volatile int abort_flag;
    __shared__ int last_piece[2];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long items = static_cast<long long>(p.tiles) * p.nsb;
    const long long f0 = item_begin(items, blockIdx.x, gridDim.x);
    const long long f1 = item_begin(items, blockIdx.x + 1, gridDim.x);
    const int count = static_cast<int>(f1 - f0);   // items of this CTA

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < SW; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], kTcDecodeWarps);
        }
        for (int s = 0; s < SB; ++s) {
            mbar_init(&bfull[s], 1);
            mbar_init(&bempty[s], 1);
        }
        for (int s = 0; s < SM; ++s) {
            mbar_init(&mfull[s], 1);
            mbar_init(&mempty[s], kTcEpiWarps);
        }
        for (int j = 0; j < kAB; ++j) {
            mbar_init(&afull[j], kTcDecodeWarps);
            mbar_init(&afree[j], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&dfull[j], 1);
            mbar_init(&dfree[j], kTcEpiWarps);
        }
        mbar_init(mma_done, 1);
        fence_mbar_init();
        tma_prefetch_map(&map_w);
    }
    if (warp == kTcMmaWarp) tmem_alloc(tmem_slot, kTcTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    // Every role walks the CTA's items f0 + it, it = 0 .. count - 1.
    if (warp == kTcWProducerWarp) {
        if (lane == 0) {
            // ------------------------------------------------- weight copies
            // (constant data: issued before the preceding kernels finish)
            int issued = 0;
            int tile = static_cast<int>(f0 / p.nsb), b = static_cast<int>(f0 % p.nsb);
            for (int it = 0; it < count && !abort_flag; ++it, b = (b + 1 == p.nsb) ? 0 : b + 1,
                     tile += (b == 0) ? 1 : 0) {
                const int s = it % SW;
                if (it >= SW && !tc_wait(&wempty[s], static_cast<uint32_t>(((it / SW) - 1) & 1))) {
                    abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(&wfull[s], kTcRawBytes);
                tma_load_2d(wring + s * kTcRawBytes, &map_w, b * kBlockBytes, tile * kTcRows, &wfull[s]);
                issued = it + 1;
            }
            if (abort_flag) {
                // let the copies still in flight land before shared memory goes
                for (int i = issued > SW ? issued - SW : 0; i < issued; ++i)
                    tc_wait(&wfull[i % SW], static_cast<uint32_t>((i / SW) & 1));
            }
        }
    } else if (warp == kTcXProducerWarp) {
        if (lane == 0) {
            // ------------------------------------ digit image / metadata copies
            pdl_wait();   // written by the digits kernel
            int issued = 0;
            int b = static_cast<int>(f0 % p.nsb);
            for (int it = 0; it < count && !abort_flag; ++it, b = (b + 1 == p.nsb) ? 0 : b + 1) {
                const int sb = it % SB, sm = it % SM;
                if ((it >= SB && !tc_wait(&bempty[sb], static_cast<uint32_t>(((it / SB) - 1) & 1))) ||
                    (it >= SM && !tc_wait(&mempty[sm], static_cast<uint32_t>(((it / SM) - 1) & 1)))) {
                    abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(&bfull[sb], kB);
                bulk_copy_g2s(bring + sb * kB, p.image + static_cast<size_t>(b) * kB, kB, &bfull[sb]);
                mbar_arrive_expect_tx(&mfull[sm], kMeta);
                bulk_copy_g2s(metaring + sm * kMeta, p.meta + static_cast<size_t>(b) * MP * kTcMetaDoubles,
                              kMeta, &mfull[sm]);
                issued = it + 1;
            }
            if (abort_flag) {
                for (int i = issued > SB ? issued - SB : 0; i < issued; ++i)
                    tc_wait(&bfull[i % SB], static_cast<uint32_t>((i / SB) & 1));
                for (int i = issued > SM ? issued - SM : 0; i < issued; ++i)
                    tc_wait(&mfull[i % SM], static_cast<uint32_t>((i / SM) & 1));
            }
        }
    } else if (warp == kTcMmaWarp) {
        // ------------------------------------------------------------ MMA
        // The warp runs converged (operands and descriptors warp-uniform) and
        // one elected lane issues the MMAs and commits.
        for (int it = 0; it < count; ++it) {
            const int sb = it % SB, a = it % kAB, d = it & 1;
            const bool ok = !abort_flag && tc_wait(&bfull[sb], static_cast<uint32_t>((it / SB) & 1)) &&
                            tc_wait(&afull[a], static_cast<uint32_t>((it / kAB) & 1)) &&
                            (it < 2 || tc_wait(&dfree[d], static_cast<uint32_t>(((it >> 1) - 1) & 1)));
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            const uint64_t bdesc = sw128_kmajor_desc(smem_addr(bring + sb * kB));
            const uint32_t dcol = tmem + static_cast<uint32_t>(kDcol0 + d * kDstride);
            const uint32_t acol = tmem + static_cast<uint32_t>(a * kTcAcols);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kQK / kTcMmaK; ++kk) {
                    // K step kk: atom kk / 4 (N * 128 bytes each), 32 bytes per step
                    // inside it; the descriptor holds the address in 16-byte units
                    const uint64_t bk = bdesc + static_cast<uint64_t>(((kk >> 2) * (N * 128) + (kk & 3) * 32) >> 4);
                    mma_f16_tmem_a(dcol, acol + static_cast<uint32_t>(8 * kk), bk, kIdesc, kk > 0 ? 1u : 0u);
                }
                mma_commit(&afree[a]);
                mma_commit(&dfull[d]);
                mma_commit(&bempty[sb]);
            }
            __syncwarp();
        }
        if (elect_one()) {
            mma_commit(mma_done);   // every MMA issued above has completed
            tc_wait(mma_done, 0u);
        }
        __syncwarp();
    } else if (warp < kTcDecodeWarps) {
        // ------------------------------------------------------------ decode
        const int quarter = warp;                 // TMEM lanes 32*quarter ..
        const int row = 32 * quarter + lane;      // row within the tile
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
        const __half2 m1024 = __float2half2_rn(-1024.f);
        for (int it = 0; it < count; ++it) {
            {   // one superblock column
                const int s = it % SW, a = it % kAB;
                const bool ok = !abort_flag && tc_wait(&wfull[s], static_cast<uint32_t>((it / SW) & 1)) &&
                                (it < kAB || tc_wait(&afree[a], static_cast<uint32_t>(((it / kAB) - 1) & 1)));
                if (!__all_sync(0xFFFFFFFFu, ok)) {
                    abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                const uint8_t* rr = wring + s * kTcRawBytes + row * kBlockBytes;
                const Header hd = decode_header(*reinterpret_cast<const uint4*>(rr));
#pragma unroll
                for (int g = 0; g < 4; ++g) {   // group: sub-blocks 2g (low nibbles), 2g+1 (high)
                    const uint32_t scw = g < 2 ? hd.sc_lo : hd.sc_hi;
                    const __half2 sc0 = scale_pair(scw, (2 * g) & 3);
                    const __half2 sc1 = scale_pair(scw, (2 * g + 1) & 3);
                    const __half2 nsc0 = __hmul2(sc0, m1024), nsc1 = __hmul2(sc1, m1024);
                    const uint4 q0 = *reinterpret_cast<const uint4*>(rr + kQsOffset + 32 * g);
                    const uint4 q1 = *reinterpret_cast<const uint4*>(rr + kQsOffset + 32 * g + 16);
                    const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                    uint32_t cols[32];
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const uint32_t w = words[v];
                        cols[4 * v + 0] = sc_times_q(w, sc0, nsc0);
                        cols[4 * v + 1] = sc_times_q(w >> 4, sc1, nsc1);
                        cols[4 * v + 2] = sc_times_q(w >> 8, sc0, nsc0);
                        cols[4 * v + 3] = sc_times_q(w >> 12, sc1, nsc1);
                    }
                    tmem_store_32cols(lane_base + static_cast<uint32_t>(a * kTcAcols + 32 * g), cols);
                }
                tmem_wait_st();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&afull[a]);
                    mbar_arrive(&wempty[s]);
                }
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        // No early exit: where a tile is cut between CTAs the epilogue warps
        // meet at named barriers, so after a failed wait they keep walking the
        // items with every wait and store skipped.
        const int ew = warp - kTcDecodeWarps;
        const int wg = ew >> 2;                   // half of the vectors
        const int quarter = ew & 3;
        const int row = 32 * quarter + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
        const size_t row_bytes = static_cast<size_t>(p.nsb) * kBlockBytes;
        const int first_tile = static_cast<int>(f0 / p.nsb);
        pdl_wait();   // y and the partial-sum buffers follow the preceding kernels
        double ytot[kHalfV];
#pragma unroll
        for (int v = 0; v < kHalfV; ++v) ytot[v] = 0.0;
        bool has0 = false, has1 = false;   // cut pieces written (slot 0 / 1)
        int tile1 = 0;                     // tile of the slot-1 piece
        int tile = first_tile, b = static_cast<int>(f0 % p.nsb);
        int bstart = b;                    // first superblock column of the current piece
        for (int it = 0; it < count; ++it) {
            const int grow = tile * kTcRows + row;
            const int d = it & 1, sm = it % SM;
            // this row's superblock header (d, dmin, m_j), from L2: the weight
            // copy of this superblock has just brought it there
            const uint4 hraw = grow < p.n
                                   ? ldg_nc_v4(p.w + static_cast<size_t>(grow) * row_bytes +
                                               static_cast<size_t>(b) * kBlockBytes)
                                   : make_uint4(0, 0, 0, 0);
            const bool ok = !abort_flag && tc_wait(&dfull[d], static_cast<uint32_t>((it >> 1) & 1)) &&
                            tc_wait(&mfull[sm], static_cast<uint32_t>((it / SM) & 1));
            if (__all_sync(0xFFFFFFFFu, ok)) {
                tc_fence_after_sync();
                uint32_t rg[kTcLimbs][kHalfV];
#pragma unroll
                for (int l = 0; l < kTcLimbs; ++l) {
                    const uint32_t col =
                        lane_base + static_cast<uint32_t>(kDcol0 + d * kDstride + l * MP + wg * kHalfV);
                    if constexpr (kHalfV == 8) tmem_load_8cols(col, rg[l]);
                    else tmem_load_4cols(col, rg[l]);
                }
                tmem_wait_ld();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dfree[d]);
                const Header hd = decode_header(hraw);
                const double dd = hd.d, dm = hd.dmin;
                double mj[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) mj[j] = small_u32_to_f64(byte_of(j < 4 ? hd.m_lo : hd.m_hi, j & 3));
                const double2* mt = reinterpret_cast<const double2*>(metaring + sm * kMeta);
#pragma unroll
                for (int v = 0; v < kHalfV; ++v) {
                    const double2* mi = mt + (wg * kHalfV + v) * (kTcMetaDoubles / 2);
                    double s1 = static_cast<double>(__uint_as_float(rg[kTcLimbs - 1][v]));
#pragma unroll
                    for (int l = kTcLimbs - 2; l >= 0; --l)
                        s1 = fma(s1, 128.0, static_cast<double>(__uint_as_float(rg[l][v])));
                    const double2 c0 = mi[0], c1 = mi[1], c2 = mi[2], c3 = mi[3], c4 = mi[4];
                    // two independent chains (exact: every partial sum is an
                    // integer below 2^53)
                    double ma = mj[0] * c0.y, mb = mj[1] * c1.x;
                    ma = fma(mj[2], c1.y, ma);
                    mb = fma(mj[3], c2.x, mb);
                    ma = fma(mj[4], c2.y, ma);
                    mb = fma(mj[5], c3.x, mb);
                    ma = fma(mj[6], c3.y, ma);
                    mb = fma(mj[7], c4.x, mb);
                    const double mm = ma + mb;
                    ytot[v] = fma(c0.x, fma(dd, s1, -(dm * mm)), ytot[v]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&mempty[sm]);
            } else {
                abort_flag = 1;
            }
            if (b == p.nsb - 1 || it == count - 1) {
                // end of this CTA's piece of `tile`
                if (bstart == 0 && b == p.nsb - 1) {
                    // the whole tile
                    if (!abort_flag) {
#pragma unroll
                        for (int v = 0; v < kHalfV; ++v) {
                            const int i = wg * kHalfV + v;
                            if (grow < p.n && i < p.m)
                                p.y[static_cast<size_t>(i) * p.n + grow] = static_cast<float>(ytot[v]);
                        }
                    }
                } else if (tile == first_tile) {
                    tc_store_piece<MP>(p, 0, ytot, wg, row);
                    has0 = true;
                } else {
                    tc_store_piece<MP>(p, 1, ytot, wg, row);
                    has1 = true;
                    tile1 = tile;
                }
#pragma unroll
                for (int v = 0; v < kHalfV; ++v) ytot[v] = 0.0;
                bstart = 0;
            }
            if (++b == p.nsb) {
                b = 0;
                ++tile;
            }
        }
        // every epilogue warp takes this branch or none (the pieces depend
        // only on the CTA's range)
        if (has0 || has1)
            tc_finish_pieces<MP>(p, items, has0, first_tile, has1, tile1, wg, ew, lane, row, last_piece,
                                 abort_flag != 0);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kTcMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

template <int MP>
cudaError_t launch_tc_group(const CUtensorMap& map, const TcParams& tp, int grid, cudaStream_t stream) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(tc_smem_bytes_mp(MP));
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, q4k_gemv_tc_kernel<MP>, map, tp);
}

cudaError_t launch_digits(const float* x, int k, int m, int mp, uint8_t* image, double* meta,
                          unsigned* done, int tiles, int num_sms, cudaStream_t stream) {
    cudaLaunchConfig_t cfg{};
    const int pairs = (k / kQK) * mp;
    const int blocks = (pairs + kTcDigitsWarps - 1) / kTcDigitsWarps;
    cfg.gridDim = dim3(static_cast<unsigned>(blocks < num_sms ? blocks : num_sms));
    cfg.blockDim = dim3(kTcDigitsThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, q4k_tc_digits_kernel, x, k, m, mp, tc_n_mp(mp), image, meta, done,
                              tiles);
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// CTAs for `tiles` 128-row tiles of nsb superblocks: one per item up to one
// per SM.
int tc_grid(int tiles, int nsb, int num_sms) {
    const long long items = static_cast<long long>(tiles) * nsb;
    return items < num_sms ? static_cast<int>(items) : num_sms;
}

// Workspace regions (byte offsets from its start), sized for the largest
// vector group: digit images, block metadata, partial tiles and counters.
struct TcLayout {
    size_t meta, part, done, total;
};

TcLayout tc_layout(int m, int n, int k, int num_sms) {
    const int mp = tc_vectors_padded(m < kTcMaxM ? m : kTcMaxM);
    const size_t nsb = static_cast<size_t>(k / kQK);
    const int tiles = (n + kTcRows - 1) / kTcRows;
    const int grid = tc_grid(tiles, k / kQK, num_sms);
    TcLayout l;
    l.meta = align256(nsb * tc_b_bytes_mp(mp));
    l.part = align256(l.meta + nsb * tc_meta_bytes_mp(mp));
    l.done = align256(l.part + static_cast<size_t>(grid) * 2 * mp * kTcRows * 8);
    l.total = align256(l.done + static_cast<size_t>(tiles) * 4);
    return l;
}

}  // namespace

// 2-D map of the Q4_K matrix as bytes: rows of nsb*144 bytes, boxes of one
// superblock column (144 bytes) by 128 rows; rows past n read as zeros.
bool make_weight_map(CUtensorMap* map, const void* w, int n, int nsb) {
    using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                       const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                       const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                       CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeTiledFn fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            ptr = nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    if (fn == nullptr) return false;
    const cuuint64_t row_bytes = static_cast<cuuint64_t>(nsb) * kBlockBytes;
    const cuuint64_t dims[2] = {row_bytes, static_cast<cuuint64_t>(n)};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBlockBytes), static_cast<cuuint32_t>(kTcRows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(w), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int tc_smem_bytes(int mp) { return tc_smem_bytes_mp(mp); }
int tc_stages(int mp) { return tc_wstages_mp(mp); }
int tc_threads() { return kTcThreads; }
int tc_k_position_host(int t) { return tc_k_position(t); }
int tc_ctas(int tiles, int nsb, int num_sms) { return tc_grid(tiles, nsb, num_sms); }

size_t tc_workspace_bytes(int m, int n, int k, int num_sms) { return tc_layout(m, n, k, num_sms).total; }

int tc_set_attributes() {
    cudaError_t e = cudaFuncSetAttribute(q4k_gemv_tc_kernel<8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, tc_smem_bytes_mp(8));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemv_tc_kernel<16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, tc_smem_bytes_mp(16));
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

int launch_gemv_tc(const DeviceInfo& dev, const void* w, const float* x, float* y, int m, int n,
                   int k, cudaStream_t stream) {
    const int nsb = k / kQK;
    const int tiles = (n + kTcRows - 1) / kTcRows;
    const int grid = tc_grid(tiles, nsb, dev.sm_count);
    CUtensorMap map;
    if (!make_weight_map(&map, w, n, nsb)) return cuda_failure(cudaErrorInvalidValue);
    const TcLayout lay = tc_layout(m, n, k, dev.sm_count);
    void* ws = nullptr;
    cudaError_t e = cudaMallocAsync(&ws, lay.total, stream);
    if (e != cudaSuccess) return cuda_failure(e);
    uint8_t* base = static_cast<uint8_t*>(ws);
    uint8_t* image = base;
    double* meta = reinterpret_cast<double*>(base + lay.meta);
    double* part = reinterpret_cast<double*>(base + lay.part);
    unsigned* done = reinterpret_cast<unsigned*>(base + lay.done);
    for (int i0 = 0; i0 < m && e == cudaSuccess; i0 += kTcMaxM) {
        const int mi = (m - i0) < kTcMaxM ? (m - i0) : kTcMaxM;
        const int mp = tc_vectors_padded(mi);
        e = launch_digits(x + static_cast<size_t>(i0) * k, k, mi, mp, image, meta, done, tiles,
                          dev.sm_count, stream);
        if (e != cudaSuccess) break;
        const TcParams tp{image, meta, part, done, y + static_cast<size_t>(i0) * n,
                          static_cast<const uint8_t*>(w), n, nsb, mi, tiles};
        e = mp == 8 ? launch_tc_group<8>(map, tp, grid, stream) : launch_tc_group<16>(map, tp, grid, stream);
    }
    const cudaError_t ef = cudaFreeAsync(ws, stream);
    if (e == cudaSuccess) e = ef;
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

int read_tc_fault_flags(unsigned* flags) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tc_fault_flags, sizeof(v));
    if (e != cudaSuccess) return cuda_failure(e);
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_tc_fault_flags, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_failure(e);
    *flags = v;
    return Q4K_OK;
}

}  // namespace q4k
