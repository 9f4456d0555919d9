// q4k_gemv_i8.cu -- y = W x for Q4_K W and one to four f32 vectors (the
// pages' `Q4KGemv`, "realizar 0.8.5, src/cuda/executor/q4k_gemv_cached.rs",
// and the small batches of `BatchedQ4KGemv`: the LM head and the larger
// projections of a decode step), on the tcgen05 tensor cores with 8-bit
// integer operands. Every product is formed exactly
// in integers; only the final combination and the output rounding are inexact.
//
// * Weights. Weight t of superblock b of a row is d*sc_j*q_t - dmin*m_j
//   (sub-block j = t/32). The MMA's A operand is the quant nibble itself as an
//   unsigned byte: the low nibbles of a quant word (w & 0x0F0F0F0F) are four
//   consecutive weights of sub-block 2g, its high nibbles (w & 0xF0F0F0F0,
//   i.e. 16 q) four of sub-block 2g+1, so one bit operation decodes four
//   weights. The decoded superblock column of a tile (128 rows x 256 bytes)
//   goes to tensor memory with tcgen05.st.
// * Vector. Each CTA scales every 256-element block b of x to
//   X = round(x * 2^(33 - E_b)), E_b the exponent of the block's largest |x|
//   (|X| < 2^33; exact where |x| >= 2^(E_b - 10), else off by at most
//   2^(E_b - 34)), and splits X into five balanced base-128 digits
//   X = sum_l 128^l X_l, X_l in [-64, 63], the rows l of the MMA's B operand
//   (signed bytes; rows 5..7 of the N = 8 operand are not read back).
// * Products. One MMA (K = 32) per sub-block j, each into its own accumulator
//   columns: D_j[row][l] = sum over the sub-block of A * X_l, an integer of at
//   most 32 * 15 * 64 (sixteen times that for odd j). The epilogue forms
//   S = sum_j sc_j * sum_l 128^l D_j[l] (/16 for odd j) exactly in 64-bit
//   integers (|S| < 2^52), M = sum_j m_j * S0_j (S0_j: the sum of X over
//   sub-block j; exact in f64), and adds 2^(E_b - 33) * (d*S - dmin*M) to the
//   row's f64 total; y is that total rounded to f32 once. So
//   |y - sum w x| <= 2^-24 (|y| + sum |w x|) + sum_t |w_t| 2^(E_t - 34), the
//   bound of the batched tensor-core path; non-finite x makes y NaN.
// * Several vectors (m = 2..4: the pages' `BatchedQ4KGemv`, "realizar 0.8.5,
//   src/cuda/executor/uses.rs", `batched_q4k_gemv_into`: W decoded once, every
//   vector multiplied by it). Each decoded superblock column meets the digits
//   of all MV = 2 or 4 vectors in the same 8 MMAs: vector v's block is scaled
//   to X = round(x * 2^(30 - E_b)) (|X| <= 2^30; exact where |x| >= 2^(E_b -
//   7), else off by at most 2^(E_b - 31)) and split into four balanced
//   base-256 digits, B rows 4v .. 4v+3 (N = 4 MV). The epilogue forms
//   P_l = sum_j sc_j D_j[l] in 32-bit integers (odd j: a separate sum, /16 at
//   the end) and S = sum_l 256^l P_l in 64 bits (|S| < 2^50), then as above;
//   the error bound's last term becomes sum_t |w_t| 2^(E_t - 31).
// * Pipeline. A persistent CTA owns whole 128-row tiles, or an equal range of
//   (tile, superblock column) items with tiles cut between CTAs finished from
//   pieces, and walks its items in order; an item is one superblock column, or
//   two where K/256 is even and four two-column stages fit (the per-item
//   waits, polls and hand-offs then cost half as much per column). A producer
//   thread streams each item (128 rows x 144 bytes per column, one 3-D TMA
//   box) through the weight stages; two sets of four decode warps (one per
//   TMEM lane quarter), alternate items each, write A into one of the TMEM
//   buffers and hand each row's superblock headers on through a shared-memory
//   ring; one elected lane of the MMA warp issues the item's 8 MMAs per column
//   into one of the accumulators; eight epilogue warps (two per lane quarter:
//   for one vector a column each, or four sub-blocks each with one column per
//   item; for several, vectors h and h + 2 each) read the accumulator
//   (tcgen05.ld) and combine it. The digit image of the vectors' blocks the
//   CTA needs stays in shared memory for the kernel.
//
// All waits are bounded: one that gives up raises Q4K_FAULT_COPY_TIMEOUT and
// the CTA lets its copies and MMAs complete (bounded) before it releases shared
// and tensor memory.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <map>
#include <mutex>
#include <utility>

#include "q4k_gemv_i8.h"
#include "q4k_gemv_tc.h"
#include "q4k_internal.h"
#include "q4k_sm100.cuh"
#include "q4k_superblock.cuh"
#include "q4k_tcgen05.cuh"

namespace q4k {

// Raised (Q4K_FAULT_COPY_TIMEOUT) by a CTA whose bounded wait gave up; read
// and cleared by q4k_device_fault_flags(). Never set in normal operation.
__device__ unsigned int g_i8_fault_flags = 0;

namespace {

// Two sets of four decode warps (one warp per TMEM lane quarter each) take
// alternate items: a warp waits for its tensor-memory stores before it
// signals the item, and the two sets keep two items' stores in flight.
// Eight epilogue warps (two per lane quarter), the producer (weight copies)
// and the MMA warp.
constexpr int kI8Quarters = 4;
constexpr int kI8DecodeSets = 2;
constexpr int kI8DecodeWarps = kI8Quarters * kI8DecodeSets;   // warps 0-7: decode into TMEM
constexpr int kI8EpiWarps = 2 * kI8Quarters;                   // warps 8-15: epilogue
constexpr int kI8ProducerWarp = 16;
constexpr int kI8MmaWarp = 17;
constexpr int kI8Warps = 18;
constexpr int kI8Threads = 32 * kI8Warps;
// named barrier of the threads publishing a piece (1-4: the quarter pairs of
// the one-vector epilogue)
constexpr unsigned kI8PieceBarrier = 5;
constexpr int kI8RawBytes = kI8Rows * kBlockBytes;   // one superblock column of a tile
constexpr int kI8ColTmem = 64;               // TMEM columns of one decoded superblock column (256 bytes)
constexpr int kI8TmemCols = 512;
constexpr int kI8VecMeta = 10;               // per vector and block: 2^(E-33) (2^(E-30)), S0_0..7, pad
// MV vectors per launch (1, 2 or 4): digit rows of the B operand (MMA N;
// rows 5..7 unused for one vector), digits per vector, one block's digit
// image (K-major, swizzled), its metadata, accumulator columns of one
// superblock column.
__host__ __device__ constexpr int i8_n(int mv) { return mv == 1 ? 8 : 4 * mv; }
__host__ __device__ constexpr int i8_limbs(int mv) { return mv == 1 ? 5 : 4; }
__host__ __device__ constexpr int i8_image_bytes(int mv) { return i8_n(mv) * kQK; }
__host__ __device__ constexpr int i8_meta_doubles(int mv) { return kI8VecMeta * mv; }
__host__ __device__ constexpr int i8_col_acc(int mv) { return 8 * i8_n(mv); }
// An item is CPI (1 or 2) superblock columns of a tile: A buffers of CPI * 64
// TMEM columns and accumulators of CPI * 8N, 4 / CPI of each (2 for four
// vectors), the A buffers first.
__host__ __device__ constexpr int i8_bufs(int cpi, int mv) { return mv == 4 ? 2 : 4 / cpi; }
__host__ __device__ constexpr int i8_dcol0(int cpi, int mv) { return i8_bufs(cpi, mv) * cpi * kI8ColTmem; }
constexpr int kI8HSlotCols = 8;              // header ring: 8 superblock columns' row headers
constexpr int kI8HeaderBytes = kI8Rows * 16;      // one column's row headers
// barriers sized for one column per item (the most buffers)
constexpr int kI8Barriers = 2 * kI8MaxWStages + 4 + 2 * 4 + 2 * kI8HSlotCols + 1;
static_assert(i8_dcol0(1, 1) + 4 * i8_col_acc(1) <= kI8TmemCols &&
              i8_dcol0(1, 4) + 2 * i8_col_acc(4) <= kI8TmemCols, "TMEM buffers");

// Shared memory: [digit images][metadata] of the CTA's `ncols` superblock
// columns, [row headers] (1024-aligned), [weight stages of CPI columns],
// [barriers], TMEM slot.
__host__ __device__ constexpr int i8_wring_offset(int ncols, int mv) {
    return (ncols * (i8_image_bytes(mv) + i8_meta_doubles(mv) * 8) + kI8HSlotCols * kI8HeaderBytes + 1023) /
           1024 * 1024;
}
__host__ __device__ constexpr int i8_fit_stages(int ncols, int cpi, int mv) {
    return (kI8SmemBudget - 1024 - i8_wring_offset(ncols, mv) - kI8Barriers * 8 - 16) / (cpi * kI8RawBytes);
}
__host__ __device__ constexpr int i8_smem_bytes_cfg(int ncols, int cpi, int wstages, int mv) {
    return 1024 + i8_wring_offset(ncols, mv) + wstages * cpi * kI8RawBytes + kI8Barriers * 8 + 16;
}

// Byte offset of (row n, K position kk) in one block's digit image of N rows:
// two 128-element atoms along K, each N rows x 128 bytes in the 128-byte
// swizzled K-major layout (8-row groups 1024 bytes apart; 16-byte chunk c of
// row n stored at chunk c ^ (n % 8)).
__host__ __device__ constexpr int i8_image_offset(int n, int kk, int nrows) {
    return (kk >> 7) * (nrows * 128) + (n >> 3) * 1024 + (n & 7) * 128 +
           ((((kk & 127) >> 4) ^ (n & 7)) << 4) + (kk & 15);
}

__device__ __forceinline__ bool i8_wait(uint64_t* bar, uint32_t parity) {
    return mbar_wait_bounded(bar, parity, &g_i8_fault_flags);
}

// Small non-negative integer (< 2^31) to f64 exactly, on the FP64 pipe.
__device__ __forceinline__ double u32_to_f64(uint32_t v) {
    return __longlong_as_double(0x4330000000000000LL | v) - 4503599627370496.0;
}

// Low bytes of four ints packed into one word (byte i from v[i]).
__device__ __forceinline__ uint32_t pack_bytes(int a, int b, int c, int d) {
    const uint32_t ab = __byte_perm(static_cast<uint32_t>(a), static_cast<uint32_t>(b), 0x0040u);
    const uint32_t cd = __byte_perm(static_cast<uint32_t>(c), static_cast<uint32_t>(d), 0x0040u);
    return __byte_perm(ab, cd, 0x5410u);
}

// Digit image and metadata of x's 256-element blocks: slot j (j = first,
// first + stride, ... < ncols) holds padded column (b0 + j) mod pnsb, which is
// block b of x if b < nsb (a padded column past the row gets nothing). One
// warp per block; lane holds K positions 8*lane .. + 7.
__device__ __forceinline__ void i8_digits(const float* __restrict__ x, int nsb, int pnsb, int b0, int ncols,
                                          uint8_t* image, double* meta, int first, int stride,
                                          int lane) {
    for (int j = first; j < ncols; j += stride) {
        const int b = (b0 + j) % pnsb;
        if (b >= nsb) continue;
        const float4* src = reinterpret_cast<const float4*>(x + static_cast<size_t>(b) * kQK + 8 * lane);
        const float4 a = src[0], c = src[1];
        const float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
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
        // 2^(33 - ex) from its exponent field (ex >= -148)
        const double up = scaled ? __longlong_as_double(static_cast<long long>(1023 + 33 - ex) << 52) : 0.0;
        long long sum = 0;
        int r[8];       // X >> 7 after the first digit (|.| < 2^27)
        int dig[8];     // current digit
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            // exact scaling, one rounding (a non-finite block has X = 0)
            const long long X = scaled ? __double2ll_rn(static_cast<double>(v[e]) * up) : 0;
            sum += X;
            dig[e] = ((static_cast<int>(X) + 64) & 127) - 64;
            r[e] = static_cast<int>((X - dig[e]) >> 7);
        }
        // S0 of sub-block j = lanes 4j .. 4j+3
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
        double* md = meta + static_cast<size_t>(j) * i8_meta_doubles(1);
        if ((lane & 3) == 0) md[1 + (lane >> 2)] = static_cast<double>(sum);
        if (lane == 0) {
            md[0] = finite ? (scaled ? __longlong_as_double(static_cast<long long>(1023 + ex - 33) << 52) : 0.0)
                           : __longlong_as_double(0x7FF8000000000000LL);
            md[9] = 0.0;
        }
        uint8_t* img = image + static_cast<size_t>(j) * i8_image_bytes(1);
#pragma unroll
        for (int l = 0; l < i8_limbs(1); ++l) {
            if (l > 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    dig[e] = ((r[e] + 64) & 127) - 64;
                    r[e] = (r[e] - dig[e]) >> 7;
                }
            }
            *reinterpret_cast<uint2*>(img + i8_image_offset(l, 8 * lane, i8_n(1))) =
                make_uint2(pack_bytes(dig[0], dig[1], dig[2], dig[3]),
                           pack_bytes(dig[4], dig[5], dig[6], dig[7]));
        }
    }
}

// The same for MV = 2 or 4 vectors (rows of x, `k` apart; vectors v >= m get
// nothing, their accumulator columns are never read): one warp per (slot,
// vector); X = round(x * 2^(30 - E_b)) split into four balanced base-256
// digits X = sum_l 256^l X_l, X_l in [-128, 127] (|X| <= 2^30 leaves the last
// one within [-64, 64]), B rows 4v + l; the vector's metadata at
// meta[slot][10 v ..]: 2^(E_b - 30), pad, then S0_j (|S0_j| <= 2^35) as the
// int pair (S0_j mod 2^18, floor(S0_j / 2^18)) for j = 0..7.
template <int MV>
__device__ __forceinline__ void i8_digits_mv(const float* __restrict__ x, int m, int k, int nsb, int pnsb, int b0,
                                             int ncols, uint8_t* image, double* meta, int first, int stride,
                                             int lane) {
    for (int job = first; job < ncols * MV; job += stride) {
        const int j = job / MV, vec = job % MV;
        const int b = (b0 + j) % pnsb;
        if (b >= nsb || vec >= m) continue;
        const float4* src = reinterpret_cast<const float4*>(x + static_cast<size_t>(vec) * k +
                                                            static_cast<size_t>(b) * kQK + 8 * lane);
        const float4 a = src[0], c = src[1];
        const float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
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
        // 2^(30 - ex) from its exponent field (ex >= -148)
        const double up = scaled ? __longlong_as_double(static_cast<long long>(1023 + 30 - ex) << 52) : 0.0;
        long long sum = 0;
        int r[8];   // remainder after the digits so far
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            // exact scaling, one rounding (a non-finite block has X = 0)
            r[e] = scaled ? __double2int_rn(static_cast<double>(v[e]) * up) : 0;
            sum += r[e];
        }
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);   // S0 of sub-block j = lanes 4j .. 4j+3
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
        double* md = meta + static_cast<size_t>(j) * i8_meta_doubles(MV) + kI8VecMeta * vec;
        if ((lane & 3) == 0)   // S0_j = 2^18 h + l, l in [0, 2^18)
            reinterpret_cast<int2*>(md + 2)[lane >> 2] =
                make_int2(static_cast<int>(sum & 0x3FFFF), static_cast<int>(sum >> 18));
        if (lane == 0) {
            md[0] = finite ? (scaled ? __longlong_as_double(static_cast<long long>(1023 + ex - 30) << 52) : 0.0)
                           : __longlong_as_double(0x7FF8000000000000LL);
            md[1] = 0.0;
        }
        uint8_t* img = image + static_cast<size_t>(j) * i8_image_bytes(MV);
#pragma unroll
        for (int l = 0; l < i8_limbs(MV); ++l) {
            int dig[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                dig[e] = ((r[e] + 128) & 255) - 128;
                r[e] = (r[e] - dig[e]) >> 8;
            }
            *reinterpret_cast<uint2*>(img + i8_image_offset(4 * vec + l, 8 * lane, i8_n(MV))) =
                make_uint2(pack_bytes(dig[0], dig[1], dig[2], dig[3]),
                           pack_bytes(dig[4], dig[5], dig[6], dig[7]));
        }
    }
}

struct I8Params {
    const float* x;      // [m][k]
    float* y;            // [m][n]
    double* part;        // tiles cut between CTAs: [CTA][2][MV][128] partial row totals
    unsigned* done;      // tiles cut between CTAs: [tiles] pieces published (zero between launches)
    int m, n, k, nsb, tiles;
    int npi;             // items per tile: ceil(nsb / CPI); the last one of a tile may
                         // hold a column past the row (zero-filled, skipped)
    int ncols;           // digit-image slots: the CTA's columns, from its first one
    int whole;           // 1: CTAs own whole tiles (no tile is cut)
    int x_ready;         // 1: x is not written by the preceding work: the digit image
                         // is formed before the grid dependency resolves, and only the
                         // epilogue (the one role writing global memory) waits for it
};

// The work is the flat sequence of items f = tile * npi + i (superblock
// columns CPI*i .. CPI*i + CPI - 1 of 128-row tile `tile`), cut into gridDim.x
// equal contiguous
// ranges: CTA c owns [i8_item_begin(c), i8_item_begin(c + 1)). A tile cut
// between CTAs is finished by the last of them to publish its piece.
__device__ __forceinline__ long long i8_item_begin(long long items, int c, int ctas) {
    return items * c / ctas;
}

// The CTA whose range holds item f.
__device__ __forceinline__ int i8_item_owner(long long items, long long f, int ctas) {
    return static_cast<int>(((f + 1) * ctas - 1) / items);
}

// Counter add with acquire-release semantics at GPU scope: it publishes every
// write the CTA ordered before it (a barrier) and sees every piece published
// before it.
__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* ptr, unsigned v) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v) : "memory");
    return old;
}

// The publishing threads (the epilogue's first half for one vector, thread =
// row; every epilogue warp for several, each with its row and vectors) publish
// the CTA's piece of tile t (slot 0: the tile its range starts in, slot 1: the
// one it ends in; the totals of its MV vectors are already stored) and, if it
// is the tile's last piece, finish the tile: add the pieces of the CTAs
// holding part of it, in CTA order, and store y for the thread's vectors v0,
// v0 + 2, ... < v1 (vector 0 for one). The leader thread takes the counter.
// (Out of line: it runs at most twice per CTA, and inlined its registers would
// spill those of the epilogue loop.)
template <int MV>
__device__ __noinline__ void i8_publish_piece(const double* part, unsigned* done, float* y, int n, int v0, int v1,
                                              int npi, long long items, int t, int row, bool leader, int* last_flag,
                                              bool aborted) {
    // one vector: the epilogue's first half; several: every epilogue warp
    constexpr unsigned nthreads = MV == 1 ? kI8Rows : 32 * kI8EpiWarps;
    constexpr int vstep = MV == 1 ? 1 : 2;
    if constexpr (MV == 1) {
        v0 = 0;
        v1 = 1;
    }
    named_barrier_sync(kI8PieceBarrier, nthreads);   // every row's total is stored
    const long long tf0 = static_cast<long long>(t) * npi;
    const int c_first = i8_item_owner(items, tf0, gridDim.x);
    const int c_last = i8_item_owner(items, tf0 + npi - 1, gridDim.x);
    if (leader) {
        bool last = false;
        if (!aborted) {
            last = atom_add_acq_rel_gpu(&done[t], 1u) == static_cast<unsigned>(c_last - c_first);
            if (last) done[t] = 0u;   // every other piece is in: the counter is free for the next launch
        }
        *last_flag = last ? 1 : 0;
    }
    named_barrier_sync(kI8PieceBarrier, nthreads);
    if (!*last_flag) return;
    // Every CTA after c_first starts inside tile t (its piece is slot 0);
    // c_first's piece is slot 0 only if its range starts at the tile.
    const int first_slot = i8_item_begin(items, c_first, gridDim.x) < tf0 ? 1 : 0;
    const int grow = t * kI8Rows + row;
    for (int v = v0; v < v1; v += vstep) {
        double tot = 0.0;
        // four pieces per round: their loads are independent and in flight together
        for (int c0 = c_first; c0 <= c_last; c0 += 4) {
            double val[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + j;
                const int cs = c == c_first ? first_slot : 0;
                val[j] = c <= c_last ? __ldcg(part + ((static_cast<size_t>(c) * 2 + cs) * MV + v) * kI8Rows + row)
                                     : 0.0;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) tot += val[j];   // pieces added in CTA order
        }
        if (grow < n) y[static_cast<size_t>(v) * n + grow] = static_cast<float>(tot);
    }
}

// The epilogue's sum for one row and one superblock column over sub-blocks
// j0 .. j0 + NJ - 1: r holds D_j[l] at r[(j - j0) * 5 + l]. Returns
// d * S - dmin * M with S = sum_j sc_j * T_j, T_j = sum_l 128^l D_j[l] (D / 16
// for odd j) = lo_j + 2^21 hi_j, lo_j = D0 + 128 D1 + 2^14 D2 (|lo| < 2^29),
// hi_j = D3 + 128 D4 (|hi| < 2^22): sum sc*lo in 64 bits, sum sc*hi in 32
// (8 * 63 * 3962880 < 2^31); M = sum_j m_j * S0_j (mb[1 + j] = S0_j, exact in
// f64, two chains).
template <int NJ>
__device__ __forceinline__ double i8_column_sum(const uint32_t* r, const Header& hd, const double* mb, int j0) {
    long long s_lo = 0;
    int s_hi = 0;
    double ma = 0.0, mc = 0.0;
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) {
        const int j = j0 + jj;
        const uint32_t* rj = r + jj * i8_limbs(1);
        const int D0 = static_cast<int>(rj[0]), D1 = static_cast<int>(rj[1]);
        const int D2 = static_cast<int>(rj[2]), D3 = static_cast<int>(rj[3]);
        const int D4 = static_cast<int>(rj[4]);
        int lo, hi;
        if (jj & 1) {   // odd j (j0 is even): A = 16 q, every D is a multiple of 16
            lo = (D0 >> 4) + 8 * D1 + 1024 * D2;
            hi = (D3 >> 4) + 8 * D4;
        } else {
            lo = D0 + 128 * D1 + 16384 * D2;
            hi = D3 + 128 * D4;
        }
        const uint32_t scw = j < 4 ? hd.sc_lo : hd.sc_hi, mw = j < 4 ? hd.m_lo : hd.m_hi;
        const int sc = static_cast<int>(byte_of(scw, j & 3));
        s_lo += static_cast<long long>(sc) * lo;
        s_hi += sc * hi;
        const double mj = u32_to_f64(byte_of(mw, j & 3)) * mb[1 + j];
        if (jj & 1) mc += mj; else ma += mj;
    }
    const long long S = s_lo + (static_cast<long long>(s_hi) << 21);   // |S| < 2^52
    const double dd = hd.d, dm = hd.dmin;
    return fma(dd, static_cast<double>(S), -(dm * (ma + mc)));
}

// The same for one of MV >= 2 vectors and one superblock column, digits in
// base 256, in two steps of four sub-blocks: i8_b256_add takes D_j[l] of
// sub-blocks j0 .. j0+3 from r[4 (j - j0) + l] into P_l = sum_j sc_j D_j[l]
// (even and odd sub-blocks summed apart: |even| <= 4 * 63 * 32 * 15 * 128 <
// 2^24, |odd| sixteen times that, < 2^28, a multiple of 16) and M = 2^18
// sum_j m_j h_j + sum_j m_j l_j (each sum within 32 bits: |h_j| < 2^17), with
// mb the vector's metadata (mb[0] = 2^(E-30); from byte 16 S0_j = 2^18 h_j +
// l_j as int pairs (l_j, h_j), l_j in [0, 2^18)); i8_b256_sum returns
// d * S - dmin * M with S = sum_l 256^l P_l (|S| < 2^50).
struct I8B256Acc {
    int pe[4], po[4], ml, mh;
};

__device__ __forceinline__ void i8_b256_add(I8B256Acc& acc, const uint32_t* r, const Header& hd, const double* mb,
                                            int j0) {
    const int4* s0 = reinterpret_cast<const int4*>(mb + 2);   // (l_0, h_0, l_1, h_1), ...
    const uint32_t scw = j0 == 0 ? hd.sc_lo : hd.sc_hi, mw = j0 == 0 ? hd.m_lo : hd.m_hi;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const int sc = static_cast<int>(byte_of(scw, jj));
#pragma unroll
        for (int l = 0; l < 4; ++l) {
            if (jj & 1) acc.po[l] += sc * static_cast<int>(r[4 * jj + l]);
            else acc.pe[l] += sc * static_cast<int>(r[4 * jj + l]);
        }
        const int4 q = s0[(j0 + jj) >> 1];
        const int mj = static_cast<int>(byte_of(mw, jj));
        acc.ml += mj * ((jj & 1) ? q.z : q.x);
        acc.mh += mj * ((jj & 1) ? q.w : q.y);
    }
}

__device__ __forceinline__ double i8_b256_sum(const I8B256Acc& acc, const Header& hd) {
    long long S = 0;
#pragma unroll
    for (int l = 0; l < 4; ++l) S += static_cast<long long>(acc.pe[l] + (acc.po[l] >> 4)) << (8 * l);
    const long long M = (static_cast<long long>(acc.mh) << 18) + acc.ml;
    const double dd = hd.d, dm = hd.dmin;
    return fma(dd, static_cast<double>(S), -(dm * static_cast<double>(M)));
}

template <int WS, int CPI, int MV>
__global__ void __launch_bounds__(kI8Threads, 1)
q4k_gemv_i8_kernel(const __grid_constant__ CUtensorMap map_w, const I8Params p) {
    constexpr int kN = i8_n(MV);                      // MMA N: digit rows
    constexpr uint32_t kIdesc = mma_i8_idesc(kI8Rows, kN);
    constexpr int kBufs = i8_bufs(CPI, MV);           // A buffers = accumulators
    constexpr int kDcol0 = i8_dcol0(CPI, MV);         // first accumulator column
    constexpr int kColAcc = i8_col_acc(MV);           // accumulator columns of one superblock column
    constexpr int kImage = i8_image_bytes(MV);
    constexpr int kMeta = i8_meta_doubles(MV);
    static_assert((MV == 1 || MV == 2 || MV == 4) && (MV != 4 || CPI == 1), "vectors per launch");
    static_assert(kDcol0 + kBufs * CPI * kColAcc <= kI8TmemCols && kBufs <= 4, "TMEM buffers");
    constexpr int kHSlots = kI8HSlotCols / CPI;       // header ring slots (items)
    constexpr int kStage = CPI * kI8RawBytes;         // one weight stage
    // Item it uses A buffer and accumulator it % kBufs: one commit per item
    // tells the decode that the A buffer is free and the epilogue that the
    // accumulator is complete.
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned (the swizzled digit images need it), as an offset from
    // smem_raw so that accesses stay shared-memory accesses
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int nsb = p.nsb, npi = p.npi;
    const int pnsb = npi * CPI;                                   // columns per tile, padded
    uint8_t* image = smem;                                        // [ncols][kImage]
    double* meta = reinterpret_cast<double*>(smem + p.ncols * kImage);   // [ncols][MV][10]
    uint4* hring = reinterpret_cast<uint4*>(meta + p.ncols * kMeta);      // [slot][CPI][128]
    uint8_t* wring = smem + i8_wring_offset(p.ncols, MV);         // [WS][128 rows][CPI][144]
    uint64_t* wfull = reinterpret_cast<uint64_t*>(wring + WS * kStage);
    uint64_t* wempty = wfull + kI8MaxWStages;
    uint64_t* afull = wempty + kI8MaxWStages;  // decoded A in TMEM buffer
    uint64_t* dfull = afull + 4;               // MMAs done: A buffer free, accumulator complete
    uint64_t* dfree = dfull + 4;               // accumulator read
    uint64_t* hfull = dfree + 4;               // row headers of an item written
    uint64_t* hfree = hfull + kI8HSlotCols;    // row headers read
    uint64_t* mma_done = hfree + kI8HSlotCols;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    __shared__ volatile int abort_flag;
    __shared__ double xchange[MV == 1 ? 2 * kI8Rows : 1];   // one vector's epilogue: half 1's totals, by piece parity
    __shared__ int last_piece[2];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // items [f0, f1) of this CTA, from item i00 of tile tile0: equal
    // contiguous item ranges, or (whole) equal contiguous tile ranges
    const long long items = static_cast<long long>(p.tiles) * npi;
    const long long f0 = p.whole ? i8_item_begin(p.tiles, blockIdx.x, gridDim.x) * npi
                                 : i8_item_begin(items, blockIdx.x, gridDim.x);
    const long long f1 = p.whole ? i8_item_begin(p.tiles, blockIdx.x + 1, gridDim.x) * npi
                                 : i8_item_begin(items, blockIdx.x + 1, gridDim.x);
    const int count = static_cast<int>(f1 - f0);
    const int tile0 = static_cast<int>(f0 / npi);
    const int i00 = static_cast<int>(f0 % npi);
    // digit-image slot of (padded) column pb: its distance from the CTA's first
    // column, modulo the padded row
    const int pb_first = i00 * CPI;
    auto slot_of = [&](int pb) { return pb >= pb_first ? pb - pb_first : pb - pb_first + pnsb; };

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < WS; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], kI8Quarters);
        }
        for (int j = 0; j < kBufs; ++j) {
            mbar_init(&afull[j], kI8Quarters);
            mbar_init(&dfull[j], 1);
            mbar_init(&dfree[j], kI8EpiWarps);
        }
        for (int j = 0; j < kHSlots; ++j) {
            mbar_init(&hfull[j], kI8Quarters);
            mbar_init(&hfree[j], kI8EpiWarps);
        }
        mbar_init(mma_done, 1);
        fence_mbar_init();
        tma_prefetch_map(&map_w);
    }
    if (warp == kI8MmaWarp) tmem_alloc(tmem_slot, kI8TmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    // Weight copies of items f0 + it: one 3-D box of CPI columns x 128 rows.
    // The first kI8PreStages are constant data: issued before the preceding
    // kernels finish; the rest of the ring follows the vector's loads (behind
    // a full ring of copies those wait microseconds).
    int p_it = 0, p_tile = tile0, p_i = i00;
    auto produce = [&](int upto) {
        for (; p_it < upto && !abort_flag; ++p_it) {
            const int s = p_it % WS;
            if (p_it >= WS && !i8_wait(&wempty[s], static_cast<uint32_t>(((p_it / WS) - 1) & 1))) {
                abort_flag = 1;
                break;
            }
            mbar_arrive_expect_tx(&wfull[s], kStage);
            tma_load_3d(wring + s * kStage, &map_w, 0, p_i * CPI, p_tile * kI8Rows, &wfull[s]);
            if (++p_i == npi) {
                p_i = 0;
                ++p_tile;
            }
        }
    };
    if (warp == kI8ProducerWarp && lane == 0) produce(count < kI8PreStages ? count : kI8PreStages);
    __syncwarp();

    // x is produced, and y and the cut-tile counters may be used, by the
    // preceding work on the stream (x excepted when the caller says so)
    if (!p.x_ready) pdl_wait();
    {
        const int ncols_used = count * CPI < pnsb ? count * CPI : pnsb;
        if constexpr (MV == 1)
            i8_digits(p.x, nsb, pnsb, pb_first, ncols_used, image, meta, warp, kI8Warps, lane);
        else
            i8_digits_mv<MV>(p.x, p.m, p.k, nsb, pnsb, pb_first, ncols_used, image, meta, warp, kI8Warps, lane);
    }
    fence_proxy_async_smem();   // the image is read by the MMAs
    __syncthreads();

    if (warp == kI8ProducerWarp) {
        if (lane == 0) {
            produce(count);
            if (abort_flag) {
                // let the copies still in flight land before shared memory goes
                const int issued = p_it;
                for (int i = issued > WS ? issued - WS : 0; i < issued; ++i)
                    i8_wait(&wfull[i % WS], static_cast<uint32_t>((i / WS) & 1));
            }
        }
    } else if (warp == kI8MmaWarp) {
        // ------------------------------------------------------------ MMA
        // The warp runs converged and one elected lane issues the MMAs and
        // commits: sub-block j of column c of the item is one MMA, A from TMEM
        // columns 64c + 8j .. +7 of the buffer, B = the column's digit rows at
        // K 32j, the accumulator columns 8N c + N j .. +N-1 (no accumulation
        // across MMAs).
        int i = i00;
        for (int it = 0; it < count; ++it, i = (i + 1 == npi) ? 0 : i + 1) {
            const int a = it % kBufs;
            const bool ok = !abort_flag && i8_wait(&afull[a], static_cast<uint32_t>((it / kBufs) & 1)) &&
                            (it < kBufs || i8_wait(&dfree[a], static_cast<uint32_t>(((it / kBufs) - 1) & 1)));
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t dcol = tmem + static_cast<uint32_t>(kDcol0 + a * CPI * kColAcc);
            const uint32_t acol = tmem + static_cast<uint32_t>(a * CPI * kI8ColTmem);
            if (elect_one()) {
#pragma unroll
                for (int c = 0; c < CPI; ++c) {
                    const int pb = i * CPI + c;
                    if (pb >= nsb) continue;   // past the row: no MMA, the epilogue skips it
                    const uint32_t img = smem_addr(image + static_cast<size_t>(slot_of(pb)) * kImage);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        // K position 32j: atom j / 4 (N * 128 bytes each), 32 bytes
                        // per MMA inside it
                        const uint64_t bdesc = sw128_kmajor_desc(img + (j >> 2) * (kN * 128) + (j & 3) * 32);
                        mma_i8_tmem_a(dcol + static_cast<uint32_t>(c * kColAcc + j * kN),
                                      acol + static_cast<uint32_t>(c * kI8ColTmem + 8 * j), bdesc, kIdesc, 0u);
                    }
                }
                mma_commit(&dfull[a]);
            }
            __syncwarp();
        }
        if (elect_one()) {
            mma_commit(mma_done);   // every MMA issued above has completed
            i8_wait(mma_done, 0u);
        }
        __syncwarp();
    } else if (warp < kI8DecodeWarps) {
        // ------------------------------------------------------------ decode
        // Lane = row of the tile; for column c of the item its quant word u of
        // group g = u / 8 gives buffer columns 64c + 16g + u % 8 (low nibbles:
        // sub-block 2g) and 64c + 16g + 8 + u % 8 (high nibbles: sub-block
        // 2g+1). The row's 16-byte superblock headers go to the header ring for
        // the epilogue.
        const int quarter = warp % kI8Quarters;
        const int row = 32 * quarter + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
        for (int it = warp / kI8Quarters; it < count; it += kI8DecodeSets) {
            const int s = it % WS, a = it % kBufs, hs = it % kHSlots;
            const bool ok = !abort_flag && i8_wait(&wfull[s], static_cast<uint32_t>((it / WS) & 1)) &&
                            (it < kBufs || i8_wait(&dfull[a], static_cast<uint32_t>(((it / kBufs) - 1) & 1))) &&
                            (it < kHSlots || i8_wait(&hfree[hs], static_cast<uint32_t>(((it / kHSlots) - 1) & 1)));
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
#pragma unroll
            for (int c = 0; c < CPI; ++c) {
                const uint4* rq = reinterpret_cast<const uint4*>(wring + s * kStage + (row * CPI + c) * kBlockBytes);
                const uint4 hdr = rq[0];
                uint4 q[8];   // the row's 128 quant bytes of column c
#pragma unroll
                for (int v = 0; v < 8; ++v) q[v] = rq[1 + v];
                if (c == CPI - 1) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&wempty[s]);   // the stage is read
                }
                hring[(hs * CPI + c) * kI8Rows + row] = hdr;
#pragma unroll
                for (int h = 0; h < 2; ++h) {   // groups 2h, 2h+1: 32 columns
                    uint32_t cols[32];
#pragma unroll
                    for (int gg = 0; gg < 2; ++gg) {
                        const uint4 q0 = q[2 * (2 * h + gg)], q1 = q[2 * (2 * h + gg) + 1];
                        const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            cols[16 * gg + k] = words[k] & 0x0F0F0F0Fu;
                            cols[16 * gg + 8 + k] = words[k] & 0xF0F0F0F0u;
                        }
                    }
                    tmem_store_32cols(lane_base + static_cast<uint32_t>(a * CPI * kI8ColTmem + c * kI8ColTmem + 32 * h),
                                      cols);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&hfull[hs]);
            tmem_wait_st();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[a]);
        }
    } else {
        // ---------------------------------------------------------- epilogue
        // Two warps per lane quarter. One vector: they share each item (with
        // two columns per item half h takes column h, with one half h takes
        // sub-blocks 4h .. 4h+3), each keeping its own f64 row total; at the
        // end of a piece (the CTA's part of a tile) half 1 hands its total to
        // half 0 (shared memory, a named barrier per quarter), which adds the
        // two in that order and stores y or the piece. MV >= 2 vectors: half h
        // takes vectors h, h + 2 of its lane quarter in every column of the
        // item, one group (column, vector) after the other, and keeps and
        // stores those vectors' row totals.
        const int quarter = warp % kI8Quarters;
        const int eg = (warp - kI8DecodeWarps) / kI8Quarters;   // half (one vector) or first vector
        constexpr int kVW = MV == 1 ? 1 : MV / 2;   // vectors this warp sums: eg + kVStep * vv
        constexpr int kVStep = 2;
        const int row = 32 * quarter + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
        // a piece of tile t is published by half 0 (one vector: the row's
        // total is there) or by every epilogue warp (its vectors)
        auto publish = [&](int t, int* flag) {
            i8_publish_piece<MV>(p.part, p.done, p.y, p.n, eg, p.m, npi, items, t, row, row == 0 && eg == 0, flag,
                                 abort_flag != 0);
        };
        if (p.x_ready) pdl_wait();   // before this role's first global write
        double ytot[kVW];
#pragma unroll
        for (int vv = 0; vv < kVW; ++vv) ytot[vv] = 0.0;
        int tile = tile0, i = i00;
        int istart = i;                    // first item of the current piece
        bool has1 = false;                 // a cut piece left to publish after the last item
        int tile1 = 0;                     // its tile
        int parity = 0;                    // alternates per piece: one barrier per piece
        for (int it = 0; it < count; ++it) {
            const int grow = tile * kI8Rows + row;
            const int a = it % kBufs, hs = it % kHSlots;
            const bool ok = !abort_flag && i8_wait(&dfull[a], static_cast<uint32_t>((it / kBufs) & 1)) &&
                            i8_wait(&hfull[hs], static_cast<uint32_t>((it / kHSlots) & 1));
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                abort_flag = 1;
            } else if constexpr (MV == 1) {
                const int c = CPI == 2 ? eg : 0;   // the item's column this half reads
                // this row's superblock header (d, dmin, sc_j, m_j)
                const uint4 hraw = hring[(hs * CPI + c) * kI8Rows + row];
                __syncwarp();
                if (lane == 0) mbar_arrive(&hfree[hs]);
                tc_fence_after_sync();
                constexpr int kNJ = CPI == 2 ? 8 : 4;   // sub-blocks this half sums
                constexpr int kL = i8_limbs(1);
                uint32_t r[kNJ * kL];                   // D_j[l] at (j - j0) * 5 + l: the digit columns only
                const uint32_t dcol = lane_base + static_cast<uint32_t>(kDcol0 + a * CPI * kColAcc +
                                                                        (CPI == 2 ? c * kColAcc : 32 * eg));
#pragma unroll
                for (int jj = 0; jj < kNJ; ++jj) tmem_load_5cols(dcol + static_cast<uint32_t>(jj * kN), r + jj * kL);
                tmem_wait_ld();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dfree[a]);
                const int pb = i * CPI + c;
                if (pb < nsb) {   // a column past the row (odd K/256, two columns per item) adds nothing
                    const Header hd = decode_header(hraw);
                    const double* mb = meta + static_cast<size_t>(slot_of(pb)) * kMeta;
                    double part;
                    if constexpr (CPI == 2) part = i8_column_sum<8>(r, hd, mb, 0);
                    else part = i8_column_sum<4>(r, hd, mb, 4 * eg);
                    ytot[0] = fma(mb[0], part, ytot[0]);
                }
            } else {
                uint4 hraw[CPI];   // this row's headers of the item's columns
#pragma unroll
                for (int c = 0; c < CPI; ++c) hraw[c] = hring[(hs * CPI + c) * kI8Rows + row];
                __syncwarp();
                if (lane == 0) mbar_arrive(&hfree[hs]);
                tc_fence_after_sync();
                // (column, vector) groups, one after the other
#pragma unroll
                for (int g = 0; g < CPI * kVW; ++g) {
                    const int c = g / kVW, vv = g % kVW, vec = eg + kVStep * vv;
                    const int pb = i * CPI + c;
                    // warp-uniform: a column past the row or a vector past m adds nothing
                    const bool use = pb < nsb && vec < p.m;
                    uint32_t r[32];   // D_j[l] of this vector at 4 j + l
                    if (use) {
                        const uint32_t dcol = lane_base + static_cast<uint32_t>(kDcol0 + (a * CPI + c) * kColAcc +
                                                                                4 * vec);
#pragma unroll
                        for (int j = 0; j < 8; ++j) tmem_load_4cols_at(dcol + static_cast<uint32_t>(j * kN), r + 4 * j);
                    }
                    tmem_wait_ld();
                    if (g == CPI * kVW - 1) {   // the item's accumulator is read
                        tc_fence_before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&dfree[a]);
                    }
                    if (use) {
                        const Header hd = decode_header(hraw[c]);
                        const double* mb = meta + static_cast<size_t>(slot_of(pb)) * kMeta + kI8VecMeta * vec;
                        I8B256Acc acc{{0, 0, 0, 0}, {0, 0, 0, 0}, 0, 0};
                        i8_b256_add(acc, r, hd, mb, 0);
                        i8_b256_add(acc, r + 16, hd, mb, 4);
                        ytot[vv] = fma(mb[0], i8_b256_sum(acc, hd), ytot[vv]);
                    }
                }
            }
            if (i == npi - 1 || it == count - 1) {
                // end of this CTA's piece of `tile`
                bool store = true;   // this thread holds totals to store
                double tot[kVW];
#pragma unroll
                for (int vv = 0; vv < kVW; ++vv) tot[vv] = ytot[vv];
                if constexpr (MV == 1) {   // the halves' totals, added
                    double* xc = xchange + parity * kI8Rows;
                    if (eg == 1) xc[row] = ytot[0];
                    named_barrier_sync(1 + quarter, 64);
                    store = eg == 0;
                    if (store) tot[0] = ytot[0] + xc[row];
                }
                if (store) {
                    if (istart == 0 && i == npi - 1) {   // the whole tile
#pragma unroll
                        for (int vv = 0; vv < kVW; ++vv) {
                            const int vec = MV == 1 ? 0 : eg + kVStep * vv;
                            if (!abort_flag && grow < p.n && vec < p.m)
                                p.y[static_cast<size_t>(vec) * p.n + grow] = static_cast<float>(tot[vv]);
                        }
                    } else {
                        // a piece: slot 0 is published at once (the rest of
                        // the range follows), slot 1 after the last item
                        const int slot = tile == tile0 ? 0 : 1;
#pragma unroll
                        for (int vv = 0; vv < kVW; ++vv) {
                            const int vec = MV == 1 ? 0 : eg + kVStep * vv;
                            p.part[((static_cast<size_t>(blockIdx.x) * 2 + slot) * MV + vec) * kI8Rows + row] = tot[vv];
                        }
                        if (slot == 0 && it < count - 1) {
                            publish(tile, &last_piece[0]);
                        } else {
                            has1 = true;
                            tile1 = tile;
                        }
                    }
                }
#pragma unroll
                for (int vv = 0; vv < kVW; ++vv) ytot[vv] = 0.0;
                istart = 0;
                parity ^= 1;
            }
            if (++i == npi) {
                i = 0;
                ++tile;
            }
        }
        // every publishing thread takes this branch or none (the pieces
        // depend only on the CTA's range)
        if (has1) publish(tile1, &last_piece[1]);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kI8MmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kI8TmemCols);
    }
}

}  // namespace

bool i8_whole_tiles(int tiles, int num_sms) {
    if (tiles < num_sms) return false;
    const long long busiest = (static_cast<long long>(tiles) + num_sms - 1) / num_sms;
    return busiest * num_sms * kI8MaxImbalance <= static_cast<long long>(tiles) * (kI8MaxImbalance + 1);
}

int i8_threads() { return kI8Threads; }

bool i8_config(int m, int n, int k, int num_sms, int max_smem, I8Config* cfg) {
    if (m < 1 || m > kI8MaxM || n < 1 || k < kQK || k % kQK != 0 || num_sms < 1) return false;
    const int mv = m == 1 ? 1 : m == 2 ? 2 : 4;
    const int nsb = k / kQK;
    const long long tiles = (static_cast<long long>(n) + kI8Rows - 1) / kI8Rows;
    if (tiles * nsb >= (1LL << 31) / num_sms) return false;   // item counts in 32 bits
    bool whole = i8_whole_tiles(static_cast<int>(tiles), num_sms);
    // whole tiles per CTA, or enough (tile, column) units per CTA that the
    // kernel's fixed cost (digit image, pipeline fill, cut tiles) pays off
    if (!whole && tiles * nsb < static_cast<long long>(kI8MinItemsPerCta) * num_sms) return false;
    // fewer tiles than SMs: one whole tile per CTA on `tiles` CTAs where the
    // columns that adds to the busiest CTA (nsb * (1 - tiles / SMs) against
    // an equal split) cost less than publishing and finishing cut tiles
    if (!whole && tiles < num_sms &&
        static_cast<long long>(nsb) * (num_sms - tiles) <= static_cast<long long>(i8_whole_extra_cols(mv)) * num_sms)
        whole = true;
    const int budget = max_smem < kI8SmemBudget ? max_smem : kI8SmemBudget;
    // two columns per item unless an odd K/256 is small (the padded column of
    // each tile's last item would be a large share of the work) or four
    // vectors' accumulators leave tensor memory for one column only
    for (int cpi = mv < 4 && (nsb % 2 == 0 || nsb >= 9) ? 2 : 1; cpi >= 1; --cpi) {
        I8Config c;
        c.mv = mv;
        c.cpi = cpi;
        c.npi = (nsb + cpi - 1) / cpi;
        c.items = tiles * c.npi;
        c.whole = whole ? 1 : 0;
        c.ctas = static_cast<int>(whole ? (tiles < num_sms ? tiles : num_sms) : (c.items < num_sms ? c.items : num_sms));
        c.items_per_cta_max = whole ? (tiles + c.ctas - 1) / c.ctas * c.npi : (c.items + c.ctas - 1) / c.ctas;
        const long long pnsb = static_cast<long long>(c.npi) * cpi;
        c.ncols = static_cast<int>(c.items_per_cta_max * cpi < pnsb ? c.items_per_cta_max * cpi : pnsb);
        const int fit = i8_fit_stages(c.ncols, cpi, mv);
        // the kernel's instantiations: 4 two-column stages; 8, 6 or 4 one-column
        if (fit < kI8MinWStages) continue;
        c.wstages = cpi == 2 ? 4 : fit >= 8 ? 8 : fit >= 6 ? 6 : 4;
        c.smem = i8_smem_bytes_cfg(c.ncols, cpi, c.wstages, mv);
        if (c.smem > budget) continue;
        c.cuts = 0;
        if (!whole)
            for (int q = 1; q < c.ctas && !c.cuts; ++q)
                if ((c.items * q / c.ctas) % c.npi != 0) c.cuts = 1;
        *cfg = c;
        return true;
    }
    return false;
}

namespace {

// Scratch for tiles cut between CTAs, one per (device, stream): the per-tile
// counters (zeroed once; every launch leaves them zero, the last publisher of a
// tile resetting its counter) and the pieces, [SMs][2][up to 4 vectors][128]
// f64. Calls on one stream run in order, so a stream's calls never share it
// concurrently.
struct I8Scratch {
    void* ptr = nullptr;
    int tiles_cap = 0;
    int ctas_cap = 0;
};
std::mutex g_i8_mu;
std::map<std::pair<int, uintptr_t>, I8Scratch> g_i8_scratch;

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// Counters then pieces: the pieces' offset for a region of `tiles` counters,
// the pieces' bytes for `ctas` CTAs.
size_t scratch_part_offset(int tiles) { return align256(static_cast<size_t>(tiles) * sizeof(unsigned)); }
size_t scratch_part_bytes(int ctas) { return static_cast<size_t>(ctas) * 2 * kI8MaxM * kI8Rows * sizeof(double); }

// The stream's scratch for `tiles` tiles and `ctas` CTAs, (re)allocated in
// stream order if missing or too small; *done stays null if the stream is
// capturing a graph and has none large enough yet (the caller then allocates
// per call).
cudaError_t stream_scratch(int device, cudaStream_t stream, int tiles, int ctas, unsigned** done,
                           double** part) {
    *done = nullptr;
    *part = nullptr;
    std::lock_guard<std::mutex> lock(g_i8_mu);
    I8Scratch& sc = g_i8_scratch[{device, reinterpret_cast<uintptr_t>(stream)}];
    if (sc.ptr == nullptr || sc.tiles_cap < tiles || sc.ctas_cap < ctas) {
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        cudaError_t e = cudaStreamIsCapturing(stream, &cap);
        if (e != cudaSuccess || cap != cudaStreamCaptureStatusNone) return e;
        const int tcap = tiles > 4096 ? tiles : 4096;
        const int ccap = ctas > 256 ? ctas : 256;
        void* p = nullptr;
        e = cudaMallocAsync(&p, scratch_part_offset(tcap) + scratch_part_bytes(ccap), stream);
        if (e != cudaSuccess) return e;
        e = cudaMemsetAsync(p, 0, static_cast<size_t>(tcap) * sizeof(unsigned), stream);
        if (e != cudaSuccess) return e;
        if (sc.ptr != nullptr) cudaFreeAsync(sc.ptr, stream);
        sc.ptr = p;
        sc.tiles_cap = tcap;
        sc.ctas_cap = ccap;
    }
    *done = static_cast<unsigned*>(sc.ptr);
    *part = reinterpret_cast<double*>(static_cast<uint8_t*>(sc.ptr) + scratch_part_offset(sc.tiles_cap));
    return cudaSuccess;
}

}  // namespace

template <int WS, int CPI, int MV>
cudaError_t i8_set_attribute() {
    return cudaFuncSetAttribute(q4k_gemv_i8_kernel<WS, CPI, MV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kI8SmemBudget);
}

int i8_set_attributes() {
    const cudaError_t es[] = {i8_set_attribute<8, 1, 1>(), i8_set_attribute<6, 1, 1>(), i8_set_attribute<4, 1, 1>(),
                              i8_set_attribute<4, 2, 1>(), i8_set_attribute<8, 1, 2>(), i8_set_attribute<6, 1, 2>(),
                              i8_set_attribute<4, 1, 2>(), i8_set_attribute<4, 2, 2>(), i8_set_attribute<8, 1, 4>(),
                              i8_set_attribute<6, 1, 4>(), i8_set_attribute<4, 1, 4>()};
    for (const cudaError_t e : es)
        if (e != cudaSuccess) return cuda_failure(e);
    return Q4K_OK;
}

namespace {

// 3-D map of the Q4_K matrix as bytes: (byte of a superblock, superblock
// column, row) with strides 144 and nsb*144; boxes of cpi superblock columns
// by 128 rows (one item); rows past n read as zeros.
bool make_weight_map3(CUtensorMap* map, const void* w, int n, int nsb, int cpi) {
    using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                       const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                       const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                       CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeTiledFn fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            ptr = nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    if (fn == nullptr) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kBlockBytes), static_cast<cuuint64_t>(nsb),
                                static_cast<cuuint64_t>(n)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kBlockBytes),
                                   static_cast<cuuint64_t>(nsb) * kBlockBytes};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kBlockBytes), static_cast<cuuint32_t>(cpi),
                               static_cast<cuuint32_t>(kI8Rows)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(w), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {

// The kernel's instantiation for a launch shape (the ones i8_config picks).
template <int MV>
cudaError_t launch_i8_mv(const cudaLaunchConfig_t& cfg, const I8Config& c, const CUtensorMap& map,
                         const I8Params& ip) {
    if constexpr (MV < 4) {
        if (c.cpi == 2) return cudaLaunchKernelEx(&cfg, q4k_gemv_i8_kernel<4, 2, MV>, map, ip);
    }
    return c.wstages >= 8 ? cudaLaunchKernelEx(&cfg, q4k_gemv_i8_kernel<8, 1, MV>, map, ip)
         : c.wstages >= 6 ? cudaLaunchKernelEx(&cfg, q4k_gemv_i8_kernel<6, 1, MV>, map, ip)
                          : cudaLaunchKernelEx(&cfg, q4k_gemv_i8_kernel<4, 1, MV>, map, ip);
}

}  // namespace

int launch_gemv_i8(const DeviceInfo& dev, const void* w, const float* x, float* y, int m, int n, int k,
                   cudaStream_t stream, bool x_ready) {
    I8Config c;
    if (!i8_config(m, n, k, dev.sm_count, dev.max_smem_optin, &c)) return Q4K_ERR_SHAPE;   // not reached
    const int nsb = k / kQK;
    const int tiles = (n + kI8Rows - 1) / kI8Rows;
    CUtensorMap map;
    if (!make_weight_map3(&map, w, n, nsb, c.cpi)) return cuda_failure(cudaErrorInvalidValue);
    // Tiles cut between CTAs: the stream's scratch, or (a graph being
    // captured on a stream without one) a stream-ordered allocation of this
    // call, counters zeroed on the stream.
    unsigned* done = nullptr;
    double* part = nullptr;
    void* own = nullptr;
    cudaError_t e = cudaSuccess;
    if (c.cuts) {
        int device = 0;
        e = cudaGetDevice(&device);
        if (e == cudaSuccess) e = stream_scratch(device, stream, tiles, c.ctas, &done, &part);
        if (e == cudaSuccess && done == nullptr) {
            e = cudaMallocAsync(&own, scratch_part_offset(tiles) + scratch_part_bytes(c.ctas), stream);
            if (e == cudaSuccess) e = cudaMemsetAsync(own, 0, static_cast<size_t>(tiles) * sizeof(unsigned), stream);
            done = static_cast<unsigned*>(own);
            part = reinterpret_cast<double*>(static_cast<uint8_t*>(own) + scratch_part_offset(tiles));
        }
        if (e != cudaSuccess) return cuda_failure(e);
    }
    const I8Params ip{x, y, part, done, m, n, k, nsb, tiles, c.npi, c.ncols, c.whole, x_ready ? 1 : 0};
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(c.ctas));
    cfg.blockDim = dim3(kI8Threads);
    cfg.dynamicSmemBytes = static_cast<size_t>(c.smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = c.mv == 1 ? launch_i8_mv<1>(cfg, c, map, ip)
      : c.mv == 2 ? launch_i8_mv<2>(cfg, c, map, ip)
                  : launch_i8_mv<4>(cfg, c, map, ip);
    if (own != nullptr) {
        const cudaError_t ef = cudaFreeAsync(own, stream);
        if (e == cudaSuccess) e = ef;
    }
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

int read_i8_fault_flags(unsigned* flags) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_i8_fault_flags, sizeof(v));
    if (e != cudaSuccess) return cuda_failure(e);
    if (v != 0) {
        // A launch that gave up may have left cut-tile counters of this
        // device's stream scratches non-zero: clear them.
        int device = 0;
        e = cudaGetDevice(&device);
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        std::lock_guard<std::mutex> lock(g_i8_mu);
        for (auto& kv : g_i8_scratch)
            if (e == cudaSuccess && kv.first.first == device && kv.second.ptr != nullptr)
                e = cudaMemset(kv.second.ptr, 0, static_cast<size_t>(kv.second.tiles_cap) * sizeof(unsigned));
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return cuda_failure(e);
    }
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_i8_fault_flags, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_failure(e);
    *flags = v;
    return Q4K_OK;
}

}  // namespace q4k
