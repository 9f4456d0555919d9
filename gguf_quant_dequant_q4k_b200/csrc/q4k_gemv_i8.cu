// q4k_gemv_i8.cu -- y = W x for Q4_K W and one f32 vector (the pages'
// `Q4KGemv`, "realizar 0.8.5, src/cuda/executor/q4k_gemv_cached.rs": the LM
// head and the larger projections of a decode step), on the tcgen05
// tensor cores with 8-bit integer operands. Every product is formed exactly
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
//   a column each, or four sub-blocks each with one column per item) read the
//   accumulator (tcgen05.ld) and combine it. The digit image of the vector's
//   blocks the CTA needs stays in shared memory for the kernel.
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
constexpr int kI8Quarters = 4;
constexpr int kI8DecodeSets = 2;
constexpr int kI8DecodeWarps = kI8Quarters * kI8DecodeSets;   // warps 0-7: decode into TMEM
constexpr int kI8EpiWarps = 2 * kI8Quarters;                   // warps 8-15: epilogue
constexpr int kI8ProducerWarp = 16;    // weight copies
constexpr int kI8MmaWarp = 17;
constexpr int kI8Warps = 18;
constexpr unsigned kI8PieceBarrier = 5;   // named barrier of the epilogue's first half (1-4: quarter pairs)
constexpr int kI8Threads = 32 * kI8Warps;
constexpr int kI8Limbs = 5;
constexpr int kI8N = 8;                      // MMA N: digit rows 0..4
constexpr int kI8ImageBytes = kI8N * kQK;    // one block's digit image (K-major, swizzled)
constexpr int kI8MetaDoubles = 10;           // 2^(E-33), S0_0..7, pad
constexpr int kI8RawBytes = kI8Rows * kBlockBytes;   // one superblock column of a tile
constexpr int kI8ColTmem = 64;               // TMEM columns of one decoded superblock column (256 bytes)
constexpr int kI8ColAcc = 8 * kI8N;          // accumulator columns of one superblock column
constexpr int kI8TmemCols = 512;
constexpr int kI8Dcol0 = 256;                // A buffers in TMEM columns 0..255, accumulators after them
// An item is CPI (1 or 2) superblock columns of a tile: A buffers and
// accumulators of CPI * 64 columns, 4 / CPI of each.
__host__ __device__ constexpr int i8_bufs(int cpi) { return 4 / cpi; }
constexpr int kI8HSlotCols = 8;              // header ring: 8 superblock columns' row headers
constexpr int kI8HeaderBytes = kI8Rows * 16;      // one column's row headers
// barriers sized for one column per item (the most buffers)
constexpr int kI8Barriers = 2 * kI8MaxWStages + 4 + 2 * 4 + 2 * kI8HSlotCols + 1;
static_assert(kI8Dcol0 + 4 * kI8ColAcc <= kI8TmemCols && 4 * kI8ColTmem <= kI8Dcol0, "TMEM buffers");

// Shared memory: [digit images][metadata] of the CTA's `ncols` superblock
// columns, [row headers] (1024-aligned), [weight stages of CPI columns],
// [barriers], TMEM slot.
__host__ __device__ constexpr int i8_wring_offset(int ncols) {
    return (ncols * (kI8ImageBytes + kI8MetaDoubles * 8) + kI8HSlotCols * kI8HeaderBytes + 1023) / 1024 * 1024;
}
__host__ __device__ constexpr int i8_fit_stages(int ncols, int cpi) {
    return (kI8SmemBudget - 1024 - i8_wring_offset(ncols) - kI8Barriers * 8 - 16) / (cpi * kI8RawBytes);
}
__host__ __device__ constexpr int i8_smem_bytes_cfg(int ncols, int cpi, int wstages) {
    return 1024 + i8_wring_offset(ncols) + wstages * cpi * kI8RawBytes + kI8Barriers * 8 + 16;
}

// Byte offset of (row n, K position kk) in one block's digit image: two
// 128-element atoms along K, each N rows x 128 bytes in the 128-byte swizzled
// K-major layout (8-row groups 1024 bytes apart; 16-byte chunk c of row n
// stored at chunk c ^ (n % 8)).
__host__ __device__ constexpr int i8_image_offset(int n, int kk) {
    return (kk >> 7) * (kI8N * 128) + (n >> 3) * 1024 + (n & 7) * 128 +
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
        double* md = meta + static_cast<size_t>(j) * kI8MetaDoubles;
        if ((lane & 3) == 0) md[1 + (lane >> 2)] = static_cast<double>(sum);
        if (lane == 0) {
            md[0] = finite ? (scaled ? __longlong_as_double(static_cast<long long>(1023 + ex - 33) << 52) : 0.0)
                           : __longlong_as_double(0x7FF8000000000000LL);
            md[9] = 0.0;
        }
        uint8_t* img = image + static_cast<size_t>(j) * kI8ImageBytes;
#pragma unroll
        for (int l = 0; l < kI8Limbs; ++l) {
            if (l > 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    dig[e] = ((r[e] + 64) & 127) - 64;
                    r[e] = (r[e] - dig[e]) >> 7;
                }
            }
            *reinterpret_cast<uint2*>(img + i8_image_offset(l, 8 * lane)) =
                make_uint2(pack_bytes(dig[0], dig[1], dig[2], dig[3]),
                           pack_bytes(dig[4], dig[5], dig[6], dig[7]));
        }
    }
}

struct I8Params {
    const float* x;      // [k]
    float* y;            // [n]
    double* part;        // tiles cut between CTAs: [CTA][2][128] partial row totals
    unsigned* done;      // tiles cut between CTAs: [tiles] pieces published (zero between launches)
    int n, nsb, tiles;
    int npi;             // items per tile: ceil(nsb / CPI); the last one of a tile may
                         // hold a column past the row (zero-filled, skipped)
    int ncols;           // digit-image slots: the CTA's columns, from its first one
    int whole;           // 1: CTAs own whole tiles (no tile is cut)
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

// The 128 threads of the epilogue's first half (thread = row) publish the
// CTA's piece of tile t (slot 0: the tile its range starts in, slot 1: the
// one it ends in; the totals are already stored) and, if it is the tile's
// last piece, finish the tile: add the pieces of the CTAs holding part of it,
// in CTA order, and store y.
// (Out of line: it runs at most twice per CTA, and inlined its registers would
// spill those of the epilogue loop.)
__device__ __noinline__ void i8_publish_piece(const double* part, unsigned* done, float* y, int n, int npi,
                                              long long items, int t, int row, int* last_flag, bool aborted) {
    named_barrier_sync(kI8PieceBarrier, kI8Rows);   // every row's total is stored
    const long long tf0 = static_cast<long long>(t) * npi;
    const int c_first = i8_item_owner(items, tf0, gridDim.x);
    const int c_last = i8_item_owner(items, tf0 + npi - 1, gridDim.x);
    if (row == 0) {
        bool last = false;
        if (!aborted) {
            last = atom_add_acq_rel_gpu(&done[t], 1u) == static_cast<unsigned>(c_last - c_first);
            if (last) done[t] = 0u;   // every other piece is in: the counter is free for the next launch
        }
        *last_flag = last ? 1 : 0;
    }
    named_barrier_sync(kI8PieceBarrier, kI8Rows);
    if (!*last_flag) return;
    // Every CTA after c_first starts inside tile t (its piece is slot 0);
    // c_first's piece is slot 0 only if its range starts at the tile.
    const int first_slot = i8_item_begin(items, c_first, gridDim.x) < tf0 ? 1 : 0;
    double tot = 0.0;
    // four pieces per round: their loads are independent and in flight together
    for (int c0 = c_first; c0 <= c_last; c0 += 4) {
        double val[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + j;
            const int cs = c == c_first ? first_slot : 0;
            val[j] = c <= c_last ? __ldcg(part + (static_cast<size_t>(c) * 2 + cs) * kI8Rows + row) : 0.0;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) tot += val[j];   // pieces added in CTA order
    }
    const int grow = t * kI8Rows + row;
    if (grow < n) y[grow] = static_cast<float>(tot);
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
        const uint32_t* rj = r + jj * kI8Limbs;
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

template <int WS, int CPI>
__global__ void __launch_bounds__(kI8Threads, 1)
q4k_gemv_i8_kernel(const __grid_constant__ CUtensorMap map_w, const I8Params p) {
    constexpr uint32_t kIdesc = mma_i8_idesc(kI8Rows, kI8N);
    constexpr int kBufs = i8_bufs(CPI);               // A buffers = accumulators
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
    uint8_t* image = smem;                                        // [ncols][kI8ImageBytes]
    double* meta = reinterpret_cast<double*>(smem + p.ncols * kI8ImageBytes);   // [ncols][10]
    uint4* hring = reinterpret_cast<uint4*>(meta + p.ncols * kI8MetaDoubles);    // [slot][CPI][128]
    uint8_t* wring = smem + i8_wring_offset(p.ncols);             // [WS][128 rows][CPI][144]
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
    __shared__ double xchange[2 * kI8Rows];   // epilogue: half 1's row totals, by piece parity
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

    pdl_wait();   // x is produced, and y may be read, by the preceding work on the stream
    i8_digits(p.x, nsb, pnsb, pb_first, count * CPI < pnsb ? count * CPI : pnsb, image, meta, warp, kI8Warps, lane);
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
        // K 32j, the accumulator columns 64c + 8j .. +7 (no accumulation
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
            const uint32_t dcol = tmem + static_cast<uint32_t>(kI8Dcol0 + a * CPI * kI8ColAcc);
            const uint32_t acol = tmem + static_cast<uint32_t>(a * CPI * kI8ColTmem);
            if (elect_one()) {
#pragma unroll
                for (int c = 0; c < CPI; ++c) {
                    const int pb = i * CPI + c;
                    if (pb >= nsb) continue;   // past the row: no MMA, the epilogue skips it
                    const uint32_t img = smem_addr(image + static_cast<size_t>(slot_of(pb)) * kI8ImageBytes);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        // K position 32j: atom j / 4 (N * 128 bytes each), 32 bytes
                        // per MMA inside it
                        const uint64_t bdesc = sw128_kmajor_desc(img + (j >> 2) * (kI8N * 128) + (j & 3) * 32);
                        mma_i8_tmem_a(dcol + static_cast<uint32_t>(c * kI8ColAcc + j * kI8N),
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
        // Two warps per lane quarter share each item: with two columns per
        // item half h takes column h, with one half h takes sub-blocks 4h ..
        // 4h+3. Each keeps its own f64 row total; at the end of a piece (the
        // CTA's part of a tile) half 1 hands its total to half 0 (shared
        // memory, a named barrier per quarter), which adds the two in that
        // order and stores y or the piece.
        const int quarter = warp % kI8Quarters;
        const int half = (warp - kI8DecodeWarps) / kI8Quarters;
        const int row = 32 * quarter + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
        double ytot = 0.0;
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
            if (__all_sync(0xFFFFFFFFu, ok)) {
                const int c = CPI == 2 ? half : 0;   // the item's column this half reads
                // this row's superblock header (d, dmin, sc_j, m_j)
                const uint4 hraw = hring[(hs * CPI + c) * kI8Rows + row];
                __syncwarp();
                if (lane == 0) mbar_arrive(&hfree[hs]);
                tc_fence_after_sync();
                constexpr int kNJ = CPI == 2 ? 8 : 4;   // sub-blocks this half sums
                uint32_t r[kNJ * kI8Limbs];            // D_j[l] at (j - j0) * 5 + l: the digit columns only
                const uint32_t dcol = lane_base + static_cast<uint32_t>(kI8Dcol0 + a * CPI * kI8ColAcc +
                                                                        (CPI == 2 ? c * kI8ColAcc : 32 * half));
#pragma unroll
                for (int jj = 0; jj < kNJ; ++jj) tmem_load_5cols(dcol + static_cast<uint32_t>(jj * kI8N), r + jj * kI8Limbs);
                tmem_wait_ld();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dfree[a]);
                const int pb = i * CPI + c;
                if (pb < nsb) {   // a column past the row (odd K/256, two columns per item) adds nothing
                    const Header hd = decode_header(hraw);
                    const double* mb = meta + static_cast<size_t>(slot_of(pb)) * kI8MetaDoubles;
                    double part;
                    if constexpr (CPI == 2) part = i8_column_sum<8>(r, hd, mb, 0);
                    else part = i8_column_sum<4>(r, hd, mb, 4 * half);
                    ytot = fma(mb[0], part, ytot);
                }
            } else {
                abort_flag = 1;
            }
            if (i == npi - 1 || it == count - 1) {
                // end of this CTA's piece of `tile`: the halves' totals, added
                double* xc = xchange + parity * kI8Rows;
                if (half == 1) xc[row] = ytot;
                named_barrier_sync(1 + quarter, 64);
                if (half == 0) {
                    const double tot = ytot + xc[row];
                    if (istart == 0 && i == npi - 1) {   // the whole tile
                        if (!abort_flag && grow < p.n) p.y[grow] = static_cast<float>(tot);
                    } else {
                        // a piece: slot 0 is published at once (the rest of
                        // the range follows), slot 1 after the last item
                        const int slot = tile == tile0 ? 0 : 1;
                        p.part[(static_cast<size_t>(blockIdx.x) * 2 + slot) * kI8Rows + row] = tot;
                        if (slot == 0 && it < count - 1) {
                            i8_publish_piece(p.part, p.done, p.y, p.n, npi, items, tile, row, &last_piece[0],
                                             abort_flag != 0);
                        } else {
                            has1 = true;
                            tile1 = tile;
                        }
                    }
                }
                ytot = 0.0;
                istart = 0;
                parity ^= 1;
            }
            if (++i == npi) {
                i = 0;
                ++tile;
            }
        }
        // every thread of the first half takes this branch or none (the
        // pieces depend only on the CTA's range)
        if (half == 0 && has1)
            i8_publish_piece(p.part, p.done, p.y, p.n, npi, items, tile1, row, &last_piece[1], abort_flag != 0);
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
    if (m != 1 || n < 1 || k < kQK || k % kQK != 0 || num_sms < 1) return false;
    const int nsb = k / kQK;
    const long long tiles = (static_cast<long long>(n) + kI8Rows - 1) / kI8Rows;
    if (tiles * nsb >= (1LL << 31) / num_sms) return false;   // item counts in 32 bits
    const bool whole = i8_whole_tiles(static_cast<int>(tiles), num_sms);
    // whole tiles per CTA, or enough (tile, column) units per CTA that the
    // kernel's fixed cost (digit image, pipeline fill, cut tiles) pays off
    if (!whole && tiles * nsb < static_cast<long long>(kI8MinItemsPerCta) * num_sms) return false;
    const int budget = max_smem < kI8SmemBudget ? max_smem : kI8SmemBudget;
    // two columns per item unless an odd K/256 is small (the padded column of
    // each tile's last item would be a large share of the work)
    for (int cpi = (nsb % 2 == 0 || nsb >= 9) ? 2 : 1; cpi >= 1; --cpi) {
        I8Config c;
        c.cpi = cpi;
        c.npi = (nsb + cpi - 1) / cpi;
        c.items = tiles * c.npi;
        c.whole = whole ? 1 : 0;
        c.ctas = whole ? num_sms : static_cast<int>(c.items < num_sms ? c.items : num_sms);
        c.items_per_cta_max = whole ? (tiles + c.ctas - 1) / c.ctas * c.npi : (c.items + c.ctas - 1) / c.ctas;
        const long long pnsb = static_cast<long long>(c.npi) * cpi;
        c.ncols = static_cast<int>(c.items_per_cta_max * cpi < pnsb ? c.items_per_cta_max * cpi : pnsb);
        const int fit = i8_fit_stages(c.ncols, cpi);
        // the kernel's instantiations: 4 two-column stages; 8, 6 or 4 one-column
        if (fit < kI8MinWStages) continue;
        c.wstages = cpi == 2 ? 4 : fit >= 8 ? 8 : fit >= 6 ? 6 : 4;
        c.smem = i8_smem_bytes_cfg(c.ncols, cpi, c.wstages);
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
// tile resetting its counter) and the pieces, [SMs][2][128] f64. Calls on one
// stream run in order, so a stream's calls never share it concurrently.
struct I8Scratch {
    void* ptr = nullptr;
    int tiles_cap = 0;
    int ctas_cap = 0;
};
std::mutex g_i8_mu;
std::map<std::pair<int, uintptr_t>, I8Scratch> g_i8_scratch;

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// Counters then pieces: the pieces' offset for a region of `tiles` counters.
size_t scratch_part_offset(int tiles) { return align256(static_cast<size_t>(tiles) * sizeof(unsigned)); }

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
        e = cudaMallocAsync(&p, scratch_part_offset(tcap) + static_cast<size_t>(ccap) * 2 * kI8Rows * sizeof(double),
                            stream);
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

int i8_set_attributes() {
    cudaError_t e = cudaFuncSetAttribute(q4k_gemv_i8_kernel<8, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kI8SmemBudget);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemv_i8_kernel<6, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kI8SmemBudget);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemv_i8_kernel<4, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kI8SmemBudget);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemv_i8_kernel<4, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kI8SmemBudget);
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
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

int launch_gemv_i8(const DeviceInfo& dev, const void* w, const float* x, float* y, int n, int k,
                   cudaStream_t stream) {
    I8Config c;
    if (!i8_config(1, n, k, dev.sm_count, dev.max_smem_optin, &c)) return Q4K_ERR_SHAPE;   // not reached
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
            e = cudaMallocAsync(&own, scratch_part_offset(tiles) + static_cast<size_t>(c.ctas) * 2 * kI8Rows * sizeof(double),
                                stream);
            if (e == cudaSuccess) e = cudaMemsetAsync(own, 0, static_cast<size_t>(tiles) * sizeof(unsigned), stream);
            done = static_cast<unsigned*>(own);
            part = reinterpret_cast<double*>(static_cast<uint8_t*>(own) + scratch_part_offset(tiles));
        }
        if (e != cudaSuccess) return cuda_failure(e);
    }
    const I8Params ip{x, y, part, done, n, nsb, tiles, c.npi, c.ncols, c.whole};
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
    e = c.cpi == 2          ? cudaLaunchKernelEx(&cfg, q4k_gemv_i8_kernel<4, 2>, map, ip)
        : c.wstages >= 8    ? cudaLaunchKernelEx(&cfg, q4k_gemv_i8_kernel<8, 1>, map, ip)
        : c.wstages >= 6    ? cudaLaunchKernelEx(&cfg, q4k_gemv_i8_kernel<6, 1>, map, ip)
                            : cudaLaunchKernelEx(&cfg, q4k_gemv_i8_kernel<4, 1>, map, ip);
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
