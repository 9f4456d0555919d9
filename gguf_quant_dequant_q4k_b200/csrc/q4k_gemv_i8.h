// q4k_gemv_i8.h -- host-side interface of the integer tensor-core GEMV for
// one to four vectors (q4k_gemv_i8.cu): when it applies, its launch sizes.
#pragma once

#include <cuda_runtime.h>

namespace q4k {

struct DeviceInfo;

constexpr int kI8Rows = 128;      // rows per tile: the MMA's M
constexpr int kI8MaxM = 4;        // vectors per launch (1, 2, or 3-4 as four)
constexpr int kI8MaxWStages = 8;  // weight stages: 8, 6 or 4 of one superblock column of a tile,
constexpr int kI8MinWStages = 4;  // or 4 of two, as many as fit beside the digit image
constexpr int kI8PreStages = 2;   // weight stages requested before the dependency wait
constexpr int kI8SmemBudget = 220 * 1024;   // dynamic shared memory a CTA may use
constexpr int kI8MaxImbalance = 8;   // whole tiles per CTA: the busiest CTA at most 1/8 above the mean
constexpr int kI8MinItemsPerCta = 5; // cut tiles: at least this many items per CTA on average
// Fewer tiles than SMs: one whole tile per CTA if that adds at most this many
// superblock columns to the busiest CTA (against equal item ranges), by
// vectors per launch: measured, cut tiles' publication is worth ~3 us, i.e.
// ~7 / 5 / 3 columns of one / two / four vectors.
constexpr int i8_whole_extra_cols(int mv) { return mv == 1 ? 7 : mv == 2 ? 5 : 3; }

// One call's launch shape on the kernel.
struct I8Config {
    int mv;                       // vectors the kernel is built for: 1, 2 or 4 (m = 3 as four)
    int cpi;                      // superblock columns per item (1 or 2; 1 for four vectors)
    int npi;                      // items per tile: ceil(nsb / cpi)
    int ncols;                    // digit-image slots a CTA keeps (its columns, padded)
    int wstages;                  // weight stages of cpi columns
    int ctas;                     // one per SM at most
    int whole;                    // 1: equal ranges of whole tiles, else of items
    int cuts;                     // 1: some tile is cut between CTAs (pieces in the scratch)
    int smem;                     // dynamic shared memory per CTA
    long long items;              // tiles * npi
    long long items_per_cta_max;
};

// Whole 128-row tiles per CTA: at least one tile per SM and the busiest CTA
// at most 1/kI8MaxImbalance above the mean (i8_config also takes one tile per
// CTA on fewer CTAs than SMs, per i8_whole_extra_cols).
bool i8_whole_tiles(int tiles, int num_sms);
int i8_threads();
// True (and *cfg filled) if q4k_gemv runs m <= kI8MaxM vectors of this shape
// on the kernel: whole tiles per CTA or at least kI8MinItemsPerCta superblock
// columns per CTA on average, and the CTA's digit image beside at least four
// weight stages (two columns per item where that fits, else one). Whole tiles
// run on min(tiles, SMs) CTAs.
bool i8_config(int m, int n, int k, int num_sms, int max_smem, I8Config* cfg);

int i8_set_attributes();
int launch_gemv_i8(const DeviceInfo& dev, const void* w, const float* x, float* y, int m, int n, int k,
                   cudaStream_t stream, bool x_ready);
int read_i8_fault_flags(unsigned* flags);

}  // namespace q4k
