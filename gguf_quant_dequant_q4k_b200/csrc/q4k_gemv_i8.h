// q4k_gemv_i8.h -- host-side interface of the one-vector tensor-core GEMV for
// tall matrices (q4k_gemv_i8.cu): when it applies, its launch sizes.
#pragma once

#include <cuda_runtime.h>

namespace q4k {

struct DeviceInfo;

constexpr int kI8Rows = 128;      // rows per tile: the MMA's M
constexpr int kI8MaxWStages = 8;  // weight stages: 8, 6 or 4 of one superblock column of a tile,
constexpr int kI8MinWStages = 4;  // or 4 of two, as many as fit beside the digit image
constexpr int kI8PreStages = 2;   // weight stages requested before the dependency wait
constexpr int kI8SmemBudget = 220 * 1024;   // dynamic shared memory a CTA may use
constexpr int kI8MaxImbalance = 8;   // whole tiles per CTA: the busiest CTA at most 1/8 above the mean
constexpr int kI8MinItemsPerCta = 5; // cut tiles: at least this many items per CTA on average

// Superblocks per row the kernel keeps the vector's digit image for (shared
// memory): K up to 256 times this.
int i8_max_nsb(int max_smem);
int i8_smem_bytes(int nsb);
// superblock columns per item (1 or 2) and weight stages (of that many columns)
int i8_cpi(int nsb);
int i8_wstages(int nsb);
int i8_threads();
// Whole 128-row tiles per CTA: at least one tile per SM and the busiest CTA
// at most 1/kI8MaxImbalance above the mean.
bool i8_whole_tiles(int tiles, int num_sms);
// CTAs: one per SM at most, owning whole tiles (i8_whole_tiles) or equal
// contiguous ranges of the tiles x nsb (tile, superblock column) items.
int i8_ctas(int tiles, int nsb, int num_sms);
// True if some CTA range starts inside a tile (the tile is then finished from
// pieces in the stream's scratch).
bool i8_cuts_tiles(int tiles, int nsb, int num_sms);
// True if q4k_gemv runs one vector of this shape on the kernel: the vector's
// digit image fits beside four weight stages, and the CTAs own whole tiles or
// at least kI8MinItemsPerCta items each on average.
bool i8_applies(int m, int n, int k, int num_sms, int max_smem);

int i8_set_attributes();
int launch_gemv_i8(const DeviceInfo& dev, const void* w, const float* x, float* y, int n, int k,
                   cudaStream_t stream);
int read_i8_fault_flags(unsigned* flags);

}  // namespace q4k
