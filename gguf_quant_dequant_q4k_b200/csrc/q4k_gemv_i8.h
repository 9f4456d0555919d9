// q4k_gemv_i8.h -- host-side interface of the one-vector tensor-core GEMV for
// tall matrices (q4k_gemv_i8.cu): when it applies, its launch sizes.
#pragma once

#include <cuda_runtime.h>

namespace q4k {

struct DeviceInfo;

constexpr int kI8Rows = 128;      // rows per tile: the MMA's M
constexpr int kI8MaxWStages = 8;  // weight stages (one superblock column of a tile each) ...
constexpr int kI8MinWStages = 4;  // ... 8, 6 or 4, as many as fit beside the digit image
constexpr int kI8PreStages = 2;   // weight stages requested before the dependency wait
constexpr int kI8MaxImbalance = 8;   // whole tiles per CTA: at most 1/8 of the CTAs' time idle
constexpr int kI8SmemBudget = 220 * 1024;   // dynamic shared memory a CTA may use

// Superblocks per row the kernel keeps the vector's digit image for (shared
// memory): K up to 256 times this.
int i8_max_nsb(int max_smem);
int i8_smem_bytes(int nsb);
int i8_wstages(int nsb);
int i8_threads();
// CTAs: one per SM at most, each owning whole 128-row tiles.
int i8_ctas(int tiles, int num_sms);
// True if q4k_gemv runs one vector of this shape on the kernel: every SM gets
// whole tiles with the busiest CTA at most 1/kI8MaxImbalance above the mean,
// and the digit image fits beside the weight stages.
bool i8_applies(int m, int n, int k, int num_sms, int max_smem);

int i8_set_attributes();
int launch_gemv_i8(const DeviceInfo& dev, const void* w, const float* x, float* y, int n, int k,
                   cudaStream_t stream);
int read_i8_fault_flags(unsigned* flags);

}  // namespace q4k
