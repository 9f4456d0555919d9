// q4k_gemv_tc.h -- host-side interface of the tensor-core batched GEMV
// (q4k_gemv_tc.cu): its constants, launch sizes and workspace.
#pragma once

#include <cstddef>
#include <cuda.h>
#include <cuda_runtime.h>

namespace q4k {

struct DeviceInfo;

constexpr int kTcRows = 128;        // rows per tile: the MMA's M
constexpr int kTcLimbs = 5;         // base-128 digits per scaled x value
constexpr int kTcMaxM = 16;         // vectors per launch
constexpr int kTcMetaDoubles = 10;  // per vector block: 2^(E-33), S0_0..7, pad
constexpr int kTcSmemBudget = 212 * 1024;   // both stage rings
constexpr int kTcMinM = 3;          // q4k_gemv runs m >= 3 on this kernel

// Vectors a launch is laid out for (8 or 16; missing ones are zero) and the
// MMA's N: digit rows l*mp + i, rounded up to a multiple of 16.
__host__ __device__ constexpr int tc_vectors_padded(int m) { return m <= 8 ? 8 : 16; }
__host__ __device__ constexpr int tc_n_mp(int mp) { return (kTcLimbs * mp + 15) / 16 * 16; }

int tc_smem_bytes(int mp);
int tc_stages(int mp);
int tc_threads();
int tc_k_position_host(int t);
// CTAs (one per SM at most) sharing the tiles x nsb superblock columns in
// equal contiguous ranges.
int tc_ctas(int tiles, int nsb, int num_sms);
// Device workspace one q4k_gemv call on this kernel allocates (stream-ordered)
// for the vectors' digit images, block metadata and the partial totals of
// tiles cut between CTAs.
size_t tc_workspace_bytes(int m, int n, int k, int num_sms);

// 2-D tensor map of a Q4_K matrix as bytes (rows of nsb*144 bytes, boxes of
// one superblock column by kTcRows rows, rows past n read as zeros); false if
// the driver's encoder is unavailable or rejects the map.
bool make_weight_map(CUtensorMap* map, const void* w, int n, int nsb);

int tc_set_attributes();
int launch_gemv_tc(const DeviceInfo& dev, const void* w, const float* x, float* y, int m, int n,
                   int k, cudaStream_t stream);
int read_tc_fault_flags(unsigned* flags);

}  // namespace q4k
