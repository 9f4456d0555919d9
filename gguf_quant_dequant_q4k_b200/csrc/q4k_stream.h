// q4k_stream.h -- host-side interface of the streaming GEMV kernel.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace q4k {

// Row segments per ring stage (a multiple of 4). Measured on B200: 8 is
// slower than 4 on every decode shape (register spills, LM head 101.7 ->
// 110.3 us).
constexpr int kStreamSegRows = 4;
constexpr int kStreamMaxM = 2;          // vectors handled by one streaming launch (1 or 2)

// Lane geometry for S 16-byte quant slices per lane and row (S = 1 or 2):
// quant bytes per lane and row, lanes per superblock, superblock positions
// per warp.
__host__ __device__ constexpr int lane_bytes(int s) { return 16 * s; }
__host__ __device__ constexpr int lanes_per_sb(int s) { return 128 / lane_bytes(s); }
__host__ __device__ constexpr int pos_per_warp(int s) { return 32 / lanes_per_sb(s); }
// Quant slices (16 bytes = 32 weights) per lane and row: 1, or 2 for one
// vector on very tall matrices (kWideMinRows rows or more per CTA: an LM
// head). Two slices halve the per-item overheads but double the x registers
// (64 per lane), so fewer warps fit; measured on B200 they win only where a
// CTA has hundreds of rows to stream (LM head 128256x4096: 96.7 vs 98.7 us)
// and lose 10-50 % on every decode projection below that.
constexpr int kWideMinRows = 512;
// Compute threads per CTA (plus one producer warp): one slice, one vector: 20
// warps (x: 32 registers per lane; five or six warps per sub-partition at 80
// registers; 23 measured no faster); two vectors or two slices: 15 warps (x:
// 64 registers per lane; four warps per
// sub-partition at 128 registers).
__host__ __device__ constexpr int stream_max_threads(int m, int slices) {
    return (m == 1 && slices == 1) ? 640 : 480;
}
// Registers per thread: each of the SM's four sub-partitions has 16384
// registers for its share of the CTA's warps (allocated in multiples of 8).
__host__ __device__ constexpr int stream_max_regs(int m, int slices) {
    return 16384 / (((stream_max_threads(m, slices) / 32 + 1 + 3) / 4) * 32) / 8 * 8;
}
// Superblocks per row one team of one-slice lanes covers (K <= 20480 for one
// vector, 15360 for two: the warps one team may have); two-slice lanes cover
// twice as many (K <= 30720, one vector).
constexpr int kStreamMaxNsb = 80;
constexpr int kStreamMaxTeams = 20;     // one producer lane per team
constexpr int kStreamMaxDepth = 8;
constexpr int kStreamSmemBudget = 220 * 1024;
// Fused SwiGLU: most shared memory for the CTA's gate/up row totals.
constexpr int kStreamMaxRowsBytes = 32 * 1024;
// Ring stages each team requests before waiting on the preceding kernel (at
// most the ring depth); the rest follow once every compute warp has issued its
// x loads, so x is not queued behind them.
constexpr int kStreamPreStages = 1;
// Bytes of one entry of the kernel's table of team ranges.
constexpr int kTeamRangeBytes = 32;

struct StreamParams {
    const uint8_t* w;
    const uint8_t* w_up;        // fused SwiGLU: the up projection (w is the gate)
    const float* x;
    float* y;
    int n, k, nsb;
    int cluster;                // CTAs per thread-block cluster (1 = no cluster)
    int rows_base, rows_extra;  // cluster q owns rows_base (+1 if q < rows_extra) rows
    int teams, team_warps, depth;
    int stage_bytes;            // bytes per ring slot
    int off_coef, off_red, off_part, off_tr, off_bar;  // shared-memory offsets (bytes)
    int off_rows, rows_cap;     // fused: row totals [M][2 * rows_cap] (gate rows, up rows)
    int slices;                 // 16-byte quant slices per lane (1 or 2; 0: one 8-byte half)
    // A K-chunk of longer rows: the kernel's rows are nsb superblocks starting
    // at superblock sb_off of rows nsb_row long (nsb_row == nsb, sb_off == 0
    // for a whole matrix); x points at the chunk's first element of vector 0
    // and vectors are x_stride floats apart.
    int nsb_row, sb_off, x_stride;
    int accumulate;             // 1: y += the chunk's sums (a later K-chunk); 0: y = sums
    int x_ready;                // 1: x is not written by the preceding work: the compute
                                // warps read it without waiting for the grid dependency
};

// Launch policy. 0: one CTA per SM with up to 20 compute warps and 220 KiB
// of shared memory. 1 / 2: compact CTAs (at most kCompactRegs registers and
// kCompactSmem bytes of shared memory, so that a CTA of the next kernel can be
// resident beside each one) wherever a team fits, kCompactCtasPerSm per SM.
// 3: as 1, except for very tall matrices (kWideMinRows rows per SM or more),
// which keep the classic CTA.
#ifndef Q4K_PLAN_MODE
#define Q4K_PLAN_MODE 3
#endif
constexpr int kPlanMode = Q4K_PLAN_MODE;
constexpr int kCompactRegs = 32768;
constexpr int kCompactSmem = 112 * 1024;
constexpr int kCompactCtasPerSm = (Q4K_PLAN_MODE == 2) ? 1 : 2;

constexpr int kStreamMaxCluster = 8;    // cluster sizes the kernel supports (portable limit)
constexpr int kClusterMaxRows = 8;      // split rows across a cluster only for N < 8 ...
constexpr int kClusterMinNsb = 32;      // ... and K >= 8192

// Fills the launch configuration; returns 0 if the streaming kernel does not
// handle (m, k) or the shared-memory budget cannot hold two stages. fused:
// gate and up rows of a CTA share its teams (no cluster split).
// max_clusters[c] (c = 1..8, may be null) is how many clusters of c CTAs can
// be resident at once; without it the planner assumes num_sms / c.
int plan_stream(int m, int n, int k, int num_sms, int max_smem, const int* max_clusters,
                bool fused, StreamParams* sp, int* grid, int* block, int* smem_bytes);

// Resident clusters of c CTAs (c = 1..8) for the streaming kernel on the
// current device, into max_clusters[c]; 0 where the query is not possible.
int stream_cluster_occupancy(int m, int* max_clusters);

// Most superblocks per row one team can cover for m vectors at `slices`
// (0 if the streaming kernel has no such configuration).
int stream_max_nsb(int m, int slices);

// w_up != null: fused gate/up SwiGLU (w is the gate projection).
int launch_stream(const StreamParams& sp, int grid, int block, int smem_bytes, const void* w,
                  const void* w_up, const float* x, float* y, int m, cudaStream_t stream);

// Per-device kernel attributes (dynamic shared memory opt-in).
int stream_set_attributes();

// Reads and clears the device fault flags (synchronises the device).
int read_fault_flags(unsigned* flags);

// Enqueues a one-thread kernel whose bounded mbarrier wait runs out (nothing
// completes the phase), raising the copy-timeout fault flag.
int selftest_wait_timeout(cudaStream_t stream);

}  // namespace q4k
