// q4k_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "q4k.h"  // include/ (on the include path)

namespace q4k {

// Per-device facts the launch planner needs, read once per device.
struct DeviceInfo {
    int sm_count;
    int max_smem_optin;        // largest dynamic shared memory a CTA may opt in to
    int max_clusters[2][9];    // resident clusters of c CTAs, streaming kernel, m = 1 / 2
};

// Returns Q4K_OK and fills *info for the current device, or Q4K_ERR_CUDA.
int current_device_info(DeviceInfo* info);

// Records `e` as the calling thread's last CUDA error and returns Q4K_ERR_CUDA.
int cuda_failure(cudaError_t e);
int q4k_last_cuda_error_value();

// Opt-in dynamic shared memory per CTA on B200 (227 KiB), assumed by the
// host-only planner when no device is queried.
constexpr int kB200SmemOptin = 232448;

// Host-only launch planning (no CUDA calls); fused: gate/up SwiGLU.
int plan_gemv(int m, int n, int k, int num_sms, bool fused, q4k_gemv_plan* plan);

// Enqueue the planned kernels on the current device. Arguments are already
// validated. w2 != null: y = silu(W x) * (W2 x) (fused gate/up SwiGLU).
// x_ready: x is not written by the preceding work on the stream (read before
// the grid dependency resolves; y still written after it).
int launch_gemv(const DeviceInfo& dev, const void* w, const void* w2, const float* x, float* y,
                int m, int n, int k, cudaStream_t stream, bool x_ready = false);

int launch_dequant(const void* w, float* out, int n, int k, int num_sms, cudaStream_t stream);

// Embedding rows: row tokens[i] (device array) or, if tokens is null, row
// `token` (n_tokens = 1), dequantised and scaled. Arguments are validated.
int launch_embed(const void* table, long long rows, int hidden, const int* tokens, unsigned token,
                 int n_tokens, float scale, float* out, int num_sms, cudaStream_t stream);

// Reads and clears the embedding kernel's fault flags (synchronises).
int read_embed_fault_flags(unsigned* flags);

// Prefill path (fp16 mirror + tensor-core GEMM). Arguments are validated.
int gemm_set_attributes();
int gemm_tile_tokens(int m, int n, int num_sms);   // tokens per CTA tile (64, 128 or 256)
int launch_gemm_f16(const void* w16, const void* x16, float* y, int m, int n, int k, int num_sms,
                    cudaStream_t stream);
int launch_f32_to_f16(const float* x, void* out, long long count, int num_sms,
                      cudaStream_t stream);
int launch_dequant_f16(const void* w, void* out, int n, int k, int num_sms, cudaStream_t stream);
int read_gemm_fault_flags(unsigned* flags);
// q4k_prefill_f16 with the file-scope scratch array of q4k_gemm_f16.cu
// (m * k <= Q4K_PREFILL_NOALLOC_MAX_ELEMS, checked by the caller); `device` is
// the current device.
int launch_prefill_noalloc(int device, const void* w16, const float* x, float* y, int m, int n,
                           int k, int num_sms, cudaStream_t stream);

}  // namespace q4k
