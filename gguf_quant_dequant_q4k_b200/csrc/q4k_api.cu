// q4k_api.cu -- the extern "C" entry points declared in include/q4k.h:
// argument validation, status codes and per-device set-up.
//
// Validation follows the pages' host wrappers: a null device pointer is
// refused before launch (`q4k_gemv_indexed_async`, "realizar 0.8.5,
// src/cuda/executor/q4k_gemv_cached.rs"); K must be a multiple of 256
// (`batched_q4k_gemv_into`, "realizar 0.8.5, src/cuda/executor/uses.rs") and is
// refused rather than padded; the byte size N*(K/256)*144 is computed with
// overflow checks (`validate_block_quant_embedding`, "turbospark-runtime
// 0.1.0, src/real_forward_dispatch.rs"); more than Q4K_MAX_M (64) vectors is
// refused rather than looped (`encode_gemm_any`, same page); a failed launch
// returns an error code to the caller (the rc convention of "memra-engine
// 0.83.1, src/f16_ffi.rs", `qmatvec_gemm_f16_raw`: a nonzero rc from
// `memra_f16_pp_gemm` names its class, a CUDA error among them).
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "q4k_gemv_i8.h"
#include "q4k_gemv_tc.h"
#include "q4k_internal.h"
#include "q4k_stream.h"

namespace q4k {

namespace {

thread_local int t_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
DeviceInfo g_dev[kMaxDevices];
int g_dev_status[kMaxDevices];

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

// Weight bytes n*(k/256)*144 in 64 bits; 0 for an invalid shape.
size_t weight_bytes_checked(int n, int k) {
    if (n <= 0 || k <= 0 || (k % Q4K_QK) != 0) return 0;
    return static_cast<size_t>(n) * static_cast<size_t>(k / Q4K_QK) * Q4K_BLOCK_BYTES;
}

}  // namespace

int cuda_failure(cudaError_t e) {
    t_last_cuda_error = static_cast<int>(e);
    return Q4K_ERR_CUDA;
}

int q4k_last_cuda_error_value() { return t_last_cuda_error; }

int current_device_info(DeviceInfo* info) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_failure(e);
    if (dev < 0 || dev >= kMaxDevices) return cuda_failure(cudaErrorInvalidDevice);
    std::call_once(g_dev_once[dev], [dev] {
        DeviceInfo d{};
        cudaError_t e1 = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
        cudaError_t e2 = cudaDeviceGetAttribute(&d.max_smem_optin,
                                                cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        g_dev[dev] = d;
        g_dev_status[dev] = (e1 != cudaSuccess) ? static_cast<int>(e1)
                                                : static_cast<int>(e2);
        if (g_dev_status[dev] == 0 && stream_set_attributes() != Q4K_OK)
            g_dev_status[dev] = q4k_last_cuda_error_value();
        if (g_dev_status[dev] == 0 && gemm_set_attributes() != Q4K_OK)
            g_dev_status[dev] = q4k_last_cuda_error_value();
        if (g_dev_status[dev] == 0 && tc_set_attributes() != Q4K_OK)
            g_dev_status[dev] = q4k_last_cuda_error_value();
        if (g_dev_status[dev] == 0 && i8_set_attributes() != Q4K_OK)
            g_dev_status[dev] = q4k_last_cuda_error_value();
        if (g_dev_status[dev] == 0) {
            stream_cluster_occupancy(1, g_dev[dev].max_clusters[0]);
            stream_cluster_occupancy(2, g_dev[dev].max_clusters[1]);
        }
    });
    if (g_dev_status[dev] != 0) return cuda_failure(static_cast<cudaError_t>(g_dev_status[dev]));
    *info = g_dev[dev];
    return Q4K_OK;
}

}  // namespace q4k

using namespace q4k;

extern "C" {

size_t q4k_weight_bytes(int n, int k) { return weight_bytes_checked(n, k); }

const char* q4k_status_string(int status) {
    switch (status) {
        case Q4K_OK: return "ok";
        case Q4K_ERR_NULL: return "null pointer argument";
        case Q4K_ERR_SHAPE: return "invalid shape (need n > 0, k > 0, k % 256 == 0)";
        case Q4K_ERR_ALIGN: return "misaligned pointer (w, x, out: 16 bytes; y: 4 bytes)";
        case Q4K_ERR_UNSUPPORTED_M: return "unsupported number of vectors (need 1 <= m <= 64)";
        case Q4K_ERR_CUDA: return "CUDA runtime error (see q4k_last_cuda_error)";
        case Q4K_ERR_OVERLAP: return "output overlaps an input";
        case Q4K_ERR_RANGE: return "embedding token outside the table's rows";
        case Q4K_ERR_CAPACITY:
            return "m * k exceeds the fixed scratch of q4k_prefill_f16_noalloc "
                   "(Q4K_PREFILL_NOALLOC_MAX_ELEMS)";
        default: return "unknown status";
    }
}

int q4k_last_cuda_error(void) { return t_last_cuda_error; }

int q4k_device_fault_flags(unsigned int* flags) {
    if (flags == nullptr) return Q4K_ERR_NULL;
    unsigned a = 0, b = 0, c = 0, t = 0, i = 0;
    int st = read_fault_flags(&a);
    if (st != Q4K_OK) return st;
    st = read_embed_fault_flags(&b);
    if (st != Q4K_OK) return st;
    st = read_gemm_fault_flags(&c);
    if (st != Q4K_OK) return st;
    st = read_tc_fault_flags(&t);
    if (st != Q4K_OK) return st;
    st = read_i8_fault_flags(&i);
    if (st != Q4K_OK) return st;
    *flags = a | b | c | t | i;
    return Q4K_OK;
}

int q4k_selftest_wait_timeout(q4k_stream_t stream) {
    DeviceInfo dev;
    int st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    return selftest_wait_timeout(reinterpret_cast<cudaStream_t>(stream));
}

int q4k_embed_lookup_f32(const void* table, unsigned long long table_bytes, int rows, int cols,
                         int hidden, unsigned int token, float embed_scale, float* out,
                         q4k_stream_t stream) {
    // The checks of `validate_block_quant_embedding`, in its order.
    if (cols != hidden) return Q4K_ERR_SHAPE;
    if (rows <= 0 || token >= static_cast<unsigned>(rows)) return Q4K_ERR_RANGE;
    if (hidden <= 0 || hidden % Q4K_QK != 0) return Q4K_ERR_SHAPE;
    const unsigned long long row_bytes =
        static_cast<unsigned long long>(hidden / Q4K_QK) * Q4K_BLOCK_BYTES;
    const unsigned long long expected = static_cast<unsigned long long>(rows) * row_bytes;
    const unsigned long long selected_end = (static_cast<unsigned long long>(token) + 1) * row_bytes;
    if (table_bytes != expected || selected_end > table_bytes) return Q4K_ERR_SHAPE;
    if (table == nullptr || out == nullptr) return Q4K_ERR_NULL;
    if (!aligned(table, 16) || !aligned(out, 16)) return Q4K_ERR_ALIGN;
    const size_t obytes = static_cast<size_t>(hidden) * sizeof(float);
    if (overlaps(out, obytes, table, static_cast<size_t>(table_bytes))) return Q4K_ERR_OVERLAP;
    DeviceInfo dev;
    int st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    return launch_embed(table, rows, hidden, nullptr, token, 1, embed_scale, out, dev.sm_count,
                        reinterpret_cast<cudaStream_t>(stream));
}

int q4k_embed_gather_f32(const void* table, unsigned long long table_bytes, int rows, int hidden,
                         const int* tokens, int n_tokens, float embed_scale, float* out,
                         q4k_stream_t stream) {
    if (table == nullptr || tokens == nullptr || out == nullptr) return Q4K_ERR_NULL;
    if (rows <= 0 || hidden <= 0 || hidden % Q4K_QK != 0 || n_tokens < 0) return Q4K_ERR_SHAPE;
    const unsigned long long row_bytes =
        static_cast<unsigned long long>(hidden / Q4K_QK) * Q4K_BLOCK_BYTES;
    if (table_bytes != static_cast<unsigned long long>(rows) * row_bytes) return Q4K_ERR_SHAPE;
    if (!aligned(table, 16) || !aligned(tokens, 4) || !aligned(out, 16)) return Q4K_ERR_ALIGN;
    const size_t obytes = static_cast<size_t>(n_tokens) * static_cast<size_t>(hidden) * sizeof(float);
    const size_t tbytes = static_cast<size_t>(n_tokens) * sizeof(int);
    if (overlaps(out, obytes, table, static_cast<size_t>(table_bytes)) ||
        overlaps(out, obytes, tokens, tbytes))
        return Q4K_ERR_OVERLAP;
    if (n_tokens == 0) return Q4K_OK;
    DeviceInfo dev;
    int st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    return launch_embed(table, rows, hidden, tokens, 0u, n_tokens, embed_scale, out, dev.sm_count,
                        reinterpret_cast<cudaStream_t>(stream));
}

int q4k_gemv_plan_for(int m, int n, int k, int num_sms, q4k_gemv_plan* plan) {
    if (plan == nullptr) return Q4K_ERR_NULL;
    if (weight_bytes_checked(n, k) == 0 || num_sms <= 0) return Q4K_ERR_SHAPE;
    if (m < 1 || m > Q4K_MAX_M) return Q4K_ERR_UNSUPPORTED_M;
    return plan_gemv(m, n, k, num_sms, false, plan);
}

int q4k_gemv(const void* w, const float* x, float* y, int m, int n, int k,
             q4k_stream_t stream) {
    return q4k_gemv_ex(w, x, y, m, n, k, 0u, stream);
}

int q4k_gemv_ex(const void* w, const float* x, float* y, int m, int n, int k, unsigned flags,
                q4k_stream_t stream) {
    if (w == nullptr || x == nullptr || y == nullptr) return Q4K_ERR_NULL;
    if ((flags & ~Q4K_GEMV_X_READY) != 0u) return Q4K_ERR_SHAPE;
    const size_t wbytes = weight_bytes_checked(n, k);
    if (wbytes == 0) return Q4K_ERR_SHAPE;
    if (m < 1 || m > Q4K_MAX_M) return Q4K_ERR_UNSUPPORTED_M;
    if (!aligned(w, 16) || !aligned(x, 16) || !aligned(y, 4)) return Q4K_ERR_ALIGN;
    const size_t xbytes = static_cast<size_t>(m) * static_cast<size_t>(k) * sizeof(float);
    const size_t ybytes = static_cast<size_t>(m) * static_cast<size_t>(n) * sizeof(float);
    if (overlaps(y, ybytes, w, wbytes) || overlaps(y, ybytes, x, xbytes)) return Q4K_ERR_OVERLAP;
    DeviceInfo dev;
    int st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    return launch_gemv(dev, w, nullptr, x, y, m, n, k, reinterpret_cast<cudaStream_t>(stream),
                       (flags & Q4K_GEMV_X_READY) != 0u);
}

int q4k_gemv_swiglu_plan_for(int m, int n, int k, int num_sms, q4k_gemv_plan* plan) {
    if (plan == nullptr) return Q4K_ERR_NULL;
    if (weight_bytes_checked(n, k) == 0 || num_sms <= 0) return Q4K_ERR_SHAPE;
    if (m < 1 || m > Q4K_MAX_M) return Q4K_ERR_UNSUPPORTED_M;
    return plan_gemv(m, n, k, num_sms, true, plan);
}

int q4k_gemv_swiglu(const void* w_gate, const void* w_up, const float* x, float* y, int m, int n,
                    int k, q4k_stream_t stream) {
    if (w_gate == nullptr || w_up == nullptr || x == nullptr || y == nullptr) return Q4K_ERR_NULL;
    const size_t wbytes = weight_bytes_checked(n, k);
    if (wbytes == 0) return Q4K_ERR_SHAPE;
    if (m < 1 || m > Q4K_MAX_M) return Q4K_ERR_UNSUPPORTED_M;
    if (!aligned(w_gate, 16) || !aligned(w_up, 16) || !aligned(x, 16) || !aligned(y, 4))
        return Q4K_ERR_ALIGN;
    const size_t xbytes = static_cast<size_t>(m) * static_cast<size_t>(k) * sizeof(float);
    const size_t ybytes = static_cast<size_t>(m) * static_cast<size_t>(n) * sizeof(float);
    if (overlaps(y, ybytes, w_gate, wbytes) || overlaps(y, ybytes, w_up, wbytes) ||
        overlaps(y, ybytes, x, xbytes))
        return Q4K_ERR_OVERLAP;
    DeviceInfo dev;
    int st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    return launch_gemv(dev, w_gate, w_up, x, y, m, n, k, reinterpret_cast<cudaStream_t>(stream));
}

int q4k_dequant_f32(const void* w, float* out, int n, int k, q4k_stream_t stream) {
    if (w == nullptr || out == nullptr) return Q4K_ERR_NULL;
    const size_t wbytes = weight_bytes_checked(n, k);
    if (wbytes == 0) return Q4K_ERR_SHAPE;
    if (!aligned(w, 16) || !aligned(out, 16)) return Q4K_ERR_ALIGN;
    const size_t obytes = static_cast<size_t>(n) * static_cast<size_t>(k) * sizeof(float);
    if (overlaps(out, obytes, w, wbytes)) return Q4K_ERR_OVERLAP;
    DeviceInfo dev;
    int st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    return launch_dequant(w, out, n, k, dev.sm_count, reinterpret_cast<cudaStream_t>(stream));
}

int q4k_dequant_f16(const void* w, void* out, int n, int k, q4k_stream_t stream) {
    if (w == nullptr || out == nullptr) return Q4K_ERR_NULL;
    const size_t wbytes = weight_bytes_checked(n, k);
    if (wbytes == 0) return Q4K_ERR_SHAPE;
    if (!aligned(w, 16) || !aligned(out, 16)) return Q4K_ERR_ALIGN;
    const size_t obytes = static_cast<size_t>(n) * static_cast<size_t>(k) * 2;
    if (overlaps(out, obytes, w, wbytes)) return Q4K_ERR_OVERLAP;
    DeviceInfo dev;
    int st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    return launch_dequant_f16(w, out, n, k, dev.sm_count, reinterpret_cast<cudaStream_t>(stream));
}

int q4k_f32_to_f16(const float* x, void* out, unsigned long long count, q4k_stream_t stream) {
    if (x == nullptr || out == nullptr) return Q4K_ERR_NULL;
    if (count > (1ull << 62)) return Q4K_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(out, 16)) return Q4K_ERR_ALIGN;
    if (overlaps(out, static_cast<size_t>(count) * 2, x, static_cast<size_t>(count) * 4))
        return Q4K_ERR_OVERLAP;
    if (count == 0) return Q4K_OK;
    DeviceInfo dev;
    int st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    return launch_f32_to_f16(x, out, static_cast<long long>(count), dev.sm_count,
                             reinterpret_cast<cudaStream_t>(stream));
}

namespace {

// Shape and pointer checks shared by the two GEMM entry points.
int check_gemm(const void* w16, const void* x16, const float* y, int m, int n, int k) {
    if (w16 == nullptr || x16 == nullptr || y == nullptr) return Q4K_ERR_NULL;
    if (m <= 0 || n <= 0 || k <= 0 || k % Q4K_GEMM_K_MULTIPLE != 0) return Q4K_ERR_SHAPE;
    if (!aligned(w16, 16) || !aligned(x16, 16) || !aligned(y, 4)) return Q4K_ERR_ALIGN;
    const size_t wbytes = static_cast<size_t>(n) * static_cast<size_t>(k) * 2;
    const size_t xbytes = static_cast<size_t>(m) * static_cast<size_t>(k) * 2;
    const size_t ybytes = static_cast<size_t>(m) * static_cast<size_t>(n) * 4;
    if (overlaps(y, ybytes, w16, wbytes) || overlaps(y, ybytes, x16, xbytes)) return Q4K_ERR_OVERLAP;
    return Q4K_OK;
}

}  // namespace

int q4k_gemm_f16(const void* w_f16, const void* x_f16, float* y, int m, int n, int k,
                 q4k_stream_t stream) {
    int st = check_gemm(w_f16, x_f16, y, m, n, k);
    if (st != Q4K_OK) return st;
    DeviceInfo dev;
    st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    return launch_gemm_f16(w_f16, x_f16, y, m, n, k, dev.sm_count,
                           reinterpret_cast<cudaStream_t>(stream));
}

int q4k_prefill_f16(const void* w_f16, const float* x, void* x_f16_scratch, float* y, int m, int n,
                    int k, q4k_stream_t stream) {
    if (x == nullptr) return Q4K_ERR_NULL;
    int st = check_gemm(w_f16, x_f16_scratch, y, m, n, k);
    if (st != Q4K_OK) return st;
    if (!aligned(x, 16)) return Q4K_ERR_ALIGN;
    const size_t xbytes = static_cast<size_t>(m) * static_cast<size_t>(k) * 4;
    const size_t hbytes = static_cast<size_t>(m) * static_cast<size_t>(k) * 2;
    const size_t wbytes = static_cast<size_t>(n) * static_cast<size_t>(k) * 2;
    const size_t ybytes = static_cast<size_t>(m) * static_cast<size_t>(n) * 4;
    if (overlaps(x_f16_scratch, hbytes, x, xbytes) || overlaps(x_f16_scratch, hbytes, w_f16, wbytes) ||
        overlaps(y, ybytes, x, xbytes))
        return Q4K_ERR_OVERLAP;
    DeviceInfo dev;
    st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = launch_f32_to_f16(x, x_f16_scratch, static_cast<long long>(m) * k, dev.sm_count, s);
    if (st != Q4K_OK) return st;
    return launch_gemm_f16(w_f16, x_f16_scratch, y, m, n, k, dev.sm_count, s);
}

int q4k_prefill_f16_noalloc(const void* w_f16, const float* x, float* y, int m, int n, int k,
                            q4k_stream_t stream) {
    if (w_f16 == nullptr || x == nullptr || y == nullptr) return Q4K_ERR_NULL;
    if (m <= 0 || n <= 0 || k <= 0 || k % Q4K_GEMM_K_MULTIPLE != 0) return Q4K_ERR_SHAPE;
    if (static_cast<long long>(m) * k > Q4K_PREFILL_NOALLOC_MAX_ELEMS) return Q4K_ERR_CAPACITY;
    if (!aligned(w_f16, 16) || !aligned(x, 16) || !aligned(y, 4)) return Q4K_ERR_ALIGN;
    const size_t xbytes = static_cast<size_t>(m) * static_cast<size_t>(k) * 4;
    const size_t wbytes = static_cast<size_t>(n) * static_cast<size_t>(k) * 2;
    const size_t ybytes = static_cast<size_t>(m) * static_cast<size_t>(n) * 4;
    if (overlaps(y, ybytes, w_f16, wbytes) || overlaps(y, ybytes, x, xbytes)) return Q4K_ERR_OVERLAP;
    DeviceInfo dev;
    int st = current_device_info(&dev);
    if (st != Q4K_OK) return st;
    int device = 0;
    const cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) return cuda_failure(e);
    return launch_prefill_noalloc(device, w_f16, x, y, m, n, k, dev.sm_count,
                                  reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
