// q4k_gemm_f16.cu -- the prefill path: the fp16 mirror of a Q4_K matrix, the
// f32 -> fp16 activation convert, and y = x16 * W16^T on the 5th-generation
// tensor cores (tcgen05) with f32 accumulation in tensor memory.
//
// What it computes follows "memra-engine 0.83.1, src/f16_ffi.rs": the module
// doc (a resident fp16 dequant mirror of the weights feeds an fp16 GEMM with
// f32 accumulation for prefill, m >= 512), `memra_q4_K_dequant_f16` (Q4_K
// superblocks -> row-major fp16 mirror, called from `build_q4k_f16_raw`),
// `memra_f16_cvt` (f32 -> fp16 activations), `memra_f16_pp_gemm_pre` (the GEMM
// on pre-converted activations: w_f16, xh_f16, y_f32, m, n, k) and
// `memra_f16_pp_gemm` (convert into a caller-provided scratch, then the GEMM).
// The page runs the GEMM through cuBLASLt ("TN": both operands K-major); here
// it is a hand-written kernel:
//
// * Tile. A CTA owns a 128 x BN tile of y^T: 128 rows of W (output features,
//   the MMA's M) by BN tokens (the MMA's N), so each TMEM lane holds one
//   feature and its BN token columns, and the epilogue's stores of one token
//   column by a warp are 32 consecutive floats of y (coalesced).
// * Operands. Each k-block is 64 fp16 (128 bytes) of K: one TMA tensor load
//   of the 128 x 64 W box and one of the BN x 64 x box, both with the
//   128-byte swizzle the MMA's shared-memory descriptors expect, into a ring
//   of `kGemmStages` stages (full / empty mbarriers). Rows past n or m are
//   filled with zeros by TMA and never stored.
// * MMA. One thread issues four tcgen05.mma (K = 16 each) per k-block and
//   commits the stage back to the producer when they complete; a final commit
//   tells the epilogue the accumulator is complete.
// * Epilogue. Each of the 4 warps reads its 32 TMEM lanes 32 columns at a
//   time (tcgen05.ld) and stores them to y (row-major m x n f32).
// All waits are bounded; a wait that gives up raises Q4K_FAULT_COPY_TIMEOUT,
// and the CTA lets the copies and MMAs it issued complete (bounded) before
// releasing shared memory and TMEM.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <mutex>

#include "q4k_internal.h"
#include "q4k_superblock.cuh"
#include "q4k_tcgen05.cuh"

namespace q4k {

// Raised (Q4K_FAULT_COPY_TIMEOUT) by a GEMM CTA whose bounded wait gave up;
// read and cleared by q4k_device_fault_flags(). Never set in normal operation.
__device__ unsigned int g_gemm_fault_flags = 0;

namespace {

constexpr int kGemmThreads = 128;
constexpr int kGemmBM = 128;          // W rows per tile (MMA M)
constexpr int kGemmBK = 64;           // K elements per k-block (128 bytes of fp16)
constexpr int kGemmMmaK = 16;         // K per tcgen05.mma of kind::f16
constexpr int kGemmRingBytes = 192 * 1024;

__host__ __device__ constexpr int stage_a_bytes() { return kGemmBM * kGemmBK * 2; }
__host__ __device__ constexpr int stage_b_bytes(int bn) { return bn * kGemmBK * 2; }
// Ring stages: as many as 192 KiB holds, at most 8 (4 for 256-token tiles,
// 6 for 128, 8 for 64).
__host__ __device__ constexpr int gemm_stages(int bn) {
    return kGemmRingBytes / (stage_a_bytes() + stage_b_bytes(bn)) < 8
               ? kGemmRingBytes / (stage_a_bytes() + stage_b_bytes(bn))
               : 8;
}
constexpr int gemm_smem_bytes(int bn) {
    return 1024 /* alignment slack */ + gemm_stages(bn) * (stage_a_bytes() + stage_b_bytes(bn)) +
           (2 * gemm_stages(bn) + 1) * 8 + 16;
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
q4k_gemm_f16_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                    float* __restrict__ y, int m, int n, int k) {
    constexpr int kGemmStages = gemm_stages(BN);
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base: the swizzled operand tiles need it
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sa = smem;                                          // [stages][128][64] fp16
    uint8_t* sb = smem + kGemmStages * stage_a_bytes();          // [stages][BN][64] fp16
    uint64_t* full = reinterpret_cast<uint64_t*>(sb + kGemmStages * stage_b_bytes(BN));
    uint64_t* empty = full + kGemmStages;
    uint64_t* accum = empty + kGemmStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
    __shared__ volatile int abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tile_n = blockIdx.x;       // 128-row block of W
    const int tile_m = blockIdx.y;       // BN-token block of x
    const int nkb = k / kGemmBK;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        fence_mbar_init();
        tma_prefetch_map(&map_w);
        tma_prefetch_map(&map_x);
    }
    if (warp == 1) tmem_alloc(tmem_slot, BN);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ TMA producer
        int issued = 0;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % kGemmStages;
            if (kb >= kGemmStages) {
                // the MMAs of k-block kb - stages released this stage
                const uint32_t par = static_cast<uint32_t>(((kb / kGemmStages) - 1) & 1);
                if (abort_flag || !mbar_wait_bounded(&empty[s], par, &g_gemm_fault_flags)) {
                    abort_flag = 1;
                    break;
                }
            }
            mbar_arrive_expect_tx(&full[s], stage_a_bytes() + stage_b_bytes(BN));
            tma_load_2d(sa + s * stage_a_bytes(), &map_w, kb * kGemmBK, tile_n * kGemmBM, &full[s]);
            tma_load_2d(sb + s * stage_b_bytes(BN), &map_x, kb * kGemmBK, tile_m * BN, &full[s]);
            ++issued;
        }
        // Copies of the last `stages` k-blocks may still be in flight if the MMA
        // side gave up: let them land (bounded) before shared memory is released.
        const int first = issued > kGemmStages ? issued - kGemmStages : 0;
        for (int kb = first; kb < issued; ++kb)
            mbar_wait_bounded(&full[kb % kGemmStages], static_cast<uint32_t>((kb / kGemmStages) & 1),
                              &g_gemm_fault_flags);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = mma_f16_idesc(kGemmBM, BN);
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % kGemmStages;
            const uint32_t par = static_cast<uint32_t>((kb / kGemmStages) & 1);
            if (abort_flag || !mbar_wait_bounded(&full[s], par, &g_gemm_fault_flags)) {
                abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t a0 = smem_addr(sa + s * stage_a_bytes());
            const uint32_t b0 = smem_addr(sb + s * stage_b_bytes(BN));
#pragma unroll
            for (int kk = 0; kk < kGemmBK / kGemmMmaK; ++kk) {
                mma_f16(tmem_base, sw128_kmajor_desc(a0 + kk * kGemmMmaK * 2),
                        sw128_kmajor_desc(b0 + kk * kGemmMmaK * 2), idesc,
                        (kb > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&empty[s]);
        }
        mma_commit(accum);   // arrives once every MMA issued above has completed
    }
    __syncwarp();

    // ---------------------------------------------------------------- epilogue
    const bool done = mbar_wait_bounded(accum, 0u, &g_gemm_fault_flags);
    tc_fence_after_sync();
    if (done && !abort_flag) {
        const int row = tile_n * kGemmBM + warp * 32 + lane;     // feature: TMEM lane
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
            uint32_t r[32];
            tmem_load_32cols(lane_addr + static_cast<uint32_t>(c0), r);
            const int tok0 = tile_m * BN + c0;
            if (row < n) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int tok = tok0 + j;
                    if (tok < m) y[static_cast<size_t>(tok) * n + row] = __uint_as_float(r[j]);
                }
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, BN);
    }
}

// f32 -> fp16 (round to nearest even), four values per thread per step.
__global__ void q4k_f32_to_f16_kernel(const float* __restrict__ x, __half* __restrict__ out,
                                      long long count) {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    const long long n4 = count / 4;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += stride) {
        const float4 v = reinterpret_cast<const float4*>(x)[i];
        __half2 lo = __floats2half2_rn(v.x, v.y);
        __half2 hi = __floats2half2_rn(v.z, v.w);
        uint2 o;
        o.x = *reinterpret_cast<uint32_t*>(&lo);
        o.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>(out)[i] = o;
    }
    for (long long i = n4 * 4 + static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
         i < count; i += stride)
        out[i] = __float2half_rn(x[i]);
}

// Q4_K -> fp16 mirror: the f32 dequantised value (one rounding) rounded to
// binary16. Same mapping as the f32 dequant: a warp per superblock per step,
// lane L writes weights 8L..8L+7 (one 16-byte store).
constexpr int kMirrorThreads = 256;

__global__ void __launch_bounds__(kMirrorThreads)
q4k_dequant_f16_kernel(const uint8_t* __restrict__ w, __half* __restrict__ out, long long total_sb) {
    const int lane = threadIdx.x & 31;
    const long long warp0 = (static_cast<long long>(blockIdx.x) * kMirrorThreads + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * kMirrorThreads) >> 5;
    const int g = lane >> 3;
    const int r = (lane & 7) * 8;
    const int high = r >= 32;
    const int l0 = r & 31;
    const int j = 2 * g + high;
    for (long long s = warp0; s < total_sb; s += nwarps) {
        const uint8_t* blk = w + s * kBlockBytes;
        const Header hd = decode_header(ldg_nc_v4(blk));
        const uint2 qb = ldg_nc_v2(blk + kQsOffset + 32 * g + l0);
        float dsc, dm;
        subblock_coeffs(hd, j, dsc, dm);
        const int shift = high ? 4 : 0;
        uint32_t packed[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const uint32_t word = (e < 4) ? qb.x : qb.y;
            const uint32_t q0 = (word >> (8 * (e & 3) + shift)) & 15u;
            const uint32_t q1 = (word >> (8 * ((e + 1) & 3) + shift)) & 15u;
            __half2 h2 = __floats2half2_rn(weight_value(dsc, dm, q0), weight_value(dsc, dm, q1));
            packed[e / 2] = *reinterpret_cast<uint32_t*>(&h2);
        }
        *reinterpret_cast<uint4*>(out + s * kQK + 8 * lane) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime once.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Row-major [rows][k] fp16 matrix, boxes of box_rows x 64 with the 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int rows, int k, int box_rows) {
    EncodeTiledFn fn = encode_tiled();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(k) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kGemmBK), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
int launch_gemm_bn(const void* w16, const void* x16, float* y, int m, int n, int k,
                   cudaStream_t stream) {
    CUtensorMap mw, mx;
    if (!make_map(&mw, w16, n, k, kGemmBM) || !make_map(&mx, x16, m, k, BN))
        return cuda_failure(cudaErrorInvalidValue);
    const dim3 grid((n + kGemmBM - 1) / kGemmBM, (m + BN - 1) / BN);
    q4k_gemm_f16_kernel<BN><<<grid, kGemmThreads, gemm_smem_bytes(BN), stream>>>(mw, mx, y, m, n, k);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

}  // namespace

int gemm_set_attributes() {
    cudaError_t e = cudaFuncSetAttribute(q4k_gemm_f16_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         gemm_smem_bytes(64));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemm_f16_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem_bytes(128));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(q4k_gemm_f16_kernel<256>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem_bytes(256));
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

// Tokens per CTA tile: the one that gives the fewest waves of tiles times the
// tile's cost, a narrower MMA (N) streaming its operands less efficiently
// through shared memory per flop (cost weights 1.5 / 1.1 / 1.0 for N = 64 /
// 128 / 256).
int gemm_tile_tokens(int m, int n, int num_sms) {
    static const int kN[3] = {256, 128, 64};
    static const double kCost[3] = {1.0, 1.1, 1.5};
    int best = 256;
    double best_t = 1e300;
    for (int i = 0; i < 3; ++i) {
        const long long tiles = static_cast<long long>((n + kGemmBM - 1) / kGemmBM) *
                                ((m + kN[i] - 1) / kN[i]);
        const long long waves = (tiles + num_sms - 1) / num_sms;
        const double t = static_cast<double>(waves) * kN[i] * kCost[i];
        if (t < best_t - 1e-9) {
            best_t = t;
            best = kN[i];
        }
    }
    return best;
}

int launch_gemm_f16(const void* w16, const void* x16, float* y, int m, int n, int k, int num_sms,
                    cudaStream_t stream) {
    switch (gemm_tile_tokens(m, n, num_sms)) {
        case 64: return launch_gemm_bn<64>(w16, x16, y, m, n, k, stream);
        case 128: return launch_gemm_bn<128>(w16, x16, y, m, n, k, stream);
        default: return launch_gemm_bn<256>(w16, x16, y, m, n, k, stream);
    }
}

int launch_f32_to_f16(const float* x, void* out, long long count, int num_sms,
                      cudaStream_t stream) {
    long long blocks = (count / 4 + 255) / 256 + 1;
    if (blocks > static_cast<long long>(num_sms) * 8) blocks = static_cast<long long>(num_sms) * 8;
    q4k_f32_to_f16_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        x, static_cast<__half*>(out), count);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

int launch_dequant_f16(const void* w, void* out, int n, int k, int num_sms, cudaStream_t stream) {
    const long long total_sb = static_cast<long long>(n) * (k / kQK);
    long long blocks = (total_sb * 32 + kMirrorThreads - 1) / kMirrorThreads;
    if (blocks > static_cast<long long>(num_sms) * 8) blocks = static_cast<long long>(num_sms) * 8;
    q4k_dequant_f16_kernel<<<static_cast<unsigned>(blocks), kMirrorThreads, 0, stream>>>(
        static_cast<const uint8_t*>(w), static_cast<__half*>(out), total_sb);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? Q4K_OK : cuda_failure(e);
}

// ------------------------------------------------ fixed-scratch prefill variant
//
// q4k_prefill_f16_noalloc needs the same fp16 copy of x as q4k_prefill_f16,
// but for callers that cannot allocate device memory it lives in this
// file-scope array instead of a caller buffer. Host code cannot use the
// array's name as a device address (on the host it names a stand-in object),
// so the address is fetched once per device with cudaGetSymbolAddress while
// that device is current, and passed to the kernels.
namespace {

static __device__ __align__(256) __half g_prefill_scratch[Q4K_PREFILL_NOALLOC_MAX_ELEMS];

constexpr int kScratchDevices = 64;
std::once_flag g_scratch_once[kScratchDevices];
void* g_scratch_ptr[kScratchDevices];
cudaError_t g_scratch_status[kScratchDevices];

}  // namespace

int launch_prefill_noalloc(int device, const void* w16, const float* x, float* y, int m, int n,
                           int k, int num_sms, cudaStream_t stream) {
    if (device < 0 || device >= kScratchDevices) return cuda_failure(cudaErrorInvalidDevice);
    std::call_once(g_scratch_once[device], [device] {
        void* ptr = nullptr;
        g_scratch_status[device] = cudaGetSymbolAddress(&ptr, g_prefill_scratch);
        g_scratch_ptr[device] = ptr;
    });
    if (g_scratch_status[device] != cudaSuccess) return cuda_failure(g_scratch_status[device]);
    void* xh = g_scratch_ptr[device];
    int st = launch_f32_to_f16(x, xh, static_cast<long long>(m) * k, num_sms, stream);
    if (st != Q4K_OK) return st;
    return launch_gemm_f16(w16, xh, y, m, n, k, num_sms, stream);
}

int read_gemm_fault_flags(unsigned* flags) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_gemm_fault_flags, sizeof(v));
    if (e != cudaSuccess) return cuda_failure(e);
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_gemm_fault_flags, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_failure(e);
    *flags = v;
    return Q4K_OK;
}

}  // namespace q4k
