// q4k_gemv.cu -- y = W x for Q4_K W and 1..64 f32 vectors (q4k_gemv).
//
// General path (any K, tiles of up to 8 vectors): one warp per output row
// (the row-per-warp mapping of the pages' `Q4KGemv`, "realizar 0.8.5,
// src/cuda/executor/q4k_gemv_cached.rs", grid (n,1) x 32 threads), with each
// decoded weight applied to all m vectors
// (`BatchedQ4KGemv`, "realizar 0.8.5, src/cuda/executor/uses.rs": dequantise
// once, multiply by M input vectors).
//
// Per step a warp covers 4 superblocks of its row: lane = 8*sb + c, where
// c = 0..7 selects the 16-byte slice 16c..16c+15 of Q. That slice's byte l
// carries weight 64g+16h+l (low nibble, sub-block 2g) and weight 64g+32+16h+l
// (high nibble, sub-block 2g+1), with g = c/2, h = c%2. The warp's 32 quant
// loads are 4 x 128 contiguous bytes.
#include "q4k_gemv_i8.h"
#include "q4k_gemv_tc.h"
#include "q4k_internal.h"
#include "q4k_stream.h"
#include "q4k_superblock.cuh"
#include "q4k_swiglu.cuh"

namespace q4k {

namespace {

constexpr int kRowsThreads = 256;
constexpr int kRowsMaxM = 8;   // vectors per launch of the general kernel

// Adds row `wr`'s products with the M vectors into acc[i] (lane's share: the
// superblocks b = sub, sub + 4, ... and quant slice c of each).
template <int M>
__device__ __forceinline__ void rows_dot(const uint8_t* __restrict__ wr, const float* __restrict__ x,
                                         int nsb, int k, int lane, float (&acc)[M]) {
    const int c = lane & 7, sub = lane >> 3, g = c >> 1, h = c & 1;
    for (int b = sub; b < nsb; b += 4) {
        const uint8_t* sb = wr + static_cast<size_t>(b) * kBlockBytes;
        const Header hd = decode_header(ldg_nc_v4(sb));
        const uint4 qv = ldg_nc_v4(sb + kQsOffset + 16 * c);
        float dsc0, dm0, dsc1, dm1;
        subblock_coeffs(hd, 2 * g, dsc0, dm0);
        subblock_coeffs(hd, 2 * g + 1, dsc1, dm1);
        const uint32_t words[4] = {qv.x, qv.y, qv.z, qv.w};
        float wl[16], wh[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint32_t byte = (words[e >> 2] >> (8 * (e & 3))) & 0xFFu;
            wl[e] = weight_value(dsc0, dm0, byte & 15u);
            wh[e] = weight_value(dsc1, dm1, byte >> 4);
        }
        const int k0 = b * kQK + 64 * g + 16 * h;
#pragma unroll
        for (int i = 0; i < M; ++i) {
            const float4* xl = reinterpret_cast<const float4*>(x + static_cast<size_t>(i) * k + k0);
            const float4* xh = xl + 8;  // +32 floats
            float s = acc[i];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 a = __ldg(xl + v);
                const float4 bq = __ldg(xh + v);
                s = fmaf(wl[4 * v + 0], a.x, s);
                s = fmaf(wl[4 * v + 1], a.y, s);
                s = fmaf(wl[4 * v + 2], a.z, s);
                s = fmaf(wl[4 * v + 3], a.w, s);
                s = fmaf(wh[4 * v + 0], bq.x, s);
                s = fmaf(wh[4 * v + 1], bq.y, s);
                s = fmaf(wh[4 * v + 2], bq.z, s);
                s = fmaf(wh[4 * v + 3], bq.w, s);
            }
            acc[i] = s;
        }
    }
}

// FUSED: y = silu(W x) * (W2 x) (the SwiGLU of a gate and an up projection).
template <int M, bool FUSED>
__global__ void __launch_bounds__(kRowsThreads)
q4k_gemv_rows_kernel(const uint8_t* __restrict__ w, const uint8_t* __restrict__ w2,
                     const float* __restrict__ x, float* __restrict__ y, int n, int k) {
    const int nsb = k / kQK;
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * kRowsThreads + threadIdx.x) >> 5;
    const int nwarps = gridDim.x * (kRowsThreads / 32);
    for (int row = warp; row < n; row += nwarps) {
        float acc[M], acc2[M];
#pragma unroll
        for (int i = 0; i < M; ++i) acc[i] = acc2[i] = 0.f;
        rows_dot<M>(w + static_cast<size_t>(row) * nsb * kBlockBytes, x, nsb, k, lane, acc);
        if (FUSED) rows_dot<M>(w2 + static_cast<size_t>(row) * nsb * kBlockBytes, x, nsb, k, lane, acc2);
#pragma unroll
        for (int i = 0; i < M; ++i) {
            float s = acc[i], s2 = acc2[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
                if (FUSED) s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, off);
            }
            if (lane == 0) y[static_cast<size_t>(i) * n + row] = FUSED ? silu_mul(s, s2) : s;
        }
    }
}

template <int M>
void launch_rows(const q4k_gemv_plan& plan, const void* w, const void* w2, const float* x,
                 float* y, int n, int k, cudaStream_t stream) {
    if (w2 != nullptr)
        q4k_gemv_rows_kernel<M, true><<<plan.grid, plan.block, 0, stream>>>(
            static_cast<const uint8_t*>(w), static_cast<const uint8_t*>(w2), x, y, n, k);
    else
        q4k_gemv_rows_kernel<M, false><<<plan.grid, plan.block, 0, stream>>>(
            static_cast<const uint8_t*>(w), nullptr, x, y, n, k);
}

}  // namespace

namespace {

// Vectors per streaming launch: 1 or 2 (q4k_gemv runs m >= 3 on the
// tensor-core kernels); the fused SwiGLU runs any m as pairs.
int group_size(int m) { return m <= 2 ? m : 2; }

// K split into the fewest equal chunks (whole superblocks) one team covers:
// each chunk is a launch over strided row segments, later chunks adding into y.
struct KChunks {
    int count, nsb;   // chunks, superblocks per chunk (the last one may be shorter)
};

KChunks k_chunks(int mk, int nsb) {
    const int maxnsb = stream_max_nsb(mk, mk == 1 ? 2 : 1);
    KChunks c{1, nsb};
    if (maxnsb <= 0 || nsb <= maxnsb) return c;
    c.count = (nsb + maxnsb - 1) / maxnsb;
    c.nsb = (nsb + c.count - 1) / c.count;
    return c;
}

}  // namespace

// m >= 3 vectors (plain projection) where the integer kernel does not take
// them: the tensor-core batched kernel, one pair of launches (digits, GEMV)
// per group of up to 16 vectors.
bool use_tc(int m, bool fused) { return !fused && m >= kTcMinM; }

// One to four vectors (plain projection) on a matrix whose tiles or items give
// every SM enough work, the digit image beside four weight stages: the
// integer tensor-core kernel, one launch (checked before use_tc).
bool use_i8(int m, int n, int k, int num_sms, int max_smem, bool fused) {
    I8Config c;
    return !fused && i8_config(m, n, k, num_sms, max_smem, &c);
}

int plan_gemv_device(int m, int n, int k, int num_sms, int max_smem, const int* max_clusters,
                     bool fused, q4k_gemv_plan* plan, StreamParams* sp) {
    I8Config ic;
    if (!fused && i8_config(m, n, k, num_sms, max_smem, &ic)) {
        const long long tiles = (static_cast<long long>(n) + kI8Rows - 1) / kI8Rows;
        plan->kernel = Q4K_KERNEL_I8;
        plan->grid = ic.ctas;
        plan->block = i8_threads();
        plan->smem_bytes = ic.smem;
        plan->cluster = 1;
        plan->teams = 0;
        plan->depth = ic.wstages;
        plan->launches = 1;
        plan->units = tiles * (k / kQK);   // (128-row tile, superblock column) units, cpi per item
        plan->units_per_cta_max = ic.items_per_cta_max * ic.cpi;
        plan->slices = ic.cpi;             // superblock columns per item
        return Q4K_OK;
    }
    if (use_tc(m, fused)) {
        const int tiles = (n + kTcRows - 1) / kTcRows;
        const int grid = tc_ctas(tiles, k / kQK, num_sms);
        const long long items = static_cast<long long>(tiles) * (k / kQK);
        const int groups = (m + kTcMaxM - 1) / kTcMaxM;
        const int mp = tc_vectors_padded(m < kTcMaxM ? m : kTcMaxM);
        plan->kernel = Q4K_KERNEL_TC;
        plan->grid = grid;
        plan->block = tc_threads();
        plan->smem_bytes = tc_smem_bytes(mp);
        plan->cluster = 1;
        plan->teams = 0;
        plan->depth = tc_stages(mp);
        plan->launches = 2 * groups;
        plan->units = items;   // (128-row tile, superblock column) items
        plan->units_per_cta_max = (items + grid - 1) / grid;
        plan->slices = 0;
        return Q4K_OK;
    }
    StreamParams q{};
    int grid = 0, block = 0, smem = 0;
    const int nsb = k / kQK;
    const int mk = group_size(m);
    const int* cl = max_clusters;
    bool ok = plan_stream(mk, n, k, num_sms, max_smem, cl, fused, &q, &grid, &block, &smem) != 0;
    int chunks = 1;
    if (!ok && !fused) {
        const KChunks c = k_chunks(mk, nsb);
        if (c.count > 1) {
            chunks = c.count;
            ok = plan_stream(mk, n, c.nsb * kQK, num_sms, max_smem, cl, false, &q, &grid, &block,
                             &smem) != 0;
        }
    }
    if (ok) {
        plan->kernel = Q4K_KERNEL_STREAM;
        plan->grid = grid;
        plan->block = block;
        plan->smem_bytes = smem;
        plan->teams = q.teams;
        plan->depth = q.depth;
        plan->launches = ((m + mk - 1) / mk) * chunks;
        plan->cluster = q.cluster;
        plan->units = n;
        plan->units_per_cta_max = q.rows_base + (q.rows_extra > 0 ? 1 : 0);
        plan->slices = q.slices;
        if (sp) *sp = q;
        return Q4K_OK;
    }
    const int warps_per_cta = kRowsThreads / 32;
    long long ctas = (static_cast<long long>(n) + warps_per_cta - 1) / warps_per_cta;
    const long long cap = static_cast<long long>(num_sms) * 8;
    if (ctas > cap) ctas = cap;
    const long long warps = ctas * warps_per_cta;
    plan->kernel = Q4K_KERNEL_WARP_ROWS;
    plan->cluster = 1;
    plan->grid = static_cast<int>(ctas);
    plan->block = kRowsThreads;
    plan->smem_bytes = 0;
    plan->teams = 0;
    plan->depth = 0;
    plan->launches = (m + kRowsMaxM - 1) / kRowsMaxM;   // tiles of up to 8 vectors
    plan->units = n;
    plan->units_per_cta_max = ((n + warps - 1) / warps) * warps_per_cta;
    plan->slices = 0;
    return Q4K_OK;
}

int plan_gemv(int m, int n, int k, int num_sms, bool fused, q4k_gemv_plan* plan) {
    return plan_gemv_device(m, n, k, num_sms, kB200SmemOptin, nullptr, fused, plan, nullptr);
}

int launch_gemv(const DeviceInfo& dev, const void* w, const void* w2, const float* x, float* y,
                int m, int n, int k, cudaStream_t stream, bool x_ready) {
    q4k_gemv_plan plan;
    const bool fused = w2 != nullptr;
    if (use_i8(m, n, k, dev.sm_count, dev.max_smem_optin, fused)) return launch_gemv_i8(dev, w, x, y, m, n, k, stream, x_ready);
    if (use_tc(m, fused)) return launch_gemv_tc(dev, w, x, y, m, n, k, stream);
    const int gsz = group_size(m);
    int st = plan_gemv_device(m, n, k, dev.sm_count, dev.max_smem_optin,
                              dev.max_clusters[gsz == 1 ? 0 : 1], fused, &plan, nullptr);
    if (st != Q4K_OK) return st;
    if (plan.kernel == Q4K_KERNEL_STREAM) {
        const int nsb = k / kQK;
        for (int i0 = 0; i0 < m; i0 += gsz) {
            const int mk = (m - i0) < gsz ? (m - i0) : gsz;     // vectors of this group
            const int* cl = dev.max_clusters[mk == 1 ? 0 : 1];
            StreamParams sp;
            int g = 0, b = 0, sm = 0;
            KChunks c{1, nsb};
            if (!plan_stream(mk, n, k, dev.sm_count, dev.max_smem_optin, cl, fused, &sp, &g, &b, &sm))
                c = k_chunks(mk, nsb);
            for (int ci = 0; ci < c.count; ++ci) {
                const int sb0 = ci * c.nsb;
                const int nsb_c = (nsb - sb0) < c.nsb ? (nsb - sb0) : c.nsb;
                if (c.count > 1 &&
                    !plan_stream(mk, n, nsb_c * kQK, dev.sm_count, dev.max_smem_optin, cl, fused, &sp,
                                 &g, &b, &sm))
                    return Q4K_ERR_SHAPE;   // not reached: a chunk never exceeds a team
                sp.nsb_row = nsb;
                sp.sb_off = sb0;
                sp.x_stride = k;
                sp.accumulate = ci > 0 ? 1 : 0;
                sp.x_ready = x_ready && !fused ? 1 : 0;
                st = launch_stream(sp, g, b, sm, w, w2,
                                   x + static_cast<size_t>(i0) * k + static_cast<size_t>(sb0) * kQK,
                                   y + static_cast<size_t>(i0) * n, mk, stream);
                if (st != Q4K_OK) return st;
            }
        }
        return Q4K_OK;
    }
    // vector tiles of up to 8 (the tiling of `batched_q4k_gemv_into`)
    for (int i0 = 0; i0 < m; i0 += kRowsMaxM) {
        const int mi = (m - i0) < kRowsMaxM ? (m - i0) : kRowsMaxM;
        const float* xi = x + static_cast<size_t>(i0) * k;
        float* yi = y + static_cast<size_t>(i0) * n;
        switch (mi) {
            case 1: launch_rows<1>(plan, w, w2, xi, yi, n, k, stream); break;
            case 2: launch_rows<2>(plan, w, w2, xi, yi, n, k, stream); break;
            case 3: launch_rows<3>(plan, w, w2, xi, yi, n, k, stream); break;
            case 4: launch_rows<4>(plan, w, w2, xi, yi, n, k, stream); break;
            case 5: launch_rows<5>(plan, w, w2, xi, yi, n, k, stream); break;
            case 6: launch_rows<6>(plan, w, w2, xi, yi, n, k, stream); break;
            case 7: launch_rows<7>(plan, w, w2, xi, yi, n, k, stream); break;
            default: launch_rows<8>(plan, w, w2, xi, yi, n, k, stream); break;
        }
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_failure(e);
    }
    return Q4K_OK;
}

}  // namespace q4k
