/*
 * q4k.h -- C ABI of libq4k_b200.so: GGUF Q4_K GEMV and dequantisation on one
 * NVIDIA B200 (sm_100a).
 *
 * The operation (y = W x with W stored as Q4_K superblocks, decoded on the fly)
 * is the one the realizar pages launch as `Q4KGemv`, `TiledQ4KGemv`,
 * `ChunkedTiledQ4KGemv`, `MwvQ4KGemv` ("realizar 0.8.5,
 * src/cuda/executor/q4k_gemv_cached.rs": `q4k_gemv_cached`,
 * `q4k_gemv_indexed_async`) and `BatchedQ4KGemv` for batches of vectors
 * ("realizar 0.8.5, src/cuda/executor/uses.rs": `batched_q4k_gemv_into`, up
 * to 8 vectors per kernel, larger batches in tiles).
 * The dequantisation is the one "memra-engine 0.83.1, src/f16_ffi.rs" declares
 * as `memra_q4_K_dequant_f16` (Q4_K 144-byte superblocks to a row-major
 * mirror), here with an f32 target.
 *
 * Q4_K superblock (256 weights, 144 bytes; the pages give the size, the field
 * layout is GGUF's block_q4_K):
 *     bytes   0..1   d     binary16, little-endian
 *     bytes   2..3   dmin  binary16, little-endian
 *     bytes   4..15  S[12] eight 6-bit scales sc_j and eight 6-bit mins m_j
 *                          (j < 4: sc_j = S[j]&63, m_j = S[j+4]&63;
 *                           j >= 4: sc_j = (S[j+4]&15) | (S[j-4]>>6)<<4,
 *                                   m_j  = (S[j+4]>>4) | (S[j]>>6)<<4)
 *     bytes  16..143 Q[128] byte Q[32g+l] holds weight 64g+l (low nibble) and
 *                          weight 64g+32+l (high nibble), g = 0..3, l = 0..31
 *     weight t (sub-block j = t/32): value = d*sc_j*q_t - dmin*m_j
 *
 * Conventions shared by every entry point:
 *   - Every pointer is DEVICE memory owned by the caller; the library never
 *     allocates, frees or keeps a pointer after the call returns.
 *   - W is row-major by output row: row r is K/256 consecutive superblocks,
 *     N*(K/256)*144 bytes in all ("weights: N x K/256 Q4_K super-blocks",
 *     `batched_q4k_gemv_into` doc comment). K must be a positive multiple of
 *     256; nothing is padded.
 *   - Work is enqueued on `stream` (NULL = the legacy default stream) and the
 *     call returns without synchronising; no host copy, allocation or JIT
 *     happens inside a call (the pages sync and copy to the host only in their
 *     debugging wrappers, and preload modules because compiling during graph
 *     capture fails).
 *   - Arguments are validated before anything is enqueued; an invalid call
 *     returns a status and enqueues nothing (a null weight pointer "poisons
 *     the CUDA context" if launched, `q4k_gemv_indexed_async`). A status of
 *     Q4K_ERR_CUDA means the launch itself failed; q4k_last_cuda_error()
 *     then returns the cudaError_t. Faults during execution surface at the
 *     caller's next synchronisation, as for any asynchronous CUDA work.
 *   - Output buffers must not overlap any input (checked: Q4K_ERR_OVERLAP).
 */
#ifndef Q4K_H
#define Q4K_H

#include <stddef.h>

#if defined(__GNUC__)
#define Q4K_API __attribute__((visibility("default")))
#else
#define Q4K_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *q4k_stream_t;

enum q4k_status {
    Q4K_OK = 0,
    Q4K_ERR_NULL = 1,           /* a required pointer is NULL                     */
    Q4K_ERR_SHAPE = 2,          /* n <= 0, k <= 0, k % 256 != 0, or size overflow  */
    Q4K_ERR_ALIGN = 3,          /* w or x not 16-byte aligned, y/out not 4-byte    */
    Q4K_ERR_UNSUPPORTED_M = 4,  /* m outside 1..Q4K_MAX_M                          */
    Q4K_ERR_CUDA = 5,           /* a CUDA runtime call failed (see last_cuda_error) */
    Q4K_ERR_OVERLAP = 6,        /* an output range overlaps an input range         */
    Q4K_ERR_RANGE = 7,          /* an embedding token outside the table's rows     */
    Q4K_ERR_CAPACITY = 8        /* q4k_prefill_f16_noalloc: m*k above its fixed scratch */
};

/* Bits of q4k_device_fault_flags(). */
#define Q4K_FAULT_COPY_TIMEOUT 1u  /* a bounded wait on a bulk copy, a tensor copy or an
                                      MMA commit gave up                               */
#define Q4K_FAULT_TOKEN_RANGE 2u   /* q4k_embed_gather_f32 met a token outside the table */

#define Q4K_QK 256          /* weights per superblock */
#define Q4K_BLOCK_BYTES 144 /* bytes per superblock   */
#define Q4K_MAX_M 64        /* most vectors per q4k_gemv call */
#define Q4K_GEMM_K_MULTIPLE 64 /* q4k_gemm_f16 / q4k_prefill_f16: k % 64 == 0 */
#define Q4K_PREFILL_NOALLOC_MAX_ELEMS 8388608 /* q4k_prefill_f16_noalloc: m*k limit (16 MiB fp16) */

/*
 * y = W x for m vectors.
 *   w  : N*(K/256)*144 bytes of Q4_K superblocks, row-major by output row,
 *        16-byte aligned.
 *   x  : m x K float32, row-major (vector i at x + i*K), 16-byte aligned
 *        ("input: M x K row-major", `batched_q4k_gemv_into`).
 *   y  : m x N float32, row-major (vector i at y + i*N); fully overwritten,
 *        never accumulated into ("output: M x N row-major").
 *   m  : 1..64 vectors. One to four vectors run on the integer tensor-core
 *        kernel (Q4K_KERNEL_I8, one launch, the weights decoded once for all
 *        of them; m = 3 as four) where the matrix gives every SM whole
 *        128-row tiles or at least 5 (tile, superblock column) items and the
 *        CTA's digit image fits beside four weight stages (one vector:
 *        K <= 256*62); otherwise one or two vectors run on the streaming
 *        kernel (one launch, or K-chunks of it for long K), and three or more
 *        on the tensor-core kernel in groups of up to 16 (the realizar page tiles
 *        m > 8 in `batched_q4k_gemv_into` and has an m = 16 / 32 branch): each
 *        group is a digits launch and a GEMV launch, the weights decoded once
 *        per group. q4k_gemv_plan_for reports the launch count. Larger m is
 *        refused, not looped (the turbospark page, "turbospark-runtime 0.1.0,
 *        src/real_forward_dispatch.rs", `encode_gemm_any`, refuses rather than
 *        silently looping): that is a GEMM's size.
 * Workspace: for m >= 3 on the tensor-core kernel the call allocates a
 * device workspace from the
 * device's default memory pool, stream-ordered on `stream`
 * (cudaMallocAsync / cudaFreeAsync; capturable in a CUDA graph), of
 * (K/256) * (N_mma*512 + 80*mp) + 2048*mp*ctas + 4*ceil(N/128) bytes
 * (mp = 8 or 16, N_mma = 48 or 80, ctas <= SM count): 2.7 MiB for
 * N = 14336, K = 4096, m = 8. m = 2, and m = 1 on the streaming kernel,
 * allocate nothing. The integer kernel with tiles cut between CTAs
 * (q4k_gemv_plan_for: kernel Q4K_KERNEL_I8, units not a multiple of the CTAs'
 * whole-tile ranges) uses a scratch the library keeps per (device, stream):
 * ceil(4*max(tiles, 4096), 256) + 8192*max(ctas, 256) bytes, allocated
 * stream-ordered on the first such call on `stream` outside graph capture
 * (inside a capture with none yet, the call allocates and frees its own,
 * capturable) and kept for the process; every launch leaves its counters
 * zero. Calls on one stream run in order, so it is never shared by two
 * launches at once; a CUDA graph that holds such a call uses the scratch of
 * the stream it was captured on and must not run concurrently with other
 * q4k_gemv calls on that stream.
 * Accuracy: per element |y - sum_k w_nk x_ik| <= 1e-4 * sum_k |w_nk x_ik| + 1e-6,
 * where w_nk is the f32 value d*sc*q - dmin*m; for m <= 2 accumulation is in
 * f32 on the streaming kernel. On the tensor-core and integer kernels the
 * products are exact integers (x scaled per 256-element block by 2^(33 - E)
 * (2^(30 - E) for two to four vectors on the integer kernel), E the exponent
 * of the block's largest |x|, and rounded to an integer) combined in f64, so
 * the bound holds with one more term, 2^-33 * sum_k |w_nk| * max_block(k)
 * |x_i| (2^-30 * ... for those), which is below 1e-6 unless that sum
 * exceeds 8590 (1074) (e.g. K = 14336 and |x| up to ~1 with most of w x
 * cancelling); an inf or NaN in x_i makes every element of y_i NaN.
 * Weight reads may start before the previous kernel on `stream` has finished
 * (programmatic dependent launch): x is read and y written only after it has.
 * W is treated as constant model data: it must not be written by work still
 * pending on `stream` when this is called.
 * Returns a q4k_status.
 */
Q4K_API int q4k_gemv(const void *w, const float *x, float *y, int m, int n, int k,
             q4k_stream_t stream);

/*
 * As q4k_gemv, with flags:
 *   Q4K_GEMV_X_READY: x is already final when the kernel enqueued on
 *     `stream` just before this call begins executing: the call may read x
 *     before that kernel has finished (programmatic dependent launch); y is
 *     still written only after it has. The q4k kernels let their successors
 *     start early, so a chain of q4k calls can run partly at once: x must not
 *     be written by any of them still pending. The typical case: x written by
 *     a kernel that does not trigger its dependents early (or by a copy),
 *     read by one q4k_gemv without the flag and then by further ones with it
 *     (the k and v projections after q, up after gate). Undefined results
 *     otherwise. Applies on the streaming and integer kernels; the batched
 *     tensor-core kernel (m >= 3 on the smaller matrices, m > 4) ignores it.
 * Other bits of `flags` must be zero (Q4K_ERR_SHAPE otherwise). Several GEMVs
 * reading one input are the pages' pattern: an input vector is uploaded once
 * and then serves a series of GEMV launches (`q4k_upload_to_input_buffer`,
 * `q4k_gemv_launch_to_ptr`, "realizar 0.8.5,
 * src/cuda/executor/q4k_gemv_cached.rs"), and a layer normalises its input
 * twice, for attention and for the FFN (`preload_batched_prefill_modules`,
 * "realizar 0.8.5, src/cuda/executor/layers/modules_utilities.rs").
 */
#define Q4K_GEMV_X_READY 0x1u
Q4K_API int q4k_gemv_ex(const void *w, const float *x, float *y, int m, int n, int k, unsigned flags,
                        q4k_stream_t stream);

/*
 * Fused gate/up projection with SwiGLU: y = silu(W_gate x) * (W_up x), where
 * silu(g) = g / (1 + exp(-g)), for m vectors ("realizar 0.8.5" kernel cache
 * page: `FusedGateUpSwigluHwDp4aQ4KGemv { k: hidden_dim, n: intermediate_dim }`;
 * here with f32 x and the exact per-weight dequantisation of q4k_gemv).
 *   w_gate, w_up: two N x K Q4_K matrices laid out as w of q4k_gemv, each
 *        16-byte aligned (they may be the same matrix).
 *   x, y, m, n, k: as for q4k_gemv (y is m x N, fully overwritten).
 * One pass streams both matrices and shares each x load between them; g and u
 * are never written to memory.
 * Accuracy: with t_g, t_u the q4k_gemv bounds of the two projections (t =
 * 1e-4 * sum|w x| + 1e-6), per element
 *   |y - silu(g) u| <= 1.1 t_g (|u| + t_u) + (|silu(g)| + 1.1 t_g) t_u + 1e-6 |y|
 * (silu' lies in [-0.1, 1.1]; the last term is the f32 epilogue: expf, one
 * divide, one multiply).
 * Validation as q4k_gemv; y must not overlap either matrix or x.
 * Returns a q4k_status.
 */
Q4K_API int q4k_gemv_swiglu(const void *w_gate, const void *w_up, const float *x, float *y,
                            int m, int n, int k, q4k_stream_t stream);

/*
 * out = W dequantised to float32, row-major n x k (out[r*k + t] is weight t of
 * row r). Each value is d*sc*q - dmin*m rounded once to f32 (the products are
 * exact in f32), so results are bit-reproducible.
 *   w  : as for q4k_gemv (16-byte aligned).
 *   out: n*k floats, 16-byte aligned, must not overlap w.
 * Returns a q4k_status.
 */
Q4K_API int q4k_dequant_f32(const void *w, float *out, int n, int k, q4k_stream_t stream);

/* Bytes of an n x k Q4_K matrix: n*(k/256)*144; 0 if n <= 0, k <= 0 or
 * k % 256 != 0 (the size rule the memra `build_q8_f16` and turbospark
 * `encode_gemv_any` pages check before every Q4_K launch). */
Q4K_API size_t q4k_weight_bytes(int n, int k);

/* A static, NUL-terminated description of a q4k_status value. Status codes
 * follow the return-code convention of the memra FFI ("memra-engine 0.83.1,
 * src/f16_ffi.rs", `qmatvec_gemm_f16_raw`): every entry point returns an int,
 * 0 on success, and a nonzero code names the class of failure (there: cudaError
 * convert, no cuBLASLt algorithm, matmul status; here: the q4k_status values). */
Q4K_API const char *q4k_status_string(int status);

/* The cudaError_t behind the most recent Q4K_ERR_CUDA returned on the calling
 * thread (0 if none): the CUDA error the memra rc convention folds into its
 * "cudaError" class ("memra-engine 0.83.1, src/f16_ffi.rs",
 * `qmatvec_gemm_f16_raw`), kept here as its own value. */
Q4K_API int q4k_last_cuda_error(void);

/*
 * Embedding lookup: out = row `token` of a Q4_K embedding table, dequantised,
 * times embed_scale ("turbospark-runtime 0.1.0, src/real_forward_dispatch.rs":
 * `validate_q4_k_embedding` then `encode_embed_lookup_q4_k(..., token, hidden,
 * embed_scale)`).
 *   table      : a [rows, cols] Q4_K matrix, table_bytes bytes, 16-byte aligned.
 *   hidden     : the model width the caller expects; out has hidden floats,
 *                16-byte aligned, and must not overlap the table.
 *   out[j]     = fl32(w[j] * embed_scale), w[j] the f32 weight d*sc*q - dmin*m.
 * Checked before launch, in the page's order: cols != hidden -> Q4K_ERR_SHAPE;
 * token >= rows -> Q4K_ERR_RANGE; hidden not a positive multiple of 256 ->
 * Q4K_ERR_SHAPE; table_bytes != rows * (hidden/256) * 144, or the selected row
 * not ending inside the table -> Q4K_ERR_SHAPE. Then NULL, alignment and
 * overlap. Nothing is launched unless every check passes.
 * Returns a q4k_status.
 */
Q4K_API int q4k_embed_lookup_f32(const void *table, unsigned long long table_bytes, int rows,
                                 int cols, int hidden, unsigned int token, float embed_scale,
                                 float *out, q4k_stream_t stream);

/*
 * Row gather for n_tokens tokens held in device memory (a batch of lookups
 * whose tokens were produced on the device): out[i*hidden + j] = fl32(w[j] of
 * row tokens[i] * embed_scale).
 *   table, table_bytes, rows, hidden: as above (the table is [rows, hidden];
 *                table_bytes must equal rows * (hidden/256) * 144).
 *   tokens     : n_tokens int32 in device memory, 4-byte aligned.
 *   out        : n_tokens x hidden float32, 16-byte aligned, no overlap.
 * A token outside 0..rows-1 cannot be refused before launch: its output row is
 * written as zeros and Q4K_FAULT_TOKEN_RANGE is raised in the device fault
 * flags. n_tokens == 0 launches nothing.
 * Returns a q4k_status.
 */
Q4K_API int q4k_embed_gather_f32(const void *table, unsigned long long table_bytes, int rows,
                                 int hidden, const int *tokens, int n_tokens, float embed_scale,
                                 float *out, q4k_stream_t stream);

/*
 * Reads and clears the calling device's fault flags (Q4K_FAULT_* bits). The
 * pages report every failure to the caller as a return code (the rc classes of
 * `memra_f16_pp_gemm`, "memra-engine 0.83.1, src/f16_ffi.rs",
 * `qmatvec_gemm_f16_raw`); a failure found inside a running kernel cannot
 * return one, so it is recorded here and read after the fact:
 * Q4K_FAULT_COPY_TIMEOUT if a bounded wait inside a kernel on a bulk copy into
 * shared memory gave up (the kernel then skipped its remaining work and
 * returned; its output is invalid; never happens in normal operation);
 * Q4K_FAULT_TOKEN_RANGE if q4k_embed_gather_f32 met a token outside its table.
 * Synchronises the device. Returns a q4k_status; *flags receives the flags.
 */
Q4K_API int q4k_device_fault_flags(unsigned int *flags);

/*
 * Self-test of the bounded waits: enqueues on `stream` a one-thread kernel
 * that waits on a shared-memory mbarrier phase nothing completes. The wait
 * gives up after its bounded number of tries (each try may sleep up to 1 us;
 * about a second in all), raises Q4K_FAULT_COPY_TIMEOUT and the kernel
 * returns: the same path a kernel takes when a bulk copy is lost, with the
 * CUDA context left usable. Read the flag with q4k_device_fault_flags().
 * Returns a q4k_status.
 */
Q4K_API int q4k_selftest_wait_timeout(q4k_stream_t stream);

/*
 * How q4k_gemv would run a problem on a B200 with `num_sms` SMs (host-only,
 * no CUDA call). Fills *plan and returns Q4K_OK, or the status q4k_gemv would
 * return for these sizes.
 */
typedef struct q4k_gemv_plan {
    int kernel;          /* Q4K_KERNEL_* below                                  */
    int grid;            /* CTAs                                                */
    int block;           /* threads per CTA                                     */
    int smem_bytes;      /* dynamic shared memory per CTA                       */
    int cluster;         /* CTAs per thread-block cluster; > 1 splits rows (split-K) */
    int teams;           /* warp teams per CTA (streaming kernel; else 0)       */
    int depth;           /* bulk-copy ring stages per team (streaming; else 0)  */
    int launches;        /* kernels one call enqueues                           */
    long long units;     /* output rows shared out among the CTAs               */
    long long units_per_cta_max; /* most rows any cluster (CTA if cluster = 1) owns */
    int slices;          /* streaming kernel: 16-byte quant slices per lane (1 or 2) */
} q4k_gemv_plan;

/* As q4k_gemv_plan_for, for q4k_gemv_swiglu (both matrices share one pass;
 * `units` counts output rows, each the pair of a gate and an up row). */
Q4K_API int q4k_gemv_swiglu_plan_for(int m, int n, int k, int num_sms, q4k_gemv_plan *plan);

enum q4k_kernel {
    Q4K_KERNEL_WARP_ROWS = 1,   /* any K: one warp per row, loads via L1; m > 8
                                   runs as ceil(m/8) launches on vector tiles   */
    Q4K_KERNEL_STREAM = 2,      /* K <= 30720 (m = 1) / 15360 (m >= 2); m > 2 runs
                                   as ceil(m/2) launches on vector pairs;
                                   bulk-copy streamed rows, x held in registers,
                                   balanced per-SM ranges; small N splits rows
                                   across the CTAs of a cluster (split-K) and
                                   finishes them through distributed shared
                                   memory                                         */
    Q4K_KERNEL_TC = 3,          /* m >= 3: tcgen05 tensor cores, each superblock
                                   decoded once for up to 16 vectors (groups of
                                   16 beyond), exact integer products of sc*q
                                   and base-128 digits of the scaled x; two
                                   launches per group (digits, GEMV); `units`
                                   counts (128-row tile, superblock column)
                                   items, shared out in equal contiguous ranges;
                                   `depth` is the weight-ring depth             */
    Q4K_KERNEL_I8 = 4           /* m <= 4, the digit image beside four weight
                                   stages (m = 1: K <= 256 * 62), and whole
                                   128-row tiles for every SM (the busiest SM
                                   at most 1/8 above the mean) or >= 5 items
                                   per SM: tcgen05 kind::i8, the quant nibbles
                                   times base-128 (m = 1) or base-256 digits
                                   of the scaled x, exact integer products;
                                   one launch; `slices` is the superblock
                                   columns per item; `units` counts
                                   (128-row tile, superblock column) items, in
                                   whole-tile or equal ranges (cut tiles are
                                   finished from pieces in the stream's
                                   scratch); `depth` is the weight-ring depth  */
};

Q4K_API int q4k_gemv_plan_for(int m, int n, int k, int num_sms, q4k_gemv_plan *plan);

/*
 * ---- Prefill path: fp16 mirror + tensor-core GEMM ----
 * "memra-engine 0.83.1, src/f16_ffi.rs" (module doc): for prefill (m >= 512
 * tokens) the weights are dequantised once into a resident fp16 mirror and
 * each projection is an fp16 GEMM with f32 accumulation; activations are
 * converted f32 -> fp16 first. The page calls cuBLASLt; here the GEMM is a
 * hand-written tcgen05 kernel. Its accuracy contract differs from q4k_gemv's:
 * the operands are rounded to binary16 (relative error up to 2^-11 each), and
 * against the exact products of the fp16 operands the result satisfies, per
 * element, |y - sum_k w16 x16| <= k * 2^-23 * sum_k |w16 x16| + 1e-6.
 */

/*
 * out = the fp16 mirror of W: row-major n x k binary16, out[r*k + t] = the
 * round-to-nearest-even binary16 of weight t of row r's f32 value
 * d*sc*q - dmin*m (that value is itself rounded once), so results are
 * bit-reproducible (`memra_q4_K_dequant_f16`, called from `build_q4k_f16_raw`
 * with (w, dst, out_f, nsb_row, stream)).
 *   w  : as for q4k_gemv (16-byte aligned).
 *   out: n*k*2 bytes, 16-byte aligned, must not overlap w.
 * Values beyond binary16's range become +-inf.
 * Returns a q4k_status.
 */
Q4K_API int q4k_dequant_f16(const void *w, void *out, int n, int k, q4k_stream_t stream);

/*
 * out[i] = binary16 round-to-nearest-even of x[i], i < count (`memra_f16_cvt`:
 * the standalone f32 -> fp16 activation convert, one convert feeding several
 * GEMMs). x and out 16-byte aligned, not overlapping. count == 0 launches
 * nothing. Returns a q4k_status.
 */
Q4K_API int q4k_f32_to_f16(const float *x, void *out, unsigned long long count,
                           q4k_stream_t stream);

/*
 * y = x16 * W16^T (`memra_f16_pp_gemm_pre`: the GEMM on pre-converted fp16
 * activations, "TN": both operands K-major).
 *   w_f16: n x k binary16, row-major (the mirror), 16-byte aligned.
 *   x_f16: m x k binary16, row-major (token-major), 16-byte aligned.
 *   y    : m x n float32, row-major, fully overwritten, must not overlap
 *          either operand.
 *   m, n >= 1; k >= 64 and a multiple of Q4K_GEMM_K_MULTIPLE (64).
 * Accuracy: see the block comment above. Returns a q4k_status.
 */
Q4K_API int q4k_gemm_f16(const void *w_f16, const void *x_f16, float *y, int m, int n, int k,
                         q4k_stream_t stream);

/*
 * y = fp16(x) * W16^T in one call (`memra_f16_pp_gemm`: f32 -> fp16 convert
 * into a caller-provided scratch, then the GEMM, on one stream).
 *   x            : m x k float32, row-major, 16-byte aligned.
 *   x_f16_scratch: m*k*2 bytes of device memory the caller owns, 16-byte
 *                  aligned; overwritten with fp16(x) (the GEMM's B operand);
 *                  must not overlap x, w_f16 or y.
 *   w_f16, y, m, n, k: as for q4k_gemm_f16.
 * Returns a q4k_status.
 */
Q4K_API int q4k_prefill_f16(const void *w_f16, const float *x, void *x_f16_scratch, float *y,
                            int m, int n, int k, q4k_stream_t stream);

/*
 * q4k_prefill_f16 without a caller-provided scratch, for callers that cannot
 * allocate device memory: for instance a plugin running inside a host
 * application that owns all device memory through its own allocator and
 * hands out no allocation hook, or a latency-critical loop where cudaMalloc
 * (which may synchronise the device) is not allowed. The pages have no
 * counterpart to this entry point (their GEMM always takes a scratch buffer).
 *   w_f16, x, y, m, n, k: as for q4k_prefill_f16 (y fully overwritten).
 * The fp16 copy of x goes to a fixed device array inside the library of
 * Q4K_PREFILL_NOALLOC_MAX_ELEMS binary16 values (16 MiB), which every GPU that
 * loads the library holds until the process exits. m*k above that limit is
 * refused with Q4K_ERR_CAPACITY before anything is enqueued.
 * Nothing is allocated or freed by the call: no cudaMalloc, no cudaFree, no
 * allocating library routine. The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture.
 * Every call shares the one array, which keeps the last call's contents: each
 * call overwrites the m*k values its GEMM then reads, so nothing needs to be
 * cleared, but calls that overlap on the GPU (on different streams, or on
 * different host threads without ordering) race on it and must be serialised
 * by the caller.
 * Accuracy and results: identical to q4k_prefill_f16 on the same inputs.
 * Returns a q4k_status.
 */
Q4K_API int q4k_prefill_f16_noalloc(const void *w_f16, const float *x, float *y, int m, int n,
                                    int k, q4k_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* Q4K_H */
