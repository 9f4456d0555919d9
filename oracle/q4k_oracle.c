/*
 * q4k_oracle.c -- CPU oracle for GGUF Q4_K dequantisation and Q4_K GEMV.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg may load or call this code. The product (the
 * CUDA library) never links, loads or calls it, and it shares no code, header,
 * table or constant with the product.
 *
 * It is deliberately plain and slow: one superblock at a time, one weight at a
 * time, in the order the format defines them; dot products in double.
 *
 * What it follows
 * ---------------
 * GEMV  y[i][n] = sum_k W[n][k] * x[i][k]: "realizar 0.8.5,
 *   src/cuda/executor/uses.rs", doc comment of `batched_q4k_gemv_into`
 *   (input M x K row-major, output M x N row-major, weights N x K/256 Q4_K
 *   super-blocks, K a multiple of 256).
 * Superblock = 256 weights in 144 bytes: "memra-engine 0.83.1, src/f16_ffi.rs",
 *   `memra_q4_K_dequant_f16` declaration and the row-bytes check in
 *   `build_q8_f16` (row_bytes == (in_f/256)*144).
 * Field layout, scale/min packing and nibble order: the pages never print them;
 *   the readings taken here (GGUF's published block_q4_K layout) are:
 *     bytes 0-1   d     binary16 little-endian
 *     bytes 2-3   dmin  binary16 little-endian
 *     bytes 4-15  S[12] eight 6-bit scales sc_j and eight 6-bit mins m_j:
 *                   j < 4 : sc_j = S[j] & 63,           m_j = S[j+4] & 63
 *                   j >= 4: sc_j = (S[j+4] & 15) | ((S[j-4] >> 6) << 4)
 *                           m_j  = (S[j+4] >> 4) | ((S[j]   >> 6) << 4)
 *     bytes 16-143 Q[128]: byte Q[32g+l] (g = 0..3, l = 0..31) carries weight
 *                   64g+l in its low nibble and weight 64g+32+l in its high
 *                   nibble; weight t belongs to sub-block j = t/32.
 *   value(t) = d*sc_j*q_t - dmin*m_j   (minus: mins are stored non-negative).
 *
 * Precision
 * ---------
 * Dequantised weights are the f32 expression  fl32(fl32(d*sc)*q - fl32(dmin*m)).
 * d and dmin carry at most 11 significant bits, sc and m at most 6, q at most 4,
 * so d*sc, d*sc*q and dmin*m are exact in f32 and the only rounding is the final
 * subtraction: the value is the correctly rounded f32 of d*sc*q - dmin*m.
 * GEMV terms are (double)w * (double)x, summed in double, in k order.
 * The fp16 mirror (end of file) rounds those f32 values once more, to binary16.
 *
 * Build: gcc -O2 -fPIC -shared -ffp-contract=off -fno-fast-math -pthread
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define QK 256
#define SB_BYTES 144

/* IEEE 754 binary16 -> double, exactly: sign, 5-bit exponent (bias 15),
 * 10-bit fraction; exponent 0 is zero/subnormal (fraction * 2^-24), exponent 31
 * is infinity (fraction 0) or NaN. */
double q4k_oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 31;
    int frac = h & 1023;
    double v;
    if (expo == 0) {
        v = ldexp((double)frac, -24);
    } else if (expo == 31) {
        v = frac ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + frac), expo - 25);
    }
    return sign ? -v : v;
}

static uint16_t u16le(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* Unpack one superblock into its integer fields (readings above). */
void q4k_oracle_unpack(const uint8_t *sb, uint16_t *d_bits, uint16_t *dmin_bits,
                       int32_t sc[8], int32_t mn[8], int32_t q[256])
{
    const uint8_t *S = sb + 4;
    const uint8_t *Q = sb + 16;
    *d_bits = u16le(sb + 0);
    *dmin_bits = u16le(sb + 2);
    for (int j = 0; j < 8; ++j) {
        if (j < 4) {
            sc[j] = S[j] & 63;
            mn[j] = S[j + 4] & 63;
        } else {
            sc[j] = (S[j + 4] & 15) | ((S[j - 4] >> 6) << 4);
            mn[j] = (S[j + 4] >> 4) | ((S[j] >> 6) << 4);
        }
    }
    for (int g = 0; g < 4; ++g) {
        for (int l = 0; l < 32; ++l) {
            q[64 * g + l] = Q[32 * g + l] & 15;
            q[64 * g + 32 + l] = Q[32 * g + l] >> 4;
        }
    }
}

/* The inverse of q4k_oracle_unpack, written from the same readings in the
 * packing direction. Used only to pin the unpacker. Field values are masked to
 * their widths (sc, mn: 6 bits; q: 4 bits). */
void q4k_oracle_pack(uint16_t d_bits, uint16_t dmin_bits, const int32_t sc[8],
                     const int32_t mn[8], const int32_t q[256], uint8_t *out)
{
    uint8_t *S = out + 4;
    uint8_t *Q = out + 16;
    memset(out, 0, SB_BYTES);
    out[0] = (uint8_t)(d_bits & 0xff);
    out[1] = (uint8_t)(d_bits >> 8);
    out[2] = (uint8_t)(dmin_bits & 0xff);
    out[3] = (uint8_t)(dmin_bits >> 8);
    for (int j = 0; j < 4; ++j) {
        S[j] |= (uint8_t)(sc[j] & 63);
        S[j + 4] |= (uint8_t)(mn[j] & 63);
    }
    for (int j = 4; j < 8; ++j) {
        int s = sc[j] & 63, m = mn[j] & 63;
        S[j + 4] |= (uint8_t)((s & 15) | ((m & 15) << 4));   /* low 4 bits of each */
        S[j - 4] |= (uint8_t)((s >> 4) << 6);                /* top 2 bits of sc_j */
        S[j] |= (uint8_t)((m >> 4) << 6);                    /* top 2 bits of m_j  */
    }
    for (int t = 0; t < 256; ++t) {
        int g = t / 64, r = t % 64;
        int byte = 32 * g + (r % 32);
        if (r < 32)
            Q[byte] |= (uint8_t)(q[t] & 15);
        else
            Q[byte] |= (uint8_t)((q[t] & 15) << 4);
    }
}

/* Dequantise one superblock to 256 f32 values. */
static void dequant_block(const uint8_t *sb, float *out)
{
    uint16_t db, mb;
    int32_t sc[8], mn[8], q[256];
    q4k_oracle_unpack(sb, &db, &mb, sc, mn, q);
    float d = (float)q4k_oracle_half_to_double(db);     /* exact: binary16 is a subset of f32 */
    float dmin = (float)q4k_oracle_half_to_double(mb);
    for (int t = 0; t < 256; ++t) {
        int j = t / 32;
        float dsc = d * (float)sc[j];                    /* exact */
        float dm = dmin * (float)mn[j];                  /* exact */
        out[t] = dsc * (float)q[t] - dm;                 /* one rounding */
    }
}

/* out[n][k] (row-major, n rows of k floats) = dequantised W. */
void q4k_oracle_dequant_f32(const uint8_t *w, int64_t n, int64_t k, float *out)
{
    int64_t nsb = k / QK;
    for (int64_t r = 0; r < n; ++r)
        for (int64_t b = 0; b < nsb; ++b)
            dequant_block(w + (r * nsb + b) * SB_BYTES, out + r * k + b * QK);
}

/* Dequantise only the listed rows: out[i][k] = W[rows[i]][k]. */
void q4k_oracle_dequant_rows(const uint8_t *w, int64_t k, const int64_t *rows,
                             int64_t nrows, float *out)
{
    int64_t nsb = k / QK;
    for (int64_t i = 0; i < nrows; ++i)
        for (int64_t b = 0; b < nsb; ++b)
            dequant_block(w + (rows[i] * nsb + b) * SB_BYTES, out + i * k + b * QK);
}

/* One output row r for all m vectors: y[i] = sum_k W[r][k] x[i][k] in double,
 * a[i] = sum_k |W[r][k] x[i][k]|. */
static void gemv_row(const uint8_t *w, const float *x, int32_t m, int64_t k, int64_t r,
                     double *y, double *a, int64_t ystride)
{
    int64_t nsb = k / QK;
    float wv[QK];
    for (int32_t i = 0; i < m; ++i) {
        y[i * ystride] = 0.0;
        a[i * ystride] = 0.0;
    }
    for (int64_t b = 0; b < nsb; ++b) {
        dequant_block(w + (r * nsb + b) * SB_BYTES, wv);
        for (int32_t i = 0; i < m; ++i) {
            const float *xi = x + (int64_t)i * k + b * QK;
            double s = y[i * ystride], sa = a[i * ystride];
            for (int t = 0; t < QK; ++t) {
                double p = (double)wv[t] * (double)xi[t];
                s += p;
                sa += fabs(p);
            }
            y[i * ystride] = s;
            a[i * ystride] = sa;
        }
    }
}

struct gemv_job {
    const uint8_t *w;
    const float *x;
    int32_t m;
    int64_t n, k, r0, r1;
    double *y, *a;
};

static void *gemv_worker(void *arg)
{
    struct gemv_job *j = (struct gemv_job *)arg;
    for (int64_t r = j->r0; r < j->r1; ++r)
        gemv_row(j->w, j->x, j->m, j->k, r, j->y + r, j->a + r, j->n);
    return NULL;
}

/* y[i][r] and a[i][r] for all r < n, i < m (row-major m x n). Rows are split
 * into `nthreads` contiguous ranges run on POSIX threads (1 = no threads).
 * Returns 0, or -1 if a thread could not be started. */
int q4k_oracle_gemv(const uint8_t *w, const float *x, int32_t m, int64_t n, int64_t k,
                    double *y, double *a, int32_t nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > n)
        nthreads = (int32_t)n;
    if (nthreads == 1) {
        struct gemv_job j = {w, x, m, n, k, 0, n, y, a};
        gemv_worker(&j);
        return 0;
    }
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    struct gemv_job *jobs = (struct gemv_job *)calloc((size_t)nthreads, sizeof(struct gemv_job));
    int rc = 0, started = 0;
    for (int32_t t = 0; t < nthreads; ++t) {
        struct gemv_job j = {w, x, m, n, k, n * t / nthreads, n * (t + 1) / nthreads, y, a};
        jobs[t] = j;
        if (pthread_create(&th[t], NULL, gemv_worker, &jobs[t]) != 0) {
            rc = -1;
            break;
        }
        ++started;
    }
    for (int t = 0; t < started; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return rc;
}

/* Only the listed rows: y[i][s] = row rows[s] of vector i (row-major m x nrows). */
void q4k_oracle_gemv_rows(const uint8_t *w, const float *x, int32_t m, int64_t k,
                          const int64_t *rows, int64_t nrows, double *y, double *a)
{
    for (int64_t s = 0; s < nrows; ++s)
        gemv_row(w, x, m, k, rows[s], y + s, a + s, nrows);
}

/*
 * Embedding lookup from a Q4_K table ("turbospark-runtime 0.1.0,
 * src/real_forward_dispatch.rs": `validate_block_quant_embedding` with the
 * Q4_K block constants, called by `validate_q4_k_embedding` before
 * `encode_embed_lookup_q4_k(..., token, hidden, embed_scale)`).
 *
 * Validation, in the page's order; the return value says which rule failed:
 *   Q4K_ORACLE_EMBED_SHAPE     the table is not [rows, hidden] (cols != hidden)
 *   Q4K_ORACLE_EMBED_TOKEN     token >= rows
 *   Q4K_ORACLE_EMBED_WIDTH     hidden == 0 or hidden not a whole number of 256-weight blocks
 *   Q4K_ORACLE_EMBED_OVERFLOW  row size, table size or end of the selected row overflows 64 bits
 *   Q4K_ORACLE_EMBED_SIZE      table_bytes != rows * row_bytes, or the selected row
 *                              does not end inside the table
 * with row_bytes = hidden / 256 * 144.
 *
 * Value (a reading: the page names the call but does not print the kernel):
 * out[j] = fl32(w[j] * embed_scale), where w[j] is the dequantised f32 weight
 * (above) of row `token`; the product of two floats is exact in double, so the
 * double product rounded to float is that single f32 rounding.
 */
enum {
    Q4K_ORACLE_EMBED_OK = 0,
    Q4K_ORACLE_EMBED_SHAPE = 1,
    Q4K_ORACLE_EMBED_TOKEN = 2,
    Q4K_ORACLE_EMBED_WIDTH = 3,
    Q4K_ORACLE_EMBED_OVERFLOW = 4,
    Q4K_ORACLE_EMBED_SIZE = 5,
};

static int mul_overflows(uint64_t a, uint64_t b, uint64_t *out)
{
    if (a != 0 && b > UINT64_MAX / a)
        return 1;
    *out = a * b;
    return 0;
}

int q4k_oracle_embed_validate(uint64_t table_bytes, uint64_t rows, uint64_t cols,
                              uint64_t hidden, uint64_t token)
{
    if (cols != hidden)
        return Q4K_ORACLE_EMBED_SHAPE;
    if (token >= rows)
        return Q4K_ORACLE_EMBED_TOKEN;
    if (hidden == 0 || hidden % QK != 0)
        return Q4K_ORACLE_EMBED_WIDTH;
    uint64_t row_bytes, expected, selected_end;
    if (mul_overflows(hidden / QK, SB_BYTES, &row_bytes))
        return Q4K_ORACLE_EMBED_OVERFLOW;
    if (mul_overflows(rows, row_bytes, &expected))
        return Q4K_ORACLE_EMBED_OVERFLOW;
    if (token == UINT64_MAX || mul_overflows(token + 1, row_bytes, &selected_end))
        return Q4K_ORACLE_EMBED_OVERFLOW;
    if (table_bytes != expected || selected_end > table_bytes)
        return Q4K_ORACLE_EMBED_SIZE;
    return Q4K_ORACLE_EMBED_OK;
}

/* out[0..hidden) = row `token` of the table times embed_scale; returns the
 * validation result and writes nothing unless it is Q4K_ORACLE_EMBED_OK. */
int q4k_oracle_embed_lookup(const uint8_t *table, uint64_t table_bytes, uint64_t rows,
                            uint64_t cols, uint64_t hidden, uint64_t token, float embed_scale,
                            float *out)
{
    int st = q4k_oracle_embed_validate(table_bytes, rows, cols, hidden, token);
    if (st != Q4K_ORACLE_EMBED_OK)
        return st;
    uint64_t nsb = hidden / QK;
    float wv[QK];
    for (uint64_t b = 0; b < nsb; ++b) {
        dequant_block(table + (token * nsb + b) * SB_BYTES, wv);
        for (int t = 0; t < QK; ++t)
            out[b * QK + t] = (float)((double)wv[t] * (double)embed_scale);
    }
    return Q4K_ORACLE_EMBED_OK;
}

/* ------------------------------------------------------------------------
 * fp16 mirror for the prefill GEMM ("memra-engine 0.83.1, src/f16_ffi.rs":
 * module doc -- a resident fp16 dequant mirror of the trunk weights feeds an
 * fp16 GEMM with f32 accumulation; `memra_q4_K_dequant_f16` turns Q4_K
 * superblocks into the row-major fp16 mirror, `memra_f16_cvt` turns f32
 * activations into fp16). Reading taken where the page is silent: a mirror
 * value is the binary16 round-to-nearest-even of the f32 dequantised value
 * above, and an activation is the binary16 RNE of its f32 value.
 * ------------------------------------------------------------------------ */

/* binary32 -> binary16 by the definition of round-to-nearest, ties-to-even:
 * the finite binary16 value nearest to f, and on a tie the one whose last
 * fraction bit is 0; a magnitude of at least 65520 (the largest finite value
 * 65504 plus half of its ulp 32) becomes infinity. NaN becomes the quiet NaN
 * 0x7E00 with f's sign. The nearest values are found by bisection over the
 * positive finite bit patterns 0x0000..0x7BFF, which increase with the value. */
uint16_t q4k_oracle_float_to_half(float f)
{
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    if (isnan(f))
        return (uint16_t)(sign | 0x7E00);
    double v = fabs((double)f);
    if (v >= 65520.0)
        return (uint16_t)(sign | 0x7C00);
    int lo = 0, hi = 0x7BFF;          /* invariant: value(lo) <= v */
    if (q4k_oracle_half_to_double((uint16_t)hi) <= v) {
        lo = hi;
    } else {
        while (hi - lo > 1) {         /* value(lo) <= v < value(hi) */
            int mid = (lo + hi) / 2;
            if (q4k_oracle_half_to_double((uint16_t)mid) <= v)
                lo = mid;
            else
                hi = mid;
        }
    }
    double below = q4k_oracle_half_to_double((uint16_t)lo);
    if (below == v)
        return (uint16_t)(sign | lo);
    double above = (lo == 0x7BFF) ? 65536.0 : q4k_oracle_half_to_double((uint16_t)(lo + 1));
    double dlo = v - below, dhi = above - v;   /* exact: all three are doubles of few bits */
    int pick;
    if (dlo < dhi)
        pick = lo;
    else if (dhi < dlo)
        pick = lo + 1;
    else
        pick = (lo & 1) ? lo + 1 : lo;        /* tie: the even bit pattern */
    return (uint16_t)(sign | pick);
}

/* out[i] = binary16 RNE of x[i] (the f32 -> fp16 activation convert). */
void q4k_oracle_floats_to_half(const float *x, int64_t count, uint16_t *out)
{
    for (int64_t i = 0; i < count; ++i)
        out[i] = q4k_oracle_float_to_half(x[i]);
}

/* out[n][k] (row-major binary16 bit patterns) = the fp16 mirror of W. */
void q4k_oracle_dequant_f16(const uint8_t *w, int64_t n, int64_t k, uint16_t *out)
{
    int64_t nsb = k / QK;
    float v[QK];
    for (int64_t r = 0; r < n; ++r)
        for (int64_t b = 0; b < nsb; ++b) {
            dequant_block(w + (r * nsb + b) * SB_BYTES, v);
            for (int t = 0; t < QK; ++t)
                out[r * k + b * QK + t] = q4k_oracle_float_to_half(v[t]);
        }
}
