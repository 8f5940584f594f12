/*
 * Plain FP64 CPU oracle for MLA decoding over a paged latent KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the test-suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * path.
 *
 * What it computes is the plain definition of the operation, written out with
 * no blocking, fusion or reordering:
 *
 *   For each request b, query token s < s_q and query head h < h_q
 *   (kv head g = h / (h_q / h_kv)):
 *     n      = causal ? clamp(L_b - s_q + 1 + s, 0, L_b) : L_b
 *     k_j    = kvcache[block_table[b][j / page]][j % page][g][0 : d_qk]   (j < n)
 *     v_j    = k_j[0 : dv]        (V is the leading dv columns of the same row)
 *     x_j    = scale * <q[b,s,h,:], k_j>
 *     LSE    = log sum_j exp(x_j)         (natural log, computed as M + log sum exp(x_j - M))
 *     O      = sum_j exp(x_j - LSE) v_j
 *   and for n == 0: O = 0, LSE = -inf.
 *
 * Sources (page title, section):
 *   - "FlashMLA" usage page (deepep.org): get_mla_metadata / flash_mla_with_kvcache
 *     call, its arguments q, kvcache, block_table, cache_seqlens, dv, causal; the
 *     kernel's three stages Q-K product, softmax with scaling, output.
 *   - Upstream FlashMLA documentation, "Usage / MLA Decoding": return values
 *     (out, lse), lse = log-sum-exp of the attention scores per query head;
 *     "MLA Mode" footnote: MQA mode is head_dim_k = 576 with head_dim_v = 512.
 *   - Upstream FlashMLA documentation, FP8 KV cache format: a token row is the
 *     512-wide NoPE (latent) part followed by the 64-wide RoPE part, so V is the
 *     leading 512 columns of the row.
 *   - Upstream FlashMLA documentation, "FP8 KV Cache": the "FP8 with scale" row of
 *     656 bytes (512 float8_e4m3 latent values, 4 float32 scales, one per 128
 *     values, 64 bfloat16 RoPE values), dequantized to bfloat16 before the
 *     attention, which then runs as for a bfloat16 cache.
 *   - Upstream FlashMLA documentation, "Sparse Attention (indices tensor)": the
 *     token-level sparse decode over a flat row list per query token.
 *   - Upstream FlashMLA documentation, "Sparse MLA Prefill / Equivalent PyTorch
 *     code": the softmax written out (max, log-sum-exp, weights exp(P - lse)).
 * Readings where the pages are silent (each is listed in the design notes):
 *   LSE is the natural log of the scaled logits; causal alignment is bottom-right
 *   (the last query token sees all L_b tokens); scale is an argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* 16-bit float decoding, written from the IEEE-754 / bfloat16 layouts. */
/* ------------------------------------------------------------------ */

/* bfloat16: the upper 16 bits of an IEEE-754 binary32. */
static double oracle_bf16_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE-754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double oracle_fp16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
    } else if (e == 31) {
        v = (m == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(m | 0x400), e - 25); /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

double mla_oracle_half_to_double(uint16_t h, int dtype)
{
    return dtype == 0 ? oracle_bf16_to_double(h) : oracle_fp16_to_double(h);
}

/* ------------------------------------------------------------------ */
/* "FP8 with scale" KV cache rows.                                      */
/* ------------------------------------------------------------------ */

/*
 * One 8-bit float in the E4M3 encoding (the "float8_e4m3" of the FP8 cache
 * format; the OCP 8-bit floating-point E4M3 layout, which has no infinities):
 * 1 sign bit, 4 exponent bits with bias 7, 3 fraction bits.  Exponent field 0
 * holds the subnormals (m/8) * 2^-6; S.1111.111 is the only NaN, so the largest
 * finite magnitude is 1.75 * 2^8 = 448.
 */
double mla_oracle_e4m3_to_double(uint8_t x)
{
    int sign = x >> 7;
    int e = (x >> 3) & 0xf;
    int m = x & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);           /* (m / 8) * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m / 8) * 2^(e - 7) */
    return sign ? -v : v;
}

/* Round a binary32 value to bfloat16 (its upper 16 bits), to nearest with ties to even. */
static uint16_t oracle_float_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u); /* NaN stays NaN */
    uint32_t hi = u >> 16, rest = u & 0xffffu;
    if (rest > 0x8000u || (rest == 0x8000u && (hi & 1u))) hi += 1; /* a carry into the exponent is right */
    return (uint16_t)hi;
}

/*
 * Dequantize n token rows of the "FP8 with scale" KV cache (upstream FlashMLA
 * documentation reproduced on the "FlashMLA vLLM Optimization" page, section
 * "FP8 KV Cache"): a row is 656 bytes, the 512 float8_e4m3 latent ("NoPE")
 * values, then 4 float32 scales (scale k belongs to latent values
 * [128k, 128k + 128)), then the 64 bfloat16 RoPE values, which are not
 * quantized.  The kernel "dequantizes the cache to bfloat16": latent value i
 * becomes bf16(e4m3_i * scale_{i/128}), the product taken in binary32 (the
 * scales' type: the exact product, rounded once to binary32) and then rounded
 * to bfloat16; the RoPE values are kept as they are.  Output: n rows of 576
 * bfloat16 bit patterns, latent first, the layout of the 16-bit cache.
 * Multi-byte fields are little-endian.
 */
void mla_oracle_dequant_fp8_rows(const uint8_t* rows, long n, uint16_t* out)
{
    for (long t = 0; t < n; ++t) {
        const uint8_t* row = rows + (size_t)t * 656;
        uint16_t* o = out + (size_t)t * 576;
        float scale[4];
        memcpy(scale, row + 512, sizeof scale);
        for (int i = 0; i < 512; ++i) {
            double exact = mla_oracle_e4m3_to_double(row[i]) * (double)scale[i / 128]; /* exact in fp64 */
            o[i] = oracle_float_to_bf16((float)exact);
        }
        for (int i = 0; i < 64; ++i) memcpy(o + 512 + i, row + 528 + 2 * i, 2);
    }
}

int mla_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Shape of one problem; plain struct so the ctypes side can fill it. */
typedef struct {
    int batch, s_q, h_q, h_kv, d_qk, dv;
    int page_size, max_blocks_per_seq, num_blocks;
    int dtype;   /* 0 = bfloat16, 1 = float16 */
    int causal;  /* bottom-right aligned */
    double scale;
} mla_oracle_shape;

/* Number of cached tokens visible to query token s of request b. */
static long oracle_visible(const mla_oracle_shape* sh, long L, int s)
{
    if (!sh->causal) return L;
    long n = L - sh->s_q + 1 + s;
    if (n < 0) n = 0;
    if (n > L) n = L;
    return n;
}

/*
 * Attention of one (b, s, h) over the visible tokens j with lo <= j < hi.
 * Writes dv outputs and returns the LSE of that token range; an empty range
 * gives O = 0 and LSE = -inf.  With lo = 0, hi = L_b this is the full result;
 * other ranges give the partial results that the split / combine invariant
 * uses.
 */
static double oracle_one_row(const mla_oracle_shape* sh, const uint16_t* q,
                             const uint16_t* kv, const int32_t* block_table,
                             long L, int b, int s, int h, long lo, long hi,
                             double* x /* scratch, >= hi-lo */, double* qrow,
                             double* o_row)
{
    const int d_qk = sh->d_qk, dv = sh->dv, P = sh->page_size;
    const int g = h / (sh->h_q / sh->h_kv);
    long n = oracle_visible(sh, L, s);
    if (hi > n) hi = n;
    if (lo < 0) lo = 0;
    for (int d = 0; d < dv; ++d) o_row[d] = 0.0;
    if (hi <= lo) return -INFINITY;

    const uint16_t* qp = q + (((size_t)b * sh->s_q + s) * sh->h_q + h) * (size_t)d_qk;
    for (int d = 0; d < d_qk; ++d) qrow[d] = mla_oracle_half_to_double(qp[d], sh->dtype);

    /* x_j = scale * <q, k_j>, k_j gathered through the block table. */
    double M = -INFINITY;
    for (long j = lo; j < hi; ++j) {
        long page = block_table[(size_t)b * sh->max_blocks_per_seq + j / P];
        const uint16_t* kp = kv + (((size_t)page * P + (j % P)) * sh->h_kv + g) * (size_t)d_qk;
        double acc = 0.0;
        for (int d = 0; d < d_qk; ++d) acc += qrow[d] * mla_oracle_half_to_double(kp[d], sh->dtype);
        x[j - lo] = sh->scale * acc;
        if (x[j - lo] > M) M = x[j - lo];
    }
    /* LSE = M + log sum exp(x_j - M) */
    double sum = 0.0;
    for (long j = lo; j < hi; ++j) sum += exp(x[j - lo] - M);
    double lse = M + log(sum);
    /* O = sum_j exp(x_j - LSE) v_j, v_j = k_j[0:dv] */
    for (long j = lo; j < hi; ++j) {
        long page = block_table[(size_t)b * sh->max_blocks_per_seq + j / P];
        const uint16_t* vp = kv + (((size_t)page * P + (j % P)) * sh->h_kv + g) * (size_t)d_qk;
        double w = exp(x[j - lo] - lse);
        for (int d = 0; d < dv; ++d) o_row[d] += w * mla_oracle_half_to_double(vp[d], sh->dtype);
    }
    return lse;
}

static long oracle_max_len(const mla_oracle_shape* sh, const int32_t* seqlens)
{
    long mx = 1;
    for (int b = 0; b < sh->batch; ++b)
        if (seqlens[b] > mx) mx = seqlens[b];
    return mx;
}

/*
 * Partial attention over the token range [lo, hi) of every request (the same
 * range for all requests; hi is clipped to each row's visible length).
 * o: [batch, s_q, h_q, dv] f64, lse: [batch, s_q, h_q] f64.
 * Returns 0 on success, -1 on bad arguments.
 */
int mla_oracle_decode_range(const mla_oracle_shape* sh, const uint16_t* q, const uint16_t* kv,
                            const int32_t* block_table, const int32_t* seqlens, long lo,
                            long hi, double* o, double* lse)
{
    if (sh->batch < 0 || sh->s_q <= 0 || sh->h_q <= 0 || sh->h_kv <= 0 ||
        sh->h_q % sh->h_kv != 0 || sh->dv > sh->d_qk || sh->page_size <= 0)
        return -1;
    const long maxlen = oracle_max_len(sh, seqlens);
    const long rows = (long)sh->batch * sh->s_q * sh->h_q;
    int err = 0;
#pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)maxlen);
        double* qrow = (double*)malloc(sizeof(double) * (size_t)sh->d_qk);
        if (!x || !qrow) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long r = 0; r < rows; ++r) {
                int h = (int)(r % sh->h_q);
                int s = (int)((r / sh->h_q) % sh->s_q);
                int b = (int)(r / ((long)sh->h_q * sh->s_q));
                long L = seqlens[b];
                long h_end = hi < 0 ? L : hi;
                lse[r] = oracle_one_row(sh, q, kv, block_table, L, b, s, h, lo, h_end, x, qrow,
                                        o + (size_t)r * sh->dv);
            }
        }
        free(x);
        free(qrow);
    }
    return err ? -1 : 0;
}

/* Full attention: the range [0, L_b) of each request. */
int mla_oracle_decode(const mla_oracle_shape* sh, const uint16_t* q, const uint16_t* kv,
                      const int32_t* block_table, const int32_t* seqlens, double* o,
                      double* lse)
{
    return mla_oracle_decode_range(sh, q, kv, block_table, seqlens, 0, -1, o, lse);
}

/*
 * Same as mla_oracle_decode but only for the listed flat rows r = (b*s_q+s)*h_q+h;
 * used to check sampled outputs of large problems.  o: [n_rows, dv], lse: [n_rows].
 */
int mla_oracle_decode_rows(const mla_oracle_shape* sh, const uint16_t* q, const uint16_t* kv,
                           const int32_t* block_table, const int32_t* seqlens,
                           const int64_t* row_ids, long n_rows, double* o, double* lse)
{
    const long maxlen = oracle_max_len(sh, seqlens);
    const long rows = (long)sh->batch * sh->s_q * sh->h_q;
    int err = 0;
#pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)maxlen);
        double* qrow = (double*)malloc(sizeof(double) * (size_t)sh->d_qk);
        if (!x || !qrow) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long i = 0; i < n_rows; ++i) {
                long r = row_ids[i];
                if (r < 0 || r >= rows) {
#pragma omp atomic write
                    err = 1;
                    continue;
                }
                int h = (int)(r % sh->h_q);
                int s = (int)((r / sh->h_q) % sh->s_q);
                int b = (int)(r / ((long)sh->h_q * sh->s_q));
                long L = seqlens[b];
                lse[i] = oracle_one_row(sh, q, kv, block_table, L, b, s, h, 0, L, x, qrow,
                                        o + (size_t)i * sh->dv);
            }
        }
        free(x);
        free(qrow);
    }
    return err ? -1 : 0;
}

/*
 * Token-level sparse decoding (upstream FlashMLA documentation, "Sparse Attention
 * (indices tensor)" under "Usage / MLA Decoding"): request b's query token s attends
 * the cache rows listed in indices[b][s][0 : topk]; an entry is the flat row index
 * page * page_size + offset, so no block table is used.  Entries of -1 are invalid;
 * read here: every entry outside [0, num_blocks * page_size) is invalid (the sparse
 * prefill section on the same page allows -1 or any index past the end) and
 * contributes nothing.  Each valid entry contributes one term, so a row listed twice
 * counts twice: the entries are gathered, as the sparse prefill's equivalent code
 * gathers kv[indices].  There is no causal mask: the list is what the query sees.
 *   x_k = scale * <q[b,s,h,:], k_{row_k}>  (valid k),   LSE = log sum_k exp(x_k),
 *   O   = sum_k exp(x_k - LSE) v_{row_k},  v = the leading dv columns of the row;
 * with no valid entry, O = 0 and LSE = -inf.
 * indices: [batch, s_q, topk] int32; o: [batch, s_q, h_q, dv] f64; lse: [batch, s_q, h_q] f64.
 * Returns 0 on success, -1 on bad arguments.
 */
int mla_oracle_decode_sparse(const mla_oracle_shape* sh, const uint16_t* q, const uint16_t* kv,
                             const int32_t* indices, int topk, double* o, double* lse)
{
    if (!sh || sh->batch < 0 || sh->s_q <= 0 || sh->h_q <= 0 || sh->h_kv <= 0 || sh->h_q % sh->h_kv ||
        sh->dv > sh->d_qk || topk < 0 || sh->page_size <= 0 || sh->num_blocks < 0)
        return -1;
    const int d_qk = sh->d_qk, dv = sh->dv;
    const long n_rows = (long)sh->num_blocks * sh->page_size;
    const long rows = (long)sh->batch * sh->s_q * sh->h_q;
    int err = 0;
#pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)(topk > 0 ? topk : 1));
        double* qrow = (double*)malloc(sizeof(double) * (size_t)d_qk);
        if (!x || !qrow) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (long r = 0; r < rows; ++r) {
                const int h = (int)(r % sh->h_q);
                const long bs = r / sh->h_q; /* b * s_q + s */
                const int g = h / (sh->h_q / sh->h_kv);
                const int32_t* ix = indices + (size_t)bs * topk;
                double* o_row = o + (size_t)r * dv;
                for (int d = 0; d < dv; ++d) o_row[d] = 0.0;
                const uint16_t* qp = q + (size_t)r * d_qk;
                for (int d = 0; d < d_qk; ++d) qrow[d] = mla_oracle_half_to_double(qp[d], sh->dtype);
                double M = -INFINITY;
                int any = 0;
                for (int k = 0; k < topk; ++k) {
                    const long row = ix[k];
                    if (row < 0 || row >= n_rows) continue; /* invalid entry */
                    const uint16_t* kp = kv + ((size_t)row * sh->h_kv + g) * (size_t)d_qk;
                    double acc = 0.0;
                    for (int d = 0; d < d_qk; ++d) acc += qrow[d] * mla_oracle_half_to_double(kp[d], sh->dtype);
                    x[k] = sh->scale * acc;
                    if (!any || x[k] > M) M = x[k];
                    any = 1;
                }
                if (!any) {
                    lse[r] = -INFINITY;
                    continue;
                }
                double sum = 0.0;
                for (int k = 0; k < topk; ++k)
                    if (ix[k] >= 0 && ix[k] < n_rows) sum += exp(x[k] - M);
                const double L = M + log(sum);
                lse[r] = L;
                for (int k = 0; k < topk; ++k) {
                    const long row = ix[k];
                    if (row < 0 || row >= n_rows) continue;
                    const uint16_t* vp = kv + ((size_t)row * sh->h_kv + g) * (size_t)d_qk;
                    const double w = exp(x[k] - L);
                    for (int d = 0; d < dv; ++d) o_row[d] += w * mla_oracle_half_to_double(vp[d], sh->dtype);
                }
            }
        }
        free(x);
        free(qrow);
    }
    return err ? -1 : 0;
}

/*
 * Sparse MLA prefill (upstream FlashMLA documentation, "Sparse MLA Prefill / Return Values
 * and Equivalent PyTorch Code"), step by step in the documentation's order and base-2 notation.
 * q [s_q, h_q, d_qk], kv [s_kv, h_kv, d_qk] (16-bit bit patterns), indices [s_q, h_kv, topk].
 * For query i, head h (kv head g = h / (h_q / h_kv)), over the valid entries k (0 <= idx < s_kv;
 * -1 or any index >= s_kv is invalid):
 *   focused_k  = kv[idx_k, g, :]
 *   P_k        = <q[i,h,:], focused_k> * sm_scale * log2(e)
 *   max_logits = max_k P_k
 *   lse        = log2(sum_k 2^{P_k})          (computed as max_logits + log2 sum_k 2^{P_k - max_logits})
 *   S_k        = 2^{P_k - lse}
 *   out        = sum_k S_k * focused_k[0 : dv]  (V is the leading dv columns of the row)
 * With no valid entry: out = 0, max_logits = lse = -inf.
 * out [s_q, h_q, dv], max_logits / lse [s_q, h_q].  Returns 0, or -1 for bad arguments.
 */
int mla_oracle_sparse_prefill(int s_q, int h_q, int h_kv, int d_qk, int dv, long s_kv, int topk, int dtype,
                              double sm_scale, const uint16_t* q, const uint16_t* kv, const int32_t* indices,
                              double* out, double* max_logits, double* lse)
{
    if (s_q < 0 || h_q <= 0 || h_kv <= 0 || h_q % h_kv || d_qk <= 0 || dv <= 0 || dv > d_qk || s_kv < 0 ||
        topk < 0)
        return -1;
    const double log2e = 1.4426950408889634073599246810019;
    const long rows = (long)s_q * h_q;
    int err = 0;
#pragma omp parallel
    {
        double* P = (double*)malloc(sizeof(double) * (size_t)(topk > 0 ? topk : 1));
        double* qrow = (double*)malloc(sizeof(double) * (size_t)d_qk);
        if (!P || !qrow) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (long r = 0; r < rows; ++r) {
                const long i = r / h_q;
                const int h = (int)(r % h_q);
                const int g = h / (h_q / h_kv);
                const int32_t* ix = indices + ((size_t)i * h_kv + g) * topk;
                double* o_row = out + (size_t)r * dv;
                for (int d = 0; d < dv; ++d) o_row[d] = 0.0;
                const uint16_t* qp = q + (size_t)r * d_qk;
                for (int d = 0; d < d_qk; ++d) qrow[d] = mla_oracle_half_to_double(qp[d], dtype);
                /* P = (Q @ focused_kv^T) * sm_scale * log2(e); max_logits = P.max() */
                double mx = -INFINITY;
                for (int k = 0; k < topk; ++k) {
                    const long row = ix[k];
                    if (row < 0 || row >= s_kv) continue;
                    const uint16_t* kp = kv + ((size_t)row * h_kv + g) * (size_t)d_qk;
                    double acc = 0.0;
                    for (int d = 0; d < d_qk; ++d) acc += qrow[d] * mla_oracle_half_to_double(kp[d], dtype);
                    P[k] = acc * sm_scale * log2e;
                    if (P[k] > mx) mx = P[k];
                }
                max_logits[r] = mx;
                if (mx == -INFINITY) { /* no valid entry */
                    lse[r] = -INFINITY;
                    continue;
                }
                /* lse = log2 sum 2^P */
                double sum = 0.0;
                for (int k = 0; k < topk; ++k)
                    if (ix[k] >= 0 && ix[k] < s_kv) sum += exp2(P[k] - mx);
                const double l2 = mx + log2(sum);
                lse[r] = l2;
                /* S = 2^(P - lse); out = S @ focused_kv[:, :dv] */
                for (int k = 0; k < topk; ++k) {
                    const long row = ix[k];
                    if (row < 0 || row >= s_kv) continue;
                    const uint16_t* vp = kv + ((size_t)row * h_kv + g) * (size_t)d_qk;
                    const double w = exp2(P[k] - l2);
                    for (int d = 0; d < dv; ++d) o_row[d] += w * mla_oracle_half_to_double(vp[d], dtype);
                }
            }
        }
        free(P);
        free(qrow);
    }
    return err ? -1 : 0;
}

/*
 * Merge of n_parts partial results of the same rows, each the attention over a
 * disjoint token range:  LSE = log sum_k exp(lse_k),  O = sum_k exp(lse_k - LSE) O_k.
 * Parts with lse_k = -inf carry no tokens and get weight 0; if every part is
 * empty the result is O = 0, LSE = -inf.  This is the exact identity that makes
 * splitting the KV range and combining afterwards equal to the unsplit result
 * (the split-KV and combine kernels named on the "FlashMLA vLLM Optimization"
 * page, background section).
 * o_parts: [n_parts, rows, dv], lse_parts: [n_parts, rows]; o: [rows, dv], lse: [rows].
 */
void mla_oracle_combine(int n_parts, long rows, int dv, const double* o_parts,
                        const double* lse_parts, double* o, double* lse)
{
    for (long r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int k = 0; k < n_parts; ++k)
            if (lse_parts[(size_t)k * rows + r] > M) M = lse_parts[(size_t)k * rows + r];
        for (int d = 0; d < dv; ++d) o[(size_t)r * dv + d] = 0.0;
        if (M == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int k = 0; k < n_parts; ++k) sum += exp(lse_parts[(size_t)k * rows + r] - M);
        double L = M + log(sum);
        lse[r] = L;
        for (int k = 0; k < n_parts; ++k) {
            double w = exp(lse_parts[(size_t)k * rows + r] - L);
            if (w == 0.0) continue;
            const double* op = o_parts + ((size_t)k * rows + r) * dv;
            for (int d = 0; d < dv; ++d) o[(size_t)r * dv + d] += w * op[d];
        }
    }
}
