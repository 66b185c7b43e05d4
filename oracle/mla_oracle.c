/*
 * Oracle for paged MLA decode -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of what the decode path computes.  It is used by the
 * tests, by the package's smoke check and by the benchmark's CPU-baseline leg; the
 * product path never calls it.  It shares no code with the CUDA library.
 *
 * Definition (FlashMLA-style decode over a latent KV cache):
 *   - "DeepSeek FlashMLA ... practitioner notes" (dpshk.com), section 2.1: with key
 *     k_t = W^UK c_t the score is q_t . k_t = (W^UK^T q_t) . c_t, i.e. the absorbed query
 *     dots the cached latent row c directly; the key IS the latent row.
 *   - Same page, section 2.2: online softmax gives exactly the standard softmax; here we use
 *     the plain two-pass softmax (max, then normalised exponentials).
 *   - "OpenSourceWeek Day 1 - FlashMLA", section II.1/II.2: fixed 64-token cache blocks
 *     found through a block table; q folded as [b, s_q, h_kv, g, d] (heads grouped
 *     consecutively per latent head); section V.2: the call carries block_table,
 *     cache_seqlens, dv and causal=True.
 *   - The value of token j is the first dv columns of the same latent row.
 *
 * For each listed (b, s, h):
 *   g   = h_q / h_kv;  kvh = h / g
 *   n   = causal ? L_b - (s_q - 1 - s) : L_b, clamped at 0        (bottom-right causal)
 *   keys j in [lo, hi) with lo = kv_begin[b] (0 if NULL), hi = min(n, kv_end[b] or n)
 *   c_j = k_cache[block_table[b][j / page], j % page, kvh, :]
 *   x_j = scale * sum_t q[b,s,h,t] * c_j[t]                     (t over all d columns)
 *   M = max_j x_j;  Z = sum_j exp(x_j - M)
 *   out = sum_j exp(x_j - M) / Z * c_j[0:dv];  lse = M + ln Z      (natural log)
 *   no keys: out = 0, lse = -inf
 *
 * bf16 inputs are decoded exactly to double.  Build: gcc -O2 -fopenmp -shared -fPIC.
 *
 * FP8 latent cache (oracle_mla_decode_rows_fp8).  The Baidu page on Flash MLA ("Flash MLA：
 * 面向可变长度序列的高效MLA解码内核库解析", section 三.2 and the flow of section 四, step 3)
 * names FP8 storage of the cache as the precision lever but gives no format.  Reading taken
 * here: every token's latent row is stored as 576 OCP E4M3 ("e4m3fn") codes with one fp32
 * scale per token and latent head, and the row the decode uses is the dequantised
 *   c_j[t] = scale_j * e4m3(code_j[t]);
 * the decode itself is the definition above applied to these rows.  k8 is [num_pages, page,
 * h_kv, d] uint8, k_scale is [h_kv, num_pages, page] fp32.
 *
 * Token-level sparse decode (oracle_mla_decode_rows_sparse).  The same Baidu page, section
 * 三.3 (the token-level sparse attention kernel), keeps only the Top-K key connections of a
 * query and stores the sparse attention pattern in CSR form; the scoring that picks them is
 * outside the decode.  Reading taken here: query token (b, s) comes with a list of key
 * positions col_idx[row_ptr[b * s_q + s] .. row_ptr[b * s_q + s + 1]) in CSR form, shared by
 * all h_q heads of that token (the cache has one latent row per token and latent head).  The
 * decode is the definition above with the keys j in [lo, hi) replaced by the list entries
 * whose position lies in [0, n) (n as above, so the causal rule still holds); other entries
 * (padding such as -1, or positions the row may not see) are pruned.  Entries are taken as
 * listed: a position listed twice counts twice.  kv_begin / kv_end, when given, select list
 * entries by their index in the list (a split of the list).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point E4M3 ("e4m3fn"): sign bit 7, exponent bits 6..3 (bias 7),
 * mantissa bits 2..0; exponent 0 holds subnormals (m / 8) * 2^-6; exponent 15 with
 * mantissa 7 is NaN; there is no infinity (the largest finite value is 448). */
static double e4m3_to_double(uint8_t v) {
    const int sgn = v >> 7, e = (v >> 3) & 15, m = v & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m / 8.0, -6);
    else mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sgn ? -mag : mag;
}

int oracle_e4m3_to_double(const uint8_t *codes, int64_t n, double *out) {
    if (!codes || !out || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_to_double(codes[i]);
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* The latent row of (page phys, slot, latent head kvh) as doubles: bf16 codes, or E4M3 codes
 * times the token's scale. */
typedef struct {
    const uint16_t *bf16;  /* [num_pages, page, h_kv, d] or NULL */
    const uint8_t *e4m3;   /* [num_pages, page, h_kv, d] or NULL */
    const float *scale;    /* [h_kv, num_pages, page] with e4m3 */
    int64_t num_pages;
    int page, h_kv, d;
} cache_t;

/* q_row . c over all d columns of the latent row of (page phys, slot, latent head kvh). */
static double row_dot(const cache_t *c, int64_t phys, int slot, int kvh, const uint16_t *q_row) {
    const int64_t row = ((phys * c->page + slot) * c->h_kv + kvh) * (int64_t)c->d;
    double acc = 0.0;
    if (c->bf16) {
        for (int t = 0; t < c->d; ++t) acc += bf16_bits_to_double(q_row[t]) * bf16_bits_to_double(c->bf16[row + t]);
    } else {
        const double sc = (double)c->scale[((int64_t)kvh * c->num_pages + phys) * c->page + slot];
        for (int t = 0; t < c->d; ++t) acc += bf16_bits_to_double(q_row[t]) * (sc * e4m3_to_double(c->e4m3[row + t]));
    }
    return acc;
}

/* o[0:dv] += p * c[0:dv] for the same latent row. */
static void row_axpy(const cache_t *c, int64_t phys, int slot, int kvh, double p, double *o, int dv) {
    const int64_t row = ((phys * c->page + slot) * c->h_kv + kvh) * (int64_t)c->d;
    if (c->bf16) {
        for (int t = 0; t < dv; ++t) o[t] += p * bf16_bits_to_double(c->bf16[row + t]);
    } else {
        const double sc = (double)c->scale[((int64_t)kvh * c->num_pages + phys) * c->page + slot];
        for (int t = 0; t < dv; ++t) o[t] += p * (sc * e4m3_to_double(c->e4m3[row + t]));
    }
}

static int decode_rows(const uint16_t *q, int64_t qs_b, int64_t qs_s, int64_t qs_h,
                       int batch, int s_q, int h_q, int d, const cache_t *cache,
                       const int32_t *block_table, int64_t bt_stride,
                       const int32_t *cache_seqlens,
                       const int32_t *kv_begin, const int32_t *kv_end,
                       const int32_t *row_ptr, const int32_t *col_idx,
                       int dv, double scale, int causal,
                       const int32_t *rows, int64_t n_rows,
                       double *out_rows, double *lse_rows) {
    const int64_t num_pages = cache->num_pages;
    const int page = cache->page, h_kv = cache->h_kv;
    if (!q || !block_table || !cache_seqlens || !rows || !out_rows || !lse_rows) return -1;
    if (cache->d != d || h_kv <= 0 || h_q % h_kv != 0 || dv > d || page <= 0 || batch <= 0 || s_q <= 0)
        return -1;
    const int g = h_q / h_kv;
    int status = 0;

#pragma omp parallel
    {
        int64_t cap = 0;
        double *x = NULL;
        int64_t *pos = NULL;
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            const int b = rows[3 * r + 0], s = rows[3 * r + 1], h = rows[3 * r + 2];
            double *o = out_rows + r * dv;
            if (b < 0 || b >= batch || s < 0 || s >= s_q || h < 0 || h >= h_q) {
#pragma omp atomic write
                status = -1;
                continue;
            }
            const int kvh = h / g;
            const int64_t L = cache_seqlens[b];
            int64_t n = causal ? L - (s_q - 1 - s) : L;
            if (n < 0) n = 0;
            /* the candidate keys: positions [0, n), or the token's list entries */
            const int64_t e0 = row_ptr ? row_ptr[(int64_t)b * s_q + s] : 0;
            const int64_t cnt = row_ptr ? row_ptr[(int64_t)b * s_q + s + 1] - e0 : n;
            int64_t lo = kv_begin ? kv_begin[b] : 0;
            int64_t hi = kv_end ? kv_end[b] : cnt;
            if (hi > cnt) hi = cnt;
            if (lo < 0) lo = 0;
            for (int t = 0; t < dv; ++t) o[t] = 0.0;
            if (hi - lo > cap) {
                free(x);
                free(pos);
                cap = hi - lo;
                x = (double *)malloc((size_t)cap * sizeof(double));
                pos = (int64_t *)malloc((size_t)cap * sizeof(int64_t));
                if (!x || !pos) {
#pragma omp atomic write
                    status = -2;
                    cap = 0;
                    continue;
                }
            }
            /* the key positions this row attends to */
            int64_t nk = 0;
            for (int64_t e = lo; e < hi; ++e) {
                const int64_t j = row_ptr ? col_idx[e0 + e] : e;
                if (j >= 0 && j < n) pos[nk++] = j;
            }
            if (nk == 0) {
                lse_rows[r] = -INFINITY;
                continue;
            }
            const uint16_t *qrow = q + b * qs_b + s * qs_s + h * qs_h;
            /* pass 1: scores and their maximum */
            double M = -INFINITY;
            int bad = 0;
            for (int64_t k = 0; k < nk; ++k) {
                const int64_t j = pos[k];
                const int64_t phys = block_table[b * bt_stride + j / page];
                if (phys < 0 || phys >= num_pages) { bad = 1; break; }
                x[k] = scale * row_dot(cache, phys, (int)(j % page), kvh, qrow);
                if (x[k] > M) M = x[k];
            }
            if (bad) {
#pragma omp atomic write
                status = -3;
                lse_rows[r] = NAN;
                continue;
            }
            /* pass 2: normaliser and weighted sum of the first dv columns */
            double Z = 0.0;
            for (int64_t k = 0; k < nk; ++k) Z += exp(x[k] - M);
            for (int64_t k = 0; k < nk; ++k) {
                const int64_t j = pos[k];
                const int64_t phys = block_table[b * bt_stride + j / page];
                row_axpy(cache, phys, (int)(j % page), kvh, exp(x[k] - M) / Z, o, dv);
            }
            lse_rows[r] = M + log(Z);
        }
        free(x);
        free(pos);
    }
    return status;
}

/*
 * rows: n_rows triples (b, s, h).  out_rows: [n_rows, dv] doubles, lse_rows: [n_rows].
 * q strides are in elements (innermost stride 1).  k_cache is [num_pages, page, h_kv, d]
 * contiguous.  block_table row stride is bt_stride elements.
 * Returns 0, or -1 on an argument error, -2 on allocation failure, -3 when a block-table
 * entry addressed by a key is out of range.
 */
int oracle_mla_decode_rows(const uint16_t *q, int64_t qs_b, int64_t qs_s, int64_t qs_h,
                           int batch, int s_q, int h_q, int d,
                           const uint16_t *k_cache, int64_t num_pages, int page, int h_kv,
                           const int32_t *block_table, int64_t bt_stride,
                           const int32_t *cache_seqlens,
                           const int32_t *kv_begin, const int32_t *kv_end,
                           int dv, double scale, int causal,
                           const int32_t *rows, int64_t n_rows,
                           double *out_rows, double *lse_rows) {
    if (!k_cache) return -1;
    cache_t c = {k_cache, NULL, NULL, num_pages, page, h_kv, d};
    return decode_rows(q, qs_b, qs_s, qs_h, batch, s_q, h_q, d, &c, block_table, bt_stride, cache_seqlens,
                       kv_begin, kv_end, NULL, NULL, dv, scale, causal, rows, n_rows, out_rows, lse_rows);
}

/* The same decode over an FP8 (E4M3 + per-token fp32 scale) latent cache. */
int oracle_mla_decode_rows_fp8(const uint16_t *q, int64_t qs_b, int64_t qs_s, int64_t qs_h,
                               int batch, int s_q, int h_q, int d,
                               const uint8_t *k8, const float *k_scale, int64_t num_pages, int page, int h_kv,
                               const int32_t *block_table, int64_t bt_stride,
                               const int32_t *cache_seqlens,
                               const int32_t *kv_begin, const int32_t *kv_end,
                               int dv, double scale, int causal,
                               const int32_t *rows, int64_t n_rows,
                               double *out_rows, double *lse_rows) {
    if (!k8 || !k_scale) return -1;
    cache_t c = {NULL, k8, k_scale, num_pages, page, h_kv, d};
    return decode_rows(q, qs_b, qs_s, qs_h, batch, s_q, h_q, d, &c, block_table, bt_stride, cache_seqlens,
                       kv_begin, kv_end, NULL, NULL, dv, scale, causal, rows, n_rows, out_rows, lse_rows);
}

/* Token-level sparse decode over a bf16 latent cache: each query token (b, s) attends to the
 * listed key positions col_idx[row_ptr[b * s_q + s] .. row_ptr[b * s_q + s + 1]) that lie in
 * [0, n) (header, last paragraph).  row_ptr has batch * s_q + 1 entries, non-decreasing. */
int oracle_mla_decode_rows_sparse(const uint16_t *q, int64_t qs_b, int64_t qs_s, int64_t qs_h,
                                  int batch, int s_q, int h_q, int d,
                                  const uint16_t *k_cache, int64_t num_pages, int page, int h_kv,
                                  const int32_t *block_table, int64_t bt_stride,
                                  const int32_t *cache_seqlens,
                                  const int32_t *row_ptr, const int32_t *col_idx,
                                  const int32_t *kv_begin, const int32_t *kv_end,
                                  int dv, double scale, int causal,
                                  const int32_t *rows, int64_t n_rows,
                                  double *out_rows, double *lse_rows) {
    if (!k_cache || !row_ptr || !col_idx) return -1;
    for (int64_t i = 0; i < (int64_t)batch * s_q; ++i)
        if (row_ptr[i + 1] < row_ptr[i] || row_ptr[0] < 0) return -1;
    cache_t c = {k_cache, NULL, NULL, num_pages, page, h_kv, d};
    return decode_rows(q, qs_b, qs_s, qs_h, batch, s_q, h_q, d, &c, block_table, bt_stride, cache_seqlens,
                       kv_begin, kv_end, row_ptr, col_idx, dv, scale, causal, rows, n_rows, out_rows, lse_rows);
}
