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

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
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
    if (!q || !k_cache || !block_table || !cache_seqlens || !rows || !out_rows || !lse_rows)
        return -1;
    if (h_kv <= 0 || h_q % h_kv != 0 || dv > d || page <= 0 || batch <= 0 || s_q <= 0)
        return -1;
    const int g = h_q / h_kv;
    int status = 0;

#pragma omp parallel
    {
        int64_t cap = 0;
        double *x = NULL;
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
            int64_t lo = kv_begin ? kv_begin[b] : 0;
            int64_t hi = kv_end ? kv_end[b] : n;
            if (hi > n) hi = n;
            if (lo < 0) lo = 0;
            for (int t = 0; t < dv; ++t) o[t] = 0.0;
            if (hi <= lo) {
                lse_rows[r] = -INFINITY;
                continue;
            }
            if (hi - lo > cap) {
                free(x);
                cap = hi - lo;
                x = (double *)malloc((size_t)cap * sizeof(double));
                if (!x) {
#pragma omp atomic write
                    status = -2;
                    cap = 0;
                    continue;
                }
            }
            const uint16_t *qrow = q + b * qs_b + s * qs_s + h * qs_h;
            /* pass 1: scores and their maximum */
            double M = -INFINITY;
            int bad = 0;
            for (int64_t j = lo; j < hi; ++j) {
                const int64_t phys = block_table[b * bt_stride + j / page];
                if (phys < 0 || phys >= num_pages) { bad = 1; break; }
                const uint16_t *c = k_cache + ((phys * page + j % page) * h_kv + kvh) * (int64_t)d;
                double acc = 0.0;
                for (int t = 0; t < d; ++t) acc += bf16_bits_to_double(qrow[t]) * bf16_bits_to_double(c[t]);
                x[j - lo] = scale * acc;
                if (x[j - lo] > M) M = x[j - lo];
            }
            if (bad) {
#pragma omp atomic write
                status = -3;
                lse_rows[r] = NAN;
                continue;
            }
            /* pass 2: normaliser and weighted sum of the first dv columns */
            double Z = 0.0;
            for (int64_t j = lo; j < hi; ++j) Z += exp(x[j - lo] - M);
            for (int64_t j = lo; j < hi; ++j) {
                const int64_t phys = block_table[b * bt_stride + j / page];
                const uint16_t *c = k_cache + ((phys * page + j % page) * h_kv + kvh) * (int64_t)d;
                const double p = exp(x[j - lo] - M) / Z;
                for (int t = 0; t < dv; ++t) o[t] += p * bf16_bits_to_double(c[t]);
            }
            lse_rows[r] = M + log(Z);
        }
        free(x);
    }
    return status;
}
