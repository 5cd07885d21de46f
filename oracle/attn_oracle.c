/*
 * Float64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this code:
 * only the test suite, the smoke check and the benchmark's CPU-baseline and
 * reference legs use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes is the plain definition, row by row: scaled dot-product
 * attention softmax(QK^T / sqrt(d_k)) V as written on "Sviluppo AI ed Algebra
 * Lineare" (the SDPA formula, and the max-subtracted softmax of its section
 * "Online Softmax (La Formalizzazione Matematica)"), for the one-row object of
 * "Attenzione: softmax online, riscalamento e memoria", section 1:
 *
 *   for every batch b, query head h and query row i
 *     g    = h / (H / H_kv)                        (grouped-query head sharing)
 *     K_i  = { j : key_mask[b][j] != 0  and  (!causal or j <= i + n_kv - n_q) }
 *     s_j  = scale * sum_m q[b][h][i][m] * k[b][g][j][m]     (float64)
 *     mu   = max_{j in K_i} s_j
 *     w_j  = exp(s_j - mu),  l = sum_j w_j
 *     o    = sum_j w_j v[b][g][j] / l,   lse = mu + ln l
 *
 * Excluded keys are left out of every sum (the row object keeps only the keys
 * the mask admits), and an empty K_i gives o = 0, lse = -inf (the pages leave
 * the fully masked row to an explicit convention; this is the one taken).
 * The whole score row is materialised and the softmax takes two passes (max,
 * then exponentials), with no blocking and no online update.
 *
 * Inputs may be float64, float32 or bfloat16 (raw 16-bit patterns); every
 * element is widened exactly to float64 before use.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

static double widen(const void* base, int dtype, int64_t i) {
    if (dtype == ORC_F64) return ((const double*)base)[i];
    if (dtype == ORC_F32) return (double)((const float*)base)[i];
    /* bfloat16: the upper 16 bits of an IEEE float32 */
    uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* One query row against an explicit list of key rows.
 * q_off: element offset of the query vector; key_off[j]: element offset of
 * key/value row j (keys and values share the offset); n_keys may be 0. */
static void attend_row(const void* q, const void* k, const void* v, int dtype, int64_t q_off,
                       const int64_t* key_off, int64_t n_keys, int d, double scale, double* s,
                       double* o, double* lse) {
    for (int m = 0; m < d; ++m) o[m] = 0.0;
    if (n_keys == 0) {
        *lse = -INFINITY;
        return;
    }
    /* pass 1: all scores, and their maximum */
    double mu = -INFINITY;
    for (int64_t j = 0; j < n_keys; ++j) {
        double acc = 0.0;
        for (int m = 0; m < d; ++m) acc += widen(q, dtype, q_off + m) * widen(k, dtype, key_off[j] + m);
        s[j] = scale * acc;
        if (s[j] > mu) mu = s[j];
    }
    /* pass 2: weights relative to the maximum, their sum, and the weighted values */
    double l = 0.0;
    for (int64_t j = 0; j < n_keys; ++j) {
        double w = exp(s[j] - mu);
        l += w;
        for (int m = 0; m < d; ++m) o[m] += w * widen(v, dtype, key_off[j] + m);
    }
    for (int m = 0; m < d; ++m) o[m] /= l;
    *lse = mu + log(l);
}

static int threads_or_default(int nthreads) {
#ifdef _OPENMP
    return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Number of OpenMP threads a call with nthreads = 0 would use. */
int oracle_default_threads(void) { return threads_or_default(0); }

/*
 * Forward attention for a list of rows.
 * q: [B, H, n_q, d]; k, v: [B, H_kv, n_kv, d]; key_mask: [B, n_kv] uint8 or NULL.
 * rows: flat row ids r = (b*H + h)*n_q + i, or NULL for all B*H*n_q rows in order.
 * o: [n_rows, d] float64; lse: [n_rows] float64.
 * Returns 0, or -1 on invalid arguments, -2 on allocation failure.
 */
int oracle_attn_rows(const void* q, const void* k, const void* v, int dtype, const uint8_t* key_mask,
                     int B, int H, int H_kv, int n_q, int n_kv, int d, double scale, int causal,
                     const int64_t* rows, int64_t n_rows, double* o, double* lse, int nthreads) {
    if (B <= 0 || H <= 0 || H_kv <= 0 || n_q < 0 || n_kv < 0 || d <= 0 || H % H_kv != 0) return -1;
    if (rows == NULL) n_rows = (int64_t)B * H * n_q;
    const int group = H / H_kv;
    int err = 0;
    int nt = threads_or_default(nthreads);
#pragma omp parallel num_threads(nt)
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(n_kv > 0 ? n_kv : 1));
        int64_t* key_off = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_kv > 0 ? n_kv : 1));
        if (!s || !key_off) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < n_rows; ++t) {
                int64_t r = rows ? rows[t] : t;
                if (r < 0 || r >= (int64_t)B * H * n_q) {
#pragma omp atomic write
                    err = -1;
                    continue;
                }
                int i = (int)(r % n_q);
                int h = (int)((r / n_q) % H);
                int b = (int)(r / ((int64_t)n_q * H));
                int g = h / group;
                int64_t n_keys = 0;
                for (int j = 0; j < n_kv; ++j) {
                    if (key_mask && key_mask[(int64_t)b * n_kv + j] == 0) continue;
                    if (causal && (int64_t)j > (int64_t)i + n_kv - n_q) continue;
                    key_off[n_keys++] = (((int64_t)b * H_kv + g) * n_kv + j) * d;
                }
                attend_row(q, k, v, dtype, r * d, key_off, n_keys, d, scale, s, o + t * d, lse + t);
            }
        }
        free(s);
        free(key_off);
    }
    return err;
}

/*
 * One-token decode over a paged KV cache (block table of fixed-size pages).
 * q: [S, H, d]; k_pages, v_pages: [num_pages, page_size, H_kv, d];
 * block_table: [S, max_pages] int32 physical page ids; seq_lens: [S] int32.
 * Token t of sequence s lives in page block_table[s][t / page_size], slot t % page_size.
 * o: [S*H, d] float64; lse: [S*H] float64.  Returns 0, or -1 on invalid
 * arguments (including a page id outside [0, num_pages) or a length beyond the table).
 */
int oracle_decode_paged(const void* q, const void* k_pages, const void* v_pages, int dtype,
                        const int32_t* block_table, const int32_t* seq_lens, int S, int H, int H_kv, int d,
                        int page_size, int max_pages, int num_pages, double scale, double* o, double* lse,
                        int nthreads) {
    if (S < 0 || H <= 0 || H_kv <= 0 || d <= 0 || page_size <= 0 || H % H_kv != 0) return -1;
    for (int s = 0; s < S; ++s) {
        if (seq_lens[s] < 0 || (int64_t)seq_lens[s] > (int64_t)max_pages * page_size) return -1;
        int used = (seq_lens[s] + page_size - 1) / page_size;
        for (int p = 0; p < used; ++p) {
            int32_t pg = block_table[(int64_t)s * max_pages + p];
            if (pg < 0 || pg >= num_pages) return -1;
        }
    }
    const int group = H / H_kv;
    int max_len = 1;
    for (int s = 0; s < S; ++s) max_len = seq_lens[s] > max_len ? seq_lens[s] : max_len;
    int err = 0;
    int nt = threads_or_default(nthreads);
#pragma omp parallel num_threads(nt)
    {
        double* sc = (double*)malloc(sizeof(double) * (size_t)max_len);
        int64_t* key_off = (int64_t*)malloc(sizeof(int64_t) * (size_t)max_len);
        if (!sc || !key_off) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < (int64_t)S * H; ++r) {
                int s = (int)(r / H), h = (int)(r % H), g = h / group;
                int64_t n = seq_lens[s];
                for (int64_t t = 0; t < n; ++t) {
                    int64_t page = block_table[(int64_t)s * max_pages + t / page_size];
                    int64_t slot = t % page_size;
                    key_off[t] = ((page * page_size + slot) * H_kv + g) * d;
                }
                attend_row(q, k_pages, v_pages, dtype, r * d, key_off, n, d, scale, sc, o + r * d, lse + r);
            }
        }
        free(sc);
        free(key_off);
    }
    return err;
}

/*
 * A block of n_q query tokens per sequence against a paged KV cache: the query
 * rows are the last n_q positions of each sequence, so with causal = 1 query i of
 * sequence s keeps the keys t <= i + len_s - n_q (the same bottom-right
 * alignment as oracle_attn_rows), and with causal = 0 all len_s keys.
 * q: [S, H, n_q, d]; k_pages, v_pages: [num_pages, page_size, H_kv, d];
 * block_table: [S, max_pages] int32; seq_lens: [S] int32.  Token t of sequence s
 * lives in page block_table[s][t / page_size], slot t % page_size.
 * o: [S*H*n_q, d] float64; lse: [S*H*n_q] float64.  Returns 0, or -1 on invalid
 * arguments (including a page id outside [0, num_pages) or a length beyond the table).
 */
int oracle_prefill_paged(const void* q, const void* k_pages, const void* v_pages, int dtype,
                         const int32_t* block_table, const int32_t* seq_lens, int S, int H, int H_kv, int n_q,
                         int d, int page_size, int max_pages, int num_pages, double scale, int causal, double* o,
                         double* lse, int nthreads) {
    if (S < 0 || H <= 0 || H_kv <= 0 || n_q < 0 || d <= 0 || page_size <= 0 || H % H_kv != 0) return -1;
    for (int s = 0; s < S; ++s) {
        if (seq_lens[s] < 0 || (int64_t)seq_lens[s] > (int64_t)max_pages * page_size) return -1;
        int used = (seq_lens[s] + page_size - 1) / page_size;
        for (int p = 0; p < used; ++p) {
            int32_t pg = block_table[(int64_t)s * max_pages + p];
            if (pg < 0 || pg >= num_pages) return -1;
        }
    }
    const int group = H / H_kv;
    int max_len = 1;
    for (int s = 0; s < S; ++s) max_len = seq_lens[s] > max_len ? seq_lens[s] : max_len;
    int err = 0;
    int nt = threads_or_default(nthreads);
#pragma omp parallel num_threads(nt)
    {
        double* sc = (double*)malloc(sizeof(double) * (size_t)max_len);
        int64_t* key_off = (int64_t*)malloc(sizeof(int64_t) * (size_t)max_len);
        if (!sc || !key_off) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < (int64_t)S * H * n_q; ++r) {
                int s = (int)(r / ((int64_t)H * n_q));
                int h = (int)((r / n_q) % H), i = (int)(r % n_q), g = h / group;
                int64_t len = seq_lens[s];
                int64_t n = causal ? (int64_t)i + len - n_q + 1 : len;
                if (n > len) n = len;
                if (n < 0) n = 0;
                for (int64_t t = 0; t < n; ++t) {
                    int64_t page = block_table[(int64_t)s * max_pages + t / page_size];
                    int64_t slot = t % page_size;
                    key_off[t] = ((page * page_size + slot) * H_kv + g) * d;
                }
                attend_row(q, k_pages, v_pages, dtype, r * d, key_off, n, d, scale, sc, o + r * d, lse + r);
            }
        }
        free(sc);
        free(key_off);
    }
    return err;
}
