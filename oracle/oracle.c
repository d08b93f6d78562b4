/*
 * oracle.c -- plain, slow, obviously correct CPU reference for the fused
 * attention library.  TEST INFRASTRUCTURE ONLY: nothing in the product path
 * links, loads or calls this file.  It shares no code, header, table or
 * helper with the CUDA kernels.
 *
 * What it computes (fkl_python PR #6, "fkl.flash_attention: FA-2 forward
 * with fused epilogue + compressed int8 KV cache", Summary and Verification;
 * Foundry attention/README.md, "What it is (and is not)"):
 *
 *   o_i = sum_j softmax_j( scale * q_i . k_j  over the visible band ) v_j
 *
 * written the plain way: one score row is materialised in fp64, then a
 * two-pass softmax (max, then exp-sum), then the weighted sum of V rows.
 * The online-softmax rescaling of the GPU method reaches the same value up
 * to rounding order (Foundry attention/README.md, References: FlashAttention
 * paper and the online softmax trick), so the plain definition is the
 * oracle.
 *
 * Readings taken where the pages are silent:
 *  - causal alignment is bottom-right: query row i of a sequence with s_q
 *    queries and s_k keys sits at key position p = i + s_k - s_q;
 *  - a window W > 0 keeps keys j with p - W < j (W keys including self when
 *    causal); W <= 0 means no window;
 *  - a row whose band is empty gets uniform weights over all s_k keys of its
 *    sequence, i.e. the mean of V (SKaiNET-transformers PR #419, Summary:
 *    a sliding-window row whose band holds no key falls back to the
 *    engine's uniform softmax);
 *    with s_k = 0 the row is zero;
 *  - the epilogue ops are applied to the normalised output in list order
 *    (fkl_python PR #6, Summary: the epilogue op list).
 *
 * The quantiser is written in IEEE fp32 because its codes and scales are
 * compared bit for bit: amax = max|x|, s = amax / 127 (fp32 division),
 * c = clamp(rne(x / s), -127, 127); an all-zero row gets s = 0 and zero
 * codes (fkl_python PR #6, Summary, "compress_kv(): per-token int8
 * quantization (one fp32 scale/token)").
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EPI_MUL 1
#define ORACLE_EPI_ADD 2

/* Visible-key predicate for query row i (sequence lengths s_q, s_k). */
static int oracle_visible(int64_t i, int64_t j, int64_t s_q, int64_t s_k,
                          int causal, int64_t window)
{
    int64_t p = i + s_k - s_q;
    if (j < 0 || j >= s_k) return 0;
    if (causal && j > p) return 0;
    if (window > 0 && j <= p - window) return 0;
    return 1;
}

/*
 * One output row.  q_row[d]; k_rows/v_rows point at key 0 of the sequence
 * for the matching KV head, consecutive keys kv_row_stride doubles apart.
 * score is caller scratch of s_k doubles.
 */
static void oracle_row(const double *q_row, const double *k_rows,
                       const double *v_rows, int64_t kv_row_stride,
                       int64_t i, int64_t s_q, int64_t s_k, int64_t d,
                       double scale, int causal, int64_t window,
                       int n_epi, const int *epi_op, const double *epi_val,
                       double *score, double *out_row)
{
    int64_t j, c;
    int64_t n_vis = 0;
    double m = -INFINITY, denom = 0.0;

    for (c = 0; c < d; ++c) out_row[c] = 0.0;

    /* scores of the visible band */
    for (j = 0; j < s_k; ++j) {
        if (!oracle_visible(i, j, s_q, s_k, causal, window)) continue;
        double dot = 0.0;
        for (c = 0; c < d; ++c) dot += q_row[c] * k_rows[j * kv_row_stride + c];
        score[j] = scale * dot;
        if (score[j] > m) m = score[j];
        ++n_vis;
    }

    if (n_vis > 0) {
        /* two-pass softmax: exponentiate against the row max, then sum */
        for (j = 0; j < s_k; ++j) {
            if (!oracle_visible(i, j, s_q, s_k, causal, window)) continue;
            score[j] = exp(score[j] - m);
            denom += score[j];
        }
        for (j = 0; j < s_k; ++j) {
            if (!oracle_visible(i, j, s_q, s_k, causal, window)) continue;
            double w = score[j] / denom;
            for (c = 0; c < d; ++c) out_row[c] += w * v_rows[j * kv_row_stride + c];
        }
    } else if (s_k > 0) {
        /* empty band: uniform softmax over every key of the sequence */
        for (j = 0; j < s_k; ++j)
            for (c = 0; c < d; ++c) out_row[c] += v_rows[j * kv_row_stride + c];
        for (c = 0; c < d; ++c) out_row[c] /= (double)s_k;
    }

    /* epilogue chain, in list order */
    for (int e = 0; e < n_epi; ++e) {
        for (c = 0; c < d; ++c) {
            if (epi_op[e] == ORACLE_EPI_MUL) out_row[c] = out_row[c] * epi_val[e];
            else if (epi_op[e] == ORACLE_EPI_ADD) out_row[c] = out_row[c] + epi_val[e];
        }
    }
}

/*
 * Batched attention over a generic row layout.  Row r of Q/O for
 * (batch b, q-head h, position i) is
 *     q_bstride*b + q_hstride*h + q_start[b] + i,
 * and row of K/V for (b, kv-head g, key j) is
 *     k_bstride*b + k_hstride*g + k_start[b] + j;
 * every row holds d doubles.  Dense (batch*heads, seq, d) and varlen
 * (heads, total, d) layouts are both instances.  Q head h reads KV head
 * h / (hq / hkv).
 *
 * If n_sel > 0, only the listed (b, h, i) triples (sel[3*n .. 3*n+2]) are
 * computed; otherwise every row of every sequence is.
 * Returns 0, or -1 on an argument error.
 */
int oracle_attention(const double *q, const double *k, const double *v,
                     double *out,
                     int64_t batch, int64_t hq, int64_t hkv, int64_t d,
                     int64_t q_bstride, int64_t q_hstride,
                     const int64_t *q_start, const int64_t *q_len,
                     int64_t k_bstride, int64_t k_hstride,
                     const int64_t *k_start, const int64_t *k_len,
                     double scale, int causal, int64_t window,
                     int n_epi, const int *epi_op, const double *epi_val,
                     int64_t n_sel, const int64_t *sel)
{
    if (batch < 0 || hq <= 0 || hkv <= 0 || d <= 0 || hq % hkv != 0) return -1;
    int64_t group = hq / hkv;
    int64_t max_sk = 0, max_sq = 0, b;
    for (b = 0; b < batch; ++b) {
        if (k_len[b] > max_sk) max_sk = k_len[b];
        if (q_len[b] > max_sq) max_sq = q_len[b];
    }

    /* enumerate the work as (b, h, i) triples */
    int64_t n_work;
    int64_t *work = NULL;
    if (n_sel > 0) {
        n_work = n_sel;
    } else {
        n_work = 0;
        for (b = 0; b < batch; ++b) n_work += hq * q_len[b];
        work = (int64_t *)malloc(sizeof(int64_t) * 3 * (size_t)(n_work > 0 ? n_work : 1));
        if (!work) return -1;
        int64_t w = 0;
        for (b = 0; b < batch; ++b)
            for (int64_t h = 0; h < hq; ++h)
                for (int64_t i = 0; i < q_len[b]; ++i) {
                    work[3 * w] = b; work[3 * w + 1] = h; work[3 * w + 2] = i; ++w;
                }
        sel = work;
    }

    int failed = 0;
#pragma omp parallel
    {
        double *score = (double *)malloc(sizeof(double) * (size_t)(max_sk > 0 ? max_sk : 1));
        if (!score) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t w = 0; w < n_work; ++w) {
            if (!score) continue;
            int64_t bb = sel[3 * w], h = sel[3 * w + 1], i = sel[3 * w + 2];
            int64_t g = h / group;
            int64_t qrow = q_bstride * bb + q_hstride * h + q_start[bb] + i;
            int64_t krow = k_bstride * bb + k_hstride * g + k_start[bb];
            oracle_row(q + qrow * d, k + krow * d, v + krow * d, d,
                       i, q_len[bb], k_len[bb], d, scale, causal, window,
                       n_epi, epi_op, epi_val, score, out + qrow * d);
        }
        free(score);
    }
    free(work);
    (void)max_sq;
    return failed ? -1 : 0;
}

/*
 * Per-row int8 quantiser in IEEE fp32.  x[rows, d] fp32 (bf16 inputs are
 * widened exactly by the caller); codes[rows, d]; scales[rows].
 */
void oracle_compress_kv(const float *x, int64_t rows, int64_t d,
                        int8_t *codes, float *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float *xr = x + r * d;
        float amax = 0.0f;
        for (int64_t c = 0; c < d; ++c) {
            float a = fabsf(xr[c]);
            if (a > amax) amax = a;
        }
        float s = amax / 127.0f;
        scales[r] = s;
        for (int64_t c = 0; c < d; ++c) {
            int q = 0;
            if (s > 0.0f) {
                float t = nearbyintf(xr[c] / s); /* round half to even */
                if (t > 127.0f) t = 127.0f;
                if (t < -127.0f) t = -127.0f;
                q = (int)t;
            }
            codes[r * d + c] = (int8_t)q;
        }
    }
}

/* Dequantise c * s into fp64 (exact: |c| <= 127 and s is an fp32 value). */
void oracle_dequantize(const int8_t *codes, const float *scales, int64_t rows,
                       int64_t d, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < d; ++c)
            out[r * d + c] = (double)codes[r * d + c] * (double)scales[r];
}
