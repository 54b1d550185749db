/*
 * oracle.c -- plain, slow, fp64 CPU oracle for exact attention, HSTU pointwise attention and the
 * single-query decode step (contiguous cache, and paged cache with grouped query heads).
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library.  It shares no code, header, table or helper with the CUDA
 * path in exact_tiled_attention_43_b200/csrc, and it must never be used to produce a product result.
 *
 * Every function below is the plain definition written out: it materialises the score row s_ij and
 * the probability row p_ij of each query row in full before touching V, so it does NOT use tiling or
 * an online softmax.  All arithmetic is IEEE double.  Inputs are the exact bf16 values the GPU sees,
 * widened to double by the caller.
 *
 * Sources (pages of the reference):
 *   [FA-TH]  "FlashAttention (TH)", section "ปัญหาของ Attention แบบมาตรฐาน":
 *            Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V.
 *   [LEDGER] "AI attention complexity ledger", section "FLOPs 账：两个矩阵乘各出 2n²d":
 *            S = Q K^T / sqrt(d), O = P V, FLOPs = 2n^2 d + 2n^2 d = 4 n^2 d.
 *            Section "带宽账：decode 阶段的真正瓶颈": s_{n+1,j} = q_{n+1}^T k_j (j <= n), o = sum_j p_j v_j.
 *   [HSTU]   "同样是Attention架构，为什么昇腾NPU跑HSTU时延降低10倍、显存省97%？", section
 *            "先搞懂：HSTU到底难在哪？" (the Python definition: x = Q K^T; x *= alpha; x = silu(x);
 *            x *= mask / n; x = x V) and section "绝杀优化三：Jagged变长张量" (packed sequences + lengths).
 *
 * Readings taken where the pages are silent (each one is listed in the design notes):
 *   - the scale is passed in by the caller (1/sqrt(d) in the pages' formula), used as given;
 *   - causal means query row i sees keys j <= i of the same sequence (diagonal included), N_q == N_k;
 *   - lse is the natural-log logsumexp of the scaled score row: lse_i = m_i + ln sum_j exp(s_ij - m_i);
 *   - an empty key set yields o = 0 and lse = -inf;
 *   - HSTU's mask is lower-triangular including the diagonal, and its n is a scalar divisor passed as
 *     inv_n = 1/n.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ---------------------------------------------------------------------------------------------- */
/* One softmax-attention row.  q_i: [d]; key j lives at k + j*kstride, value j at v + j*vstride.     */
/* Writes o_i[d] and *lse_i.  Returns the number of multiply-adds executed (for the FLOP pin).       */
/* ---------------------------------------------------------------------------------------------- */
static int64_t softmax_attention_row(const double *qi, const double *k, size_t kstride,
                                     const double *v, size_t vstride, int nk, int d, double scale,
                                     double *o_i, double *lse_i)
{
    int64_t macs = 0;
    double *s = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    /* s_ij = scale * q_i . k_j   (the score row, [FA-TH] / [LEDGER]) */
    double m = -INFINITY;
    for (int j = 0; j < nk; ++j) {
        const double *kj = k + (size_t)j * kstride;
        double acc = 0.0;
        for (int t = 0; t < d; ++t) { acc += qi[t] * kj[t]; ++macs; }
        s[j] = scale * acc;
        if (s[j] > m) m = s[j];
    }
    /* p_ij = exp(s_ij - m_i) / sum_j exp(s_ij - m_i)   (softmax over the whole row) */
    double z = 0.0;
    for (int j = 0; j < nk; ++j) z += exp(s[j] - m);
    for (int t = 0; t < d; ++t) o_i[t] = 0.0;
    for (int j = 0; j < nk; ++j) {
        const double p = exp(s[j] - m) / z;
        const double *vj = v + (size_t)j * vstride;
        /* o_i = sum_j p_ij v_j */
        for (int t = 0; t < d; ++t) { o_i[t] += p * vj[t]; ++macs; }
    }
    *lse_i = (nk > 0) ? m + log(z) : -INFINITY;
    free(s);
    return macs;
}

/*
 * Dense attention over [B,H,N,d] row-major tensors.
 *   rows == NULL : every query row; o is [B,H,N,d], lse is [B,H,N].
 *   rows != NULL : only rows[0..nrows) of every head; o is [B,H,nrows,d], lse is [B,H,nrows].
 * causal != 0 keeps keys j <= i.  Returns the FLOPs executed (2 per multiply-add).
 */
EXPORT int64_t oracle_attn(const double *q, const double *k, const double *v, int B, int H, int N, int d,
                           double scale, int causal, const int *rows, int nrows, double *o, double *lse)
{
    const int nr = rows ? nrows : N;
    const int64_t nunits = (int64_t)B * H * nr;
    int64_t macs = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(+ : macs)
    for (int64_t u = 0; u < nunits; ++u) {
        const int64_t bh = u / nr;
        const int r = (int)(u % nr);
        const int i = rows ? rows[r] : r;
        const size_t head = (size_t)bh * N * d;
        const int nk = causal ? i + 1 : N;
        macs += softmax_attention_row(q + head + (size_t)i * d, k + head, (size_t)d, v + head, (size_t)d,
                                      nk, d, scale, o + (size_t)u * d, lse + u);
    }
    return 2 * macs;
}

/*
 * Variable-length (packed) attention.  q,k,v,o are [T,H,d] with T = cu[S]; sequence s owns rows
 * cu[s] .. cu[s+1]-1.  lse is [T,H].  No attention crosses a sequence boundary.
 */
EXPORT int64_t oracle_attn_varlen(const double *q, const double *k, const double *v, const int *cu, int S,
                                  int H, int d, double scale, int causal, double *o, double *lse)
{
    const int64_t T = cu[S];
    int64_t macs = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(+ : macs)
    for (int64_t u = 0; u < T * H; ++u) {
        const int64_t row = u / H;
        const int h = (int)(u % H);
        int s = 0;
        while (cu[s + 1] <= row) ++s;
        const int i = (int)(row - cu[s]);
        const int L = cu[s + 1] - cu[s];
        const int nk = causal ? i + 1 : L;
        const size_t base = ((size_t)cu[s] * H + h) * d;
        macs += softmax_attention_row(q + ((size_t)row * H + h) * d, k + base, (size_t)H * d, v + base,
                                      (size_t)H * d, nk, d, scale, o + ((size_t)row * H + h) * d, lse + u);
    }
    return 2 * macs;
}

/*
 * HSTU pointwise attention over jagged sequences, restating the page's Python definition row by row:
 *   x_ij = q_i . k_j ;  x_ij *= alpha ;  x_ij = silu(x_ij) = x_ij / (1 + exp(-x_ij)) ;
 *   x_ij *= mask_ij * inv_n ;  o_i = sum_j x_ij v_j
 * with mask_ij = 1 for j <= i (local indices) and 0 otherwise.  Every j in [0, L) is visited, masked
 * ones included, exactly as the dense formula multiplies by the mask.  Layout as oracle_attn_varlen.
 */
EXPORT int64_t oracle_hstu_jagged(const double *q, const double *k, const double *v, const int *cu, int S,
                                  int H, int d, double alpha, double inv_n, double *o)
{
    const int64_t T = cu[S];
    int64_t macs = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(+ : macs)
    for (int64_t u = 0; u < T * H; ++u) {
        const int64_t row = u / H;
        const int h = (int)(u % H);
        int s = 0;
        while (cu[s + 1] <= row) ++s;
        const int i = (int)(row - cu[s]);
        const int L = cu[s + 1] - cu[s];
        const double *qi = q + ((size_t)row * H + h) * d;
        double *oi = o + ((size_t)row * H + h) * d;
        for (int t = 0; t < d; ++t) oi[t] = 0.0;
        for (int j = 0; j < L; ++j) {
            const size_t off = ((size_t)(cu[s] + j) * H + h) * d;
            double x = 0.0;
            for (int t = 0; t < d; ++t) { x += qi[t] * k[off + t]; ++macs; }
            x *= alpha;
            x = x / (1.0 + exp(-x));
            const double mask = (j <= i) ? 1.0 : 0.0;
            x *= mask * inv_n;
            for (int t = 0; t < d; ++t) { oi[t] += x * v[off + t]; ++macs; }
        }
    }
    return 2 * macs;
}

/*
 * Single-query decode step ([LEDGER], decode section): for each (b, h) one query q[b,h,:] attends to
 * cached keys/values 0 .. kv_lens[b]-1 of kc/vc [B,H,Lmax,d], non-causal over the cache.
 * o is [B,H,d], lse is [B,H].
 */
EXPORT int64_t oracle_decode(const double *q, const double *kc, const double *vc, const int *kv_lens, int B,
                             int H, int Lmax, int d, double scale, double *o, double *lse)
{
    int64_t macs = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : macs)
    for (int64_t u = 0; u < (int64_t)B * H; ++u) {
        const int b = (int)(u / H);
        const size_t head = (size_t)u * Lmax * d;
        macs += softmax_attention_row(q + (size_t)u * d, kc + head, (size_t)d, vc + head, (size_t)d, kv_lens[b],
                                      d, scale, o + (size_t)u * d, lse + u);
    }
    return 2 * macs;
}

/*
 * Decode step over a paged cache with grouped query heads ([LEDGER], decode section; the same section names
 * GQA as a way to shrink the KV cache; "FlashAttention (TH)", section "FlashAttention-2": MQA; the
 * ops-transformer page: KV-cache management with PagedAttention).  For each (b, hq) with G = Hq / Hkv:
 * key/value row j (j < kv_lens[b]) of sequence b is row j % page_size of page block_table[b][j / page_size]
 * for kv head hq / G, in pools k_pages / v_pages [num_pages, Hkv, page_size, d].  The rows are gathered into
 * a contiguous [L, d] copy and the plain softmax row above is applied.  o is [B,Hq,d], lse is [B,Hq].
 */
EXPORT int64_t oracle_decode_paged(const double *q, const double *k_pages, const double *v_pages,
                                   const int *block_table, const int *kv_lens, int B, int Hq, int Hkv,
                                   int page_size, int max_pages, int d, double scale, double *o, double *lse)
{
    int64_t macs = 0;
    const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : macs)
    for (int64_t u = 0; u < (int64_t)B * Hq; ++u) {
        const int b = (int)(u / Hq), hq = (int)(u % Hq), g = hq / G;
        const int L = kv_lens[b];
        double *kg = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * d);
        double *vg = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * d);
        for (int j = 0; j < L; ++j) {
            const int page = block_table[(size_t)b * max_pages + j / page_size];
            const size_t row = (((size_t)page * Hkv + g) * page_size + (size_t)(j % page_size)) * d;
            memcpy(kg + (size_t)j * d, k_pages + row, sizeof(double) * d);
            memcpy(vg + (size_t)j * d, v_pages + row, sizeof(double) * d);
        }
        macs += softmax_attention_row(q + (size_t)u * d, kg, (size_t)d, vg, (size_t)d, L, d, scale,
                                      o + (size_t)u * d, lse + u);
        free(kg);
        free(vg);
    }
    return 2 * macs;
}

/* Threads later oracle calls use (the timed CPU baseline reports a one-core figure as well); n <= 0
 * leaves the OpenMP default.  Touches no arithmetic. */
EXPORT void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Number of OpenMP threads the oracle will use (reported with timed CPU baselines). */
EXPORT int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
