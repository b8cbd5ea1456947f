/*
 * rtp_oracle.c -- plain, slow, fp64 CPU oracle of the RTPurbo decode-step attention.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check of __graft_entry__ and the CPU
 * baseline / reference legs of bench.py load this library. The CUDA library shares no code,
 * header, table or helper with it, and neither side calls the other.
 *
 * What it follows (page title, then section / equation):
 *   [P1] "Full Attention Strikes Back: Transferring Full Attention into Sparse within Hundred
 *        Training Steps" (xllm-io paper review), section 三 "核心公式 / 自适应稀疏注意力":
 *          s_h(m,n) = (W^Q_h q^pre_{m,h})^T (W^K_h k^pre_{n,h})           (indexer score)
 *          O_h(m)   = sum_{n in S_h(m)} softmax_{S_h(m)}(q^T k_n / sqrt(d_h)) v_n
 *          S_h(m)   = Top-P(s_h(m,.), p)
 *   [P1 kernel] same page, section 三 "硬件感知解码内核": the top-p is sort-free, over a
 *        256-bin histogram that needs 1 KB per head whatever the sequence length.
 *   [P1 config] same page, section 五 "测试配置": sliding window 8192, 4 sink tokens,
 *        low-rank size 16, top-p 0.9.
 *   [P3] "Technical Summary: Full Attention Strikes Back ..." (gist.science), Methodology
 *        1 (local heads: sliding window with attention sinks; retrieval heads: dynamic sparse
 *        selection in decode) and 3 (top-p accumulates attention mass in the low-dimensional
 *        space until the cumulative threshold p is reached).
 *
 * Readings taken where the pages are silent (each is also listed in the design notes):
 *   - the indexer score is scaled by 1/sqrt(r) (r = 16 -> 0.25) before anything else;
 *   - the decode step receives q_idx = W^Q q^pre and the cached 16-d keys W^K k^pre; the
 *     projections themselves (orc_indexer_project) map a KV head's group of G pre-RoPE query
 *     heads, concatenated head-major (G * D values), and its pre-RoPE key (D values) to r dims;
 *   - the attention mass of token n is w_n = exp(s_n - s_max) (softmax up to the common
 *     normaliser, which cancels in the "reaches p" comparison);
 *   - the 256 bins have equal width over [s_max - range, s_max] (range = 16) of the scaled
 *     score: bin(n) = floor((s_n - (s_max - range)) * nbins / range), clamped to
 *     [0, nbins-1]; scores below the range fall in bin 0 and s_max itself in the top bin;
 *   - C_b = sum of the masses of bins b..nbins-1, accumulated from the top bin down;
 *     b* is the highest b with C_b >= p * C_0; the selection is every token with bin >= b*;
 *   - the G query heads of a GQA group share their KV head's selection;
 *   - fixed top-k through the same histogram (the top-k / top-p comparison of [P1] section 三
 *     "洞察 3: 动态 Top-P 选择", top-2k / 4k / 16k): b* is the highest b whose suffix COUNT
 *     N_b = #{n : bin(n) >= b} reaches k (b* = 0, every token, when k >= n_tok);
 *   - a local head attends over {0..sinks-1} U {N-window..N-1} (set union, positions
 *     clipped to [0, N)); the cache already holds the current token at position N-1;
 *   - prefill ([P3] Methodology 1: retrieval heads keep the full KV cache during prefill,
 *     local heads the sliding window with sinks): prompt position i attends causally over the
 *     key set a decode step of i + 1 tokens would use, dense for a retrieval head.
 *
 * All arithmetic is fp64 over the exact stored bf16 / fp16 values. Nothing is blocked,
 * fused or reordered beyond what the definitions above state.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_NOMEM (-2)

/* ---- storage formats ------------------------------------------------------------- */

/* bfloat16: the top 16 bits of an IEEE binary32. */
double orc_bf16_to_f64(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);            /* subnormal: m * 2^-14 * 2^-10 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* ---- indexer score [P1 自适应稀疏注意力, s_h(m,n)] ------------------------------------ */

/* s[n] = scale * sum_{i<r} q_idx[i] * k_idx[n][i]  for n in [0, n_tok). */
int orc_indexer_scores(const uint16_t *q_idx, const uint16_t *k_idx, int64_t n_tok, int r,
                       double scale, double *s)
{
    if (!q_idx || !k_idx || !s || n_tok < 0 || r <= 0)
        return ORC_ERR_ARG;
    for (int64_t n = 0; n < n_tok; n++) {
        double acc = 0.0;
        for (int i = 0; i < r; i++)
            acc += orc_f16_to_f64(q_idx[i]) * orc_f16_to_f64(k_idx[n * r + i]);
        s[n] = scale * acc;
    }
    return ORC_OK;
}

/* ---- indexer production [P1 自适应稀疏注意力: W^Q_h q^pre, W^K_h k^pre, before RoPE] ---- */

/*
 * For sequence b and KV head h (G = Hq / Hkv query heads per KV head, D = head_dim):
 *   q_idx[b][h][i] = sum_{j < G*D} wq[h][i][j] * q_pre[b][h*G + j/D][j%D]
 *   k_idx[b][h][i] = sum_{d < D}   wk[h][i][d] * k_pre[b][h][d]
 * over the bf16 inputs in fp64; the caller rounds to the 16-bit storage format.
 * Layouts: q_pre [B][Hq][D], k_pre [B][Hkv][D], wq [Hkv][r][G*D], wk [Hkv][r][D] (bf16 bits);
 * q_idx, k_idx [B][Hkv][r] fp64.
 */
int orc_indexer_project(const uint16_t *q_pre, const uint16_t *k_pre, const uint16_t *wq,
                        const uint16_t *wk, int B, int Hq, int Hkv, int D, int r, double *q_idx,
                        double *k_idx)
{
    if (!q_pre || !k_pre || !wq || !wk || !q_idx || !k_idx || B <= 0 || Hkv <= 0 || D <= 0 ||
        r <= 0 || Hq % Hkv != 0)
        return ORC_ERR_ARG;
    const int G = Hq / Hkv;
    const int64_t GD = (int64_t)G * D;
    for (int b = 0; b < B; b++) {
        for (int h = 0; h < Hkv; h++) {
            const uint16_t *qg = q_pre + ((int64_t)b * Hq + (int64_t)h * G) * D;
            const uint16_t *kh = k_pre + ((int64_t)b * Hkv + h) * D;
            for (int i = 0; i < r; i++) {
                const uint16_t *wqr = wq + ((int64_t)h * r + i) * GD;
                const uint16_t *wkr = wk + ((int64_t)h * r + i) * D;
                double aq = 0.0, ak = 0.0;
                for (int64_t j = 0; j < GD; j++)
                    aq += orc_bf16_to_f64(wqr[j]) * orc_bf16_to_f64(qg[j]);
                for (int d = 0; d < D; d++)
                    ak += orc_bf16_to_f64(wkr[d]) * orc_bf16_to_f64(kh[d]);
                q_idx[((int64_t)b * Hkv + h) * r + i] = aq;
                k_idx[((int64_t)b * Hkv + h) * r + i] = ak;
            }
        }
    }
    return ORC_OK;
}

/* ---- sort-free top-p over a histogram [P1 硬件感知解码内核; P3 Methodology 3] ------ */

/*
 * Histogram top-p of the scores s[0..n_tok).
 *   lo      = s_max - range
 *   bin(n)  = clamp(floor((s_n - lo) * nbins / range), 0, nbins-1)
 *   w_n     = exp(s_n - s_max)
 *   M_b     = sum_{bin(n)=b} w_n
 *   C_b     = M_{nbins-1} + ... + M_b   (accumulated from the top bin down)
 *   b*      = max{ b : C_b >= p * C_0 }
 *   S       = { n : bin(n) >= b* }, listed ascending.
 * Optional outputs (may be NULL): bin[n_tok], mass[nbins], suffix[nbins].
 */
int orc_hist_topp(const double *s, int64_t n_tok, double p, double range, int nbins,
                  int *bin, double *mass, double *suffix, int *bstar, int64_t *sel,
                  int64_t *n_sel)
{
    if (!s || !bstar || !sel || !n_sel || n_tok <= 0 || nbins <= 0 || !(range > 0.0) ||
        !(p > 0.0 && p <= 1.0))
        return ORC_ERR_ARG;

    double s_max = s[0];
    for (int64_t n = 1; n < n_tok; n++)
        if (s[n] > s_max)
            s_max = s[n];
    double lo = s_max - range;

    int *b_of = (int *)malloc(sizeof(int) * (size_t)n_tok);
    double *M = (double *)calloc((size_t)nbins, sizeof(double));
    double *C = (double *)calloc((size_t)nbins, sizeof(double));
    if (!b_of || !M || !C) {
        free(b_of); free(M); free(C);
        return ORC_ERR_NOMEM;
    }

    for (int64_t n = 0; n < n_tok; n++) {
        double x = floor((s[n] - lo) * (double)nbins / range);
        int b = x < 0.0 ? 0 : (x > (double)(nbins - 1) ? nbins - 1 : (int)x);
        b_of[n] = b;
        M[b] += exp(s[n] - s_max);
    }

    double acc = 0.0;
    for (int b = nbins - 1; b >= 0; b--) {
        acc += M[b];
        C[b] = acc;
    }
    double target = p * C[0];
    int bs = 0;
    for (int b = nbins - 1; b >= 0; b--) {
        if (C[b] >= target) {
            bs = b;
            break;
        }
    }

    int64_t k = 0;
    for (int64_t n = 0; n < n_tok; n++)
        if (b_of[n] >= bs)
            sel[k++] = n;

    *bstar = bs;
    *n_sel = k;
    if (bin)
        memcpy(bin, b_of, sizeof(int) * (size_t)n_tok);
    if (mass)
        memcpy(mass, M, sizeof(double) * (size_t)nbins);
    if (suffix)
        memcpy(suffix, C, sizeof(double) * (size_t)nbins);
    free(b_of); free(M); free(C);
    return ORC_OK;
}

/* ---- fixed top-k through the same histogram [P1 洞察 3, top-k vs top-p] ---------------- */

/*
 * Histogram top-k of the scores s[0..n_tok), k >= 1. The bins are those of orc_hist_topp:
 *   bin(n)  = clamp(floor((s_n - (s_max - range)) * nbins / range), 0, nbins - 1)
 *   K_b     = #{n : bin(n) = b}          (count of bin b)
 *   N_b     = K_{nbins-1} + ... + K_b    (accumulated from the top bin down)
 *   b*      = max{ b : N_b >= k }, or 0 if no bin reaches k (k > n_tok)
 *   S       = { n : bin(n) >= b* }, listed ascending.
 * Optional outputs (may be NULL): bin[n_tok], count[nbins], suffix[nbins] (N_b).
 */
int orc_hist_topk(const double *s, int64_t n_tok, int64_t k, double range, int nbins,
                  int *bin, int64_t *count, int64_t *suffix, int *bstar, int64_t *sel,
                  int64_t *n_sel)
{
    if (!s || !bstar || !sel || !n_sel || n_tok <= 0 || nbins <= 0 || !(range > 0.0) || k < 1)
        return ORC_ERR_ARG;

    double s_max = s[0];
    for (int64_t n = 1; n < n_tok; n++)
        if (s[n] > s_max)
            s_max = s[n];
    double lo = s_max - range;

    int *b_of = (int *)malloc(sizeof(int) * (size_t)n_tok);
    int64_t *K = (int64_t *)calloc((size_t)nbins, sizeof(int64_t));
    int64_t *Nb = (int64_t *)calloc((size_t)nbins, sizeof(int64_t));
    if (!b_of || !K || !Nb) {
        free(b_of); free(K); free(Nb);
        return ORC_ERR_NOMEM;
    }
    for (int64_t n = 0; n < n_tok; n++) {
        double x = floor((s[n] - lo) * (double)nbins / range);
        int b = x < 0.0 ? 0 : (x > (double)(nbins - 1) ? nbins - 1 : (int)x);
        b_of[n] = b;
        K[b] += 1;
    }
    int64_t acc = 0;
    for (int b = nbins - 1; b >= 0; b--) {
        acc += K[b];
        Nb[b] = acc;
    }
    int bs = 0;
    for (int b = nbins - 1; b >= 0; b--) {
        if (Nb[b] >= k) {
            bs = b;
            break;
        }
    }
    int64_t m = 0;
    for (int64_t n = 0; n < n_tok; n++)
        if (b_of[n] >= bs)
            sel[m++] = n;

    *bstar = bs;
    *n_sel = m;
    if (bin)
        memcpy(bin, b_of, sizeof(int) * (size_t)n_tok);
    if (count)
        memcpy(count, K, sizeof(int64_t) * (size_t)nbins);
    if (suffix)
        memcpy(suffix, Nb, sizeof(int64_t) * (size_t)nbins);
    free(b_of); free(K); free(Nb);
    return ORC_OK;
}

/* ---- exact (sort-based) top-p, the definition the histogram approximates ------------ */

typedef struct {
    double s;
    int64_t n;
} orc_scored;

static int orc_cmp_desc(const void *a, const void *b)
{
    const orc_scored *x = (const orc_scored *)a, *y = (const orc_scored *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->n > y->n) - (x->n < y->n); /* ties: ascending position */
}

static int orc_cmp_i64(const void *a, const void *b)
{
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x > y) - (x < y);
}

/* Sort by score descending (ties by ascending position) and keep the shortest prefix whose
 * cumulative mass exp(s - s_max) reaches p times the total mass of the same accumulation.
 * The kept positions are returned ascending. */
int orc_exact_topp(const double *s, int64_t n_tok, double p, int64_t *sel, int64_t *n_sel)
{
    if (!s || !sel || !n_sel || n_tok <= 0 || !(p > 0.0 && p <= 1.0))
        return ORC_ERR_ARG;
    orc_scored *v = (orc_scored *)malloc(sizeof(orc_scored) * (size_t)n_tok);
    double *cum = (double *)malloc(sizeof(double) * (size_t)n_tok);
    if (!v || !cum) {
        free(v); free(cum);
        return ORC_ERR_NOMEM;
    }
    for (int64_t n = 0; n < n_tok; n++) {
        v[n].s = s[n];
        v[n].n = n;
    }
    qsort(v, (size_t)n_tok, sizeof(orc_scored), orc_cmp_desc);
    double s_max = v[0].s, acc = 0.0;
    for (int64_t i = 0; i < n_tok; i++) {
        acc += exp(v[i].s - s_max);
        cum[i] = acc;
    }
    double target = p * cum[n_tok - 1];
    int64_t k = n_tok;
    for (int64_t i = 0; i < n_tok; i++) {
        if (cum[i] >= target) {
            k = i + 1;
            break;
        }
    }
    for (int64_t i = 0; i < k; i++)
        sel[i] = v[i].n;
    qsort(sel, (size_t)k, sizeof(int64_t), orc_cmp_i64);
    *n_sel = k;
    free(v); free(cum);
    return ORC_OK;
}

/* The k highest scores (ties by ascending position; every token when k >= n_tok), returned
 * ascending: the exact selection the histogram top-k approximates. */
int orc_exact_topk(const double *s, int64_t n_tok, int64_t k, int64_t *sel, int64_t *n_sel)
{
    if (!s || !sel || !n_sel || n_tok <= 0 || k < 1)
        return ORC_ERR_ARG;
    orc_scored *v = (orc_scored *)malloc(sizeof(orc_scored) * (size_t)n_tok);
    if (!v)
        return ORC_ERR_NOMEM;
    for (int64_t n = 0; n < n_tok; n++) {
        v[n].s = s[n];
        v[n].n = n;
    }
    qsort(v, (size_t)n_tok, sizeof(orc_scored), orc_cmp_desc);
    int64_t m = k < n_tok ? k : n_tok;
    for (int64_t i = 0; i < m; i++)
        sel[i] = v[i].n;
    qsort(sel, (size_t)m, sizeof(int64_t), orc_cmp_i64);
    *n_sel = m;
    free(v);
    return ORC_OK;
}

/* ---- local heads: sinks + sliding window [P1 测试配置; P3 Methodology 1] ---------------- */

/* {0..sinks-1} U {N-window..N-1}, clipped to [0, N), ascending, no duplicates. */
int orc_window_sink_set(int64_t n_tok, int64_t window, int64_t sinks, int64_t *sel,
                        int64_t *n_sel)
{
    if (!sel || !n_sel || n_tok <= 0 || window < 0 || sinks < 0)
        return ORC_ERR_ARG;
    int64_t k = 0;
    int64_t w0 = n_tok - window;
    for (int64_t n = 0; n < n_tok; n++)
        if (n < sinks || n >= w0)
            sel[k++] = n;
    *n_sel = k;
    return ORC_OK;
}

/* ---- exact softmax attention over a token set [P1 自适应稀疏注意力, O_h(m)] ------------- */

/*
 * For each query head g < G:
 *   x_j   = scale * sum_d q[g][d] * k[idx_j][d]
 *   o[g]  = sum_j exp(x_j - max x) v[idx_j] / sum_j exp(x_j - max x)
 * q: bf16 [G][D]; k, v: bf16 rows of D values, row idx_j at k + idx_j * D; o: [G][D].
 */
int orc_sparse_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const int64_t *idx, int64_t n_idx, int G, int D, double scale,
                         double *o)
{
    if (!q || !k || !v || !idx || !o || n_idx <= 0 || G <= 0 || D <= 0)
        return ORC_ERR_ARG;
    double *x = (double *)malloc(sizeof(double) * (size_t)n_idx);
    double *qd = (double *)malloc(sizeof(double) * (size_t)D);
    if (!x || !qd) {
        free(x); free(qd);
        return ORC_ERR_NOMEM;
    }
    for (int g = 0; g < G; g++) {
        for (int d = 0; d < D; d++)
            qd[d] = orc_bf16_to_f64(q[(int64_t)g * D + d]);
        double mx = -INFINITY;
        for (int64_t j = 0; j < n_idx; j++) {
            const uint16_t *kr = k + idx[j] * (int64_t)D;
            double acc = 0.0;
            for (int d = 0; d < D; d++)
                acc += qd[d] * orc_bf16_to_f64(kr[d]);
            x[j] = scale * acc;
            if (x[j] > mx)
                mx = x[j];
        }
        double den = 0.0;
        for (int64_t j = 0; j < n_idx; j++) {
            x[j] = exp(x[j] - mx);
            den += x[j];
        }
        double *og = o + (int64_t)g * D;
        for (int d = 0; d < D; d++)
            og[d] = 0.0;
        for (int64_t j = 0; j < n_idx; j++) {
            const uint16_t *vr = v + idx[j] * (int64_t)D;
            for (int d = 0; d < D; d++)
                og[d] += x[j] * orc_bf16_to_f64(vr[d]);
        }
        for (int d = 0; d < D; d++)
            og[d] /= den;
    }
    free(x); free(qd);
    return ORC_OK;
}

/* ---- prefill: attention of every prompt position [P3 Methodology 1] --------------------- */

/*
 * Row i (0 <= i < n_tok) of the prompt attends over the key set of a context of i + 1 tokens:
 * all of it, {0..i}, for a retrieval head (retrieval heads keep the full KV cache during
 * prefill), and {0..sinks-1} U {i+1-window .. i} for a local head (sliding window with
 * attention sinks). q holds the query rows listed in rows[] ([n_rows][D]); k, v [n_tok][D];
 * o [n_rows][D]. One query head at a time (G = 1).
 */
int orc_prefill_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t n_tok,
                     const int64_t *rows, int64_t n_rows, int D, int dense, int64_t window,
                     int64_t sinks, double scale, int num_threads, double *o)
{
    if (!q || !k || !v || !rows || !o || n_tok <= 0 || n_rows < 0 || D <= 0)
        return ORC_ERR_ARG;
    for (int64_t r = 0; r < n_rows; r++)
        if (rows[r] < 0 || rows[r] >= n_tok)
            return ORC_ERR_ARG;
    int err = ORC_OK;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads > 0 ? num_threads : omp_get_max_threads())
#else
    (void)num_threads;
#endif
    for (int64_t r = 0; r < n_rows; r++) {
        const int64_t i = rows[r];
        int64_t *idx = (int64_t *)malloc(sizeof(int64_t) * (size_t)(i + 1));
        int64_t n = 0;
        int rc = idx ? ORC_OK : ORC_ERR_NOMEM;
        if (rc == ORC_OK) {
            if (dense) {
                for (int64_t j = 0; j <= i; j++)
                    idx[j] = j;
                n = i + 1;
            } else {
                rc = orc_window_sink_set(i + 1, window, sinks, idx, &n);
            }
        }
        if (rc == ORC_OK)
            rc = orc_sparse_attention(q + r * (int64_t)D, k, v, idx, n, 1, D, scale,
                                      o + r * (int64_t)D);
        free(idx);
        if (rc != ORC_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
            err = rc;
        }
    }
    return err;
}

/* ---- one layer of the decode step, every (batch, KV head) ------------------------------ */

typedef struct {
    int batch, num_q_heads, num_kv_heads, head_dim, idx_dim, num_bins;
    int64_t max_ctx, window, sinks;
    double idx_range, idx_scale, attn_scale, top_p;
    int64_t top_k;  /* > 0: retrieval heads keep the histogram (or exact) top-k, not top-p */
} orc_layer_cfg;

enum { ORC_MODE_HIST = 0, ORC_MODE_EXACT = 1, ORC_MODE_DENSE = 2 };

/*
 * mode ORC_MODE_HIST : retrieval heads use the histogram top-p, local heads the window set
 *                      (the method itself);
 * mode ORC_MODE_EXACT: retrieval heads use the exact sort-based top-p, local heads the window;
 * mode ORC_MODE_DENSE: every head attends over all N tokens (full attention).
 * Layouts (row-major): q [B][Hq][D] bf16, q_idx [B][Hkv][r] f16, k_cache / v_cache
 * [B][Hkv][max_ctx][D] bf16, k_idx [B][Hkv][max_ctx][r] f16, seq_lens [B], mask [Hkv],
 * out [B][Hq][D] fp64, n_sel [B][Hkv] (may be NULL): size of the token set each head used.
 */
int orc_decode_layer(const orc_layer_cfg *c, int mode, const uint16_t *q, const uint16_t *q_idx,
                     const uint16_t *k_cache, const uint16_t *v_cache, const uint16_t *k_idx,
                     const int64_t *seq_lens, const uint8_t *retrieval_mask, double *out,
                     int64_t *n_sel, int num_threads)
{
    if (!c || !q || !k_cache || !v_cache || !seq_lens || !retrieval_mask || !out)
        return ORC_ERR_ARG;
    if (c->num_kv_heads <= 0 || c->num_q_heads % c->num_kv_heads != 0 || c->batch <= 0)
        return ORC_ERR_ARG;
    const int B = c->batch, Hq = c->num_q_heads, Hkv = c->num_kv_heads, D = c->head_dim;
    const int R = c->idx_dim, G = Hq / Hkv;
    const int64_t Nmax = c->max_ctx;
    for (int b = 0; b < B; b++)
        if (seq_lens[b] <= 0 || seq_lens[b] > Nmax)
            return ORC_ERR_ARG;
    if (num_threads <= 0)
        num_threads = 1;
    int status = ORC_OK;

#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads)
    for (int u = 0; u < B * Hkv; u++) {
        const int b = u / Hkv, h = u % Hkv;
        const int64_t N = seq_lens[b];
        const int64_t head = (int64_t)b * Hkv + h;
        const uint16_t *kh = k_cache + head * Nmax * D;
        const uint16_t *vh = v_cache + head * Nmax * D;
        const uint16_t *qg = q + ((int64_t)b * Hq + (int64_t)h * G) * D;
        double *og = out + ((int64_t)b * Hq + (int64_t)h * G) * D;
        int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
        double *s = NULL;
        int64_t k = 0;
        int rc = sel ? ORC_OK : ORC_ERR_NOMEM;

        if (rc == ORC_OK) {
            if (mode == ORC_MODE_DENSE) {
                for (int64_t n = 0; n < N; n++)
                    sel[n] = n;
                k = N;
            } else if (retrieval_mask[h]) {
                s = (double *)malloc(sizeof(double) * (size_t)N);
                if (!s || !q_idx || !k_idx) {
                    rc = s ? ORC_ERR_ARG : ORC_ERR_NOMEM;
                } else {
                    rc = orc_indexer_scores(q_idx + head * R, k_idx + head * Nmax * R, N, R,
                                            c->idx_scale, s);
                    if (rc == ORC_OK && mode == ORC_MODE_HIST && c->top_k > 0) {
                        int bs;
                        rc = orc_hist_topk(s, N, c->top_k, c->idx_range, c->num_bins, NULL,
                                           NULL, NULL, &bs, sel, &k);
                    } else if (rc == ORC_OK && mode == ORC_MODE_HIST) {
                        int bs;
                        rc = orc_hist_topp(s, N, c->top_p, c->idx_range, c->num_bins, NULL,
                                           NULL, NULL, &bs, sel, &k);
                    } else if (rc == ORC_OK && c->top_k > 0) {
                        rc = orc_exact_topk(s, N, c->top_k, sel, &k);
                    } else if (rc == ORC_OK) {
                        rc = orc_exact_topp(s, N, c->top_p, sel, &k);
                    }
                }
            } else {
                rc = orc_window_sink_set(N, c->window, c->sinks, sel, &k);
            }
        }
        if (rc == ORC_OK)
            rc = orc_sparse_attention(qg, kh, vh, sel, k, G, D, c->attn_scale, og);
        if (n_sel)
            n_sel[head] = (rc == ORC_OK) ? k : -1;
        if (rc != ORC_OK) {
#pragma omp critical
            status = rc;
        }
        free(s);
        free(sel);
    }
    return status;
}

/* Number of OpenMP threads a parallel region of this library would use (1 without OpenMP). */
int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
