/*
 * bsa_oracle.c -- plain, slow CPU oracle for query-aware top-k block-sparse
 * causal attention.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load or call this file's library.  The product
 * path (the CUDA library and its Python binding) never does, and shares no
 * code, header, table or helper with it.
 *
 * What it computes, step by step, in the order the source pages give:
 *
 *   1. pool   -- one mean vector per block of consecutive tokens ("粗粒度
 *                Block 打分", 稀疏注意力 tutorial §4.6; block = consecutive
 *                tokens, §4.5; "按块聚合 key" in the gated-sparse essay's
 *                pseudo-code step 1; "块级池化的Token表示" in the Sparse
 *                Frontier review §2.1).
 *   2. score  -- selector score s = pooled-q . pooled-k / sqrt(d): the
 *                "continuous score per context unit" of the SAS page
 *                (核心模块 1).  For gists (SSA page, 推理时的关键模块 1) the
 *                query is scored against every chunk's gist key.
 *   3. select -- hard top-k of the history units per query unit, with the
 *                current block always kept (SAS page, 核心洞察 / 核心模块 3,
 *                推理 paragraph: "each query selects the k highest units";
 *                essay pseudo-code step 2).  Ties go to the lowest index.
 *   4. attend -- softmax(QK^T/sqrt(d) + M)V with the additive mask
 *                M in {0, -inf} (稀疏注意力 tutorial §1 formula and §2 mask
 *                formula): M = 0 exactly on keys of the selected blocks that
 *                are not in the future of the query.
 *   5. gate   -- (SAS page, 核心模块 2-3) the selector's continuous score
 *                enters the logits in log space, normalised by a softmax over
 *                the kept blocks (current block included):
 *                logit += log g_j,  g_j = exp(s_j) / sum_{l kept} exp(s_l).
 *   6. gist   -- (SSA page, 推理时的关键模块 1-3) expand the top-k chunks to
 *                their tokens; every other chunk is represented by its gist
 *                key/value; attend over the mixture.
 *
 * Precision: steps 1-2 run in fp32 in a fixed order (pooling over heads then
 * tokens ascending; dot product over the channel index ascending; every
 * product and sum rounded to fp32; no fused multiply-add -- this file is
 * compiled with -ffp-contract=off).  Steps 4-6 run in fp64.  Inputs arrive as
 * fp32 arrays (a bf16 input is upcast exactly before the call).
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes):
 *   - under GQA the selection unit is the KV-head group: one score row per
 *     group, from the query mean over the group's heads and the block's
 *     tokens; the gate uses the same group score;
 *   - the current block's score uses full-block means (block-coarse);
 *   - fewer candidates than the budget: keep them all;
 *   - decode: every cached token is history; the "last block" is block nb-1;
 *   - gist decode keeps no forced chunk and drops the gists of expanded chunks;
 *   - NaN scores rank below every number, -inf included.
 *
 * Parallelism: OpenMP over independent output units only (rows, blocks,
 * selection rows); every unit's arithmetic is sequential, so results do not
 * depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* 1. Pooling (fixed-order fp32)                                            */
/* ------------------------------------------------------------------------ */

/* kbar[b,h,j,c] = (sum_{t in block j, ascending} k[b,h,t,c]) / bs */
void oracle_pool_keys(const float* k, int64_t B, int64_t H, int64_t N, int64_t d,
                      int64_t bs, float* kbar)
{
    const int64_t nb = N / bs;
    const int64_t units = B * H * nb;
#pragma omp parallel for schedule(static)
    for (int64_t u = 0; u < units; ++u) {
        const int64_t bh = u / nb, j = u % nb;
        for (int64_t c = 0; c < d; ++c) {
            float acc = 0.0f;
            for (int64_t t = 0; t < bs; ++t)
                acc = acc + k[(bh * N + j * bs + t) * d + c];
            kbar[u * d + c] = acc / (float)bs;
        }
    }
}

/* qbar[b,g,i,c] = (sum_{h in group g asc} sum_{t in block i asc} q[b,h,t,c]) / (G*bs)
 * Group g holds query heads g*G .. g*G+G-1 (G = Hq/Hkv). */
void oracle_pool_queries_grouped(const float* q, int64_t B, int64_t Hq, int64_t Hkv,
                                 int64_t N, int64_t d, int64_t bs, float* qbar)
{
    const int64_t nb = N / bs, G = Hq / Hkv;
    const int64_t units = B * Hkv * nb;
#pragma omp parallel for schedule(static)
    for (int64_t u = 0; u < units; ++u) {
        const int64_t b = u / (Hkv * nb), g = (u / nb) % Hkv, i = u % nb;
        for (int64_t c = 0; c < d; ++c) {
            float acc = 0.0f;
            for (int64_t hh = 0; hh < G; ++hh) {
                const int64_t h = g * G + hh;
                for (int64_t t = 0; t < bs; ++t)
                    acc = acc + q[((b * Hq + h) * N + i * bs + t) * d + c];
            }
            qbar[u * d + c] = acc / (float)(G * bs);
        }
    }
}

/* Decode: one query token per sequence, q [B,Hq,d].
 * qbar[b,g,c] = (sum_{h in group g asc} q[b,h,c]) / G */
void oracle_group_mean_query(const float* q, int64_t B, int64_t Hq, int64_t Hkv,
                             int64_t d, float* qbar)
{
    const int64_t G = Hq / Hkv;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t g = 0; g < Hkv; ++g)
            for (int64_t c = 0; c < d; ++c) {
                float acc = 0.0f;
                for (int64_t hh = 0; hh < G; ++hh)
                    acc = acc + q[(b * Hq + g * G + hh) * d + c];
                qbar[(b * Hkv + g) * d + c] = acc / (float)G;
            }
}

/* ------------------------------------------------------------------------ */
/* 2. Selector scores (fixed-order fp32)                                    */
/* ------------------------------------------------------------------------ */

/* The scale 1/sqrt(d), rounded once to fp32. */
static float score_scale(int64_t d) { return (float)(1.0 / sqrt((double)d)); }

/* acc = sum_c a[c]*b[c], channel index ascending, each product and each sum
 * rounded to fp32; then one fp32 multiply by the rounded scale. */
static float score_dot(const float* a, const float* b, int64_t d, float scale)
{
    float acc = 0.0f;
    for (int64_t c = 0; c < d; ++c) {
        const float prod = a[c] * b[c];
        acc = acc + prod;
    }
    return acc * scale;
}

/* Prefill: s[b,g,i,j] = qbar[b,g,i] . kbar[b,g,j] / sqrt(d) for j <= i,
 * -inf for j > i (future blocks are never candidates). */
void oracle_scores_prefill(const float* qbar, const float* kbar, int64_t B, int64_t Hkv,
                           int64_t nb, int64_t d, float* s)
{
    const float scale = score_scale(d);
    const int64_t rows = B * Hkv * nb;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t bg = r / nb, i = r % nb;
        for (int64_t j = 0; j < nb; ++j)
            s[r * nb + j] = (j <= i) ? score_dot(qbar + r * d, kbar + (bg * nb + j) * d, d, scale)
                                     : -INFINITY;
    }
}

/* Decode: s[b,g,j] = qbar[b,g] . kbar[b,g,j] / sqrt(d) for every block j. */
void oracle_scores_decode(const float* qbar, const float* kbar, int64_t B, int64_t Hkv,
                          int64_t nb, int64_t d, float* s)
{
    const float scale = score_scale(d);
    const int64_t rows = B * Hkv;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < nb; ++j)
            s[r * nb + j] = score_dot(qbar + r * d, kbar + (r * nb + j) * d, d, scale);
}

/* Gist: s[b,h,c] = q[b,h] . gk[b,g(h),c] / sqrt(d), one row per query head
 * (SSA page: under GQA each query head chooses its own chunks). */
void oracle_scores_gist(const float* q, const float* gk, int64_t B, int64_t Hq, int64_t Hkv,
                        int64_t nc, int64_t d, float* s)
{
    const float scale = score_scale(d);
    const int64_t G = Hq / Hkv;
    const int64_t rows = B * Hq;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t b = r / Hq, h = r % Hq, g = h / G;
        for (int64_t c = 0; c < nc; ++c)
            s[r * nc + c] = score_dot(q + r * d, gk + ((b * Hkv + g) * nc + c) * d, d, scale);
    }
}

/* ------------------------------------------------------------------------ */
/* 3. Top-k selection                                                       */
/* ------------------------------------------------------------------------ */

typedef struct { float s; int32_t j; } cand_t;

/* Order: larger score first; equal scores -> lower index first; a NaN ranks
 * below every number (including -inf). */
static int cand_cmp(const void* pa, const void* pb)
{
    const cand_t* a = (const cand_t*)pa;
    const cand_t* b = (const cand_t*)pb;
    const int an = isnan(a->s), bn = isnan(b->s);
    if (an != bn) return an ? 1 : -1;
    if (!an) {
        if (a->s > b->s) return -1;
        if (a->s < b->s) return 1;
    }
    return (a->j < b->j) ? -1 : (a->j > b->j) ? 1 : 0;
}

static int int_cmp(const void* pa, const void* pb)
{
    const int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a < b) ? -1 : (a > b);
}

/* mode 0 (causal block, prefill): row r is query block i = r % ncols;
 *        candidates are blocks j < i; block i is always kept.
 * mode 1 (last block, decode): candidates are j < ncols-1; block ncols-1 is
 *        always kept.
 * mode 2 (plain, gist): candidates are all j < ncols; nothing is forced.
 * Output per row: the kept indices ascending, then -1 up to idx_stride.
 * count (optional) receives the number of kept indices per row. */
void oracle_topk(const float* s, int64_t rows, int64_t ncols, int mode, int64_t kb,
                 int32_t* idx, int64_t idx_stride, int32_t* count)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t ncand, forced;
        if (mode == 0) { ncand = r % ncols; forced = r % ncols; }
        else if (mode == 1) { ncand = ncols - 1; forced = ncols - 1; }
        else { ncand = ncols; forced = -1; }
        cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(ncand > 0 ? ncand : 1));
        for (int64_t j = 0; j < ncand; ++j) { c[j].s = s[r * ncols + j]; c[j].j = (int32_t)j; }
        qsort(c, (size_t)ncand, sizeof(cand_t), cand_cmp);
        const int64_t take = (kb < ncand) ? kb : ncand;
        int32_t* out = idx + r * idx_stride;
        int64_t n = 0;
        for (int64_t t = 0; t < take; ++t) out[n++] = c[t].j;
        if (forced >= 0) out[n++] = (int32_t)forced;
        qsort(out, (size_t)n, sizeof(int32_t), int_cmp);
        for (int64_t t = n; t < idx_stride; ++t) out[t] = -1;
        if (count) count[r] = (int32_t)n;
        free(c);
    }
}

/* ------------------------------------------------------------------------ */
/* 4. The mask M of one query row                                           */
/* ------------------------------------------------------------------------ */

/* Mark the blocks listed in one index row (entries < 0 end the list). */
static void mark_blocks(const int32_t* list, int64_t stride, int64_t nb, unsigned char* sel)
{
    memset(sel, 0, (size_t)nb);
    for (int64_t t = 0; t < stride; ++t) {
        const int32_t j = list[t];
        if (j < 0) break;
        if (j < nb) sel[j] = 1;
    }
}

/* M_u = 0 iff key u lies in a selected block and is not in the query's
 * future (u <= t); -inf otherwise. Returned as an "allowed" flag. */
static int key_allowed(const unsigned char* sel, int64_t bs, int64_t t, int64_t u)
{
    return sel[u / bs] && (u <= t);
}

/* The full mask of one (batch, group) in prefill: mask[t*N + u] = 1 where
 * M_{t,u} = 0.  idx holds one row per query block: [nb, idx_stride]. */
void oracle_prefill_mask(int64_t N, int64_t bs, const int32_t* idx, int64_t idx_stride,
                         unsigned char* mask)
{
    const int64_t nb = N / bs;
    unsigned char* sel = (unsigned char*)malloc((size_t)nb);
    for (int64_t t = 0; t < N; ++t) {
        mark_blocks(idx + (t / bs) * idx_stride, idx_stride, nb, sel);
        for (int64_t u = 0; u < N; ++u) mask[t * N + u] = (unsigned char)key_allowed(sel, bs, t, u);
    }
    free(sel);
}

/* ------------------------------------------------------------------------ */
/* 5. Gate                                                                   */
/* ------------------------------------------------------------------------ */

/* logg[j] = log g_j for every kept block j of one row, g = softmax over the
 * kept blocks' scores (fp64; the largest score is subtracted before exp,
 * which leaves g unchanged). Blocks not kept get -inf. */
static void gate_log_weights(const float* srow, const int32_t* list, int64_t stride,
                             int64_t nb, double* logg)
{
    double smax = -INFINITY;
    for (int64_t j = 0; j < nb; ++j) logg[j] = -INFINITY;
    for (int64_t t = 0; t < stride && list[t] >= 0; ++t) {
        const double sj = (double)srow[list[t]];
        if (sj > smax) smax = sj;
    }
    double z = 0.0;
    for (int64_t t = 0; t < stride && list[t] >= 0; ++t)
        z += exp((double)srow[list[t]] - smax);
    for (int64_t t = 0; t < stride && list[t] >= 0; ++t) {
        const double g = exp((double)srow[list[t]] - smax) / z;
        logg[list[t]] = log(g);
    }
}

/* ------------------------------------------------------------------------ */
/* 6. Attention rows (fp64)                                                 */
/* ------------------------------------------------------------------------ */

static double dot64(const float* a, const float* b, int64_t d)
{
    double acc = 0.0;
    for (int64_t c = 0; c < d; ++c) acc += (double)a[c] * (double)b[c];
    return acc;
}

/* softmax over the allowed keys; writes out[d] and the natural-log LSE.
 * logits[n] are the finite logits of the n allowed keys, vals[n] their
 * value rows. With no allowed key the row is 0 and LSE is -inf. */
static void softmax_rows(const double* logits, const float* const* vals, int64_t n, int64_t d,
                         double* out, double* lse)
{
    for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
    if (n == 0) { *lse = -INFINITY; return; }
    double m = -INFINITY;
    for (int64_t u = 0; u < n; ++u) if (logits[u] > m) m = logits[u];
    double z = 0.0;
    for (int64_t u = 0; u < n; ++u) {
        const double p = exp(logits[u] - m);
        z += p;
        const float* vr = vals[u];
        for (int64_t c = 0; c < d; ++c) out[c] += p * (double)vr[c];
    }
    for (int64_t c = 0; c < d; ++c) out[c] /= z;
    *lse = m + log(z);
}

/* Prefill rows.  q [B,Hq,N,d], k/v [B,Hkv,N,d], idx [B,Hkv,nb,idx_stride],
 * gate_scores (NULL = ungated) [B,Hkv,nb,nb] = the selector scores s_{i,j}.
 * rows[n] = (b*Hq + h)*N + t selects the query rows to compute.
 * out [nrows,d], lse [nrows] (natural log). */
void oracle_attend_prefill_rows(const float* q, const float* k, const float* v,
                                int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                                int64_t bs, const int32_t* idx, int64_t idx_stride,
                                const float* gate_scores, double scale,
                                const int64_t* rows, int64_t nrows, double* out, double* lse)
{
    const int64_t nb = N / bs, G = Hq / Hkv;
    (void)B;
#pragma omp parallel
    {
        unsigned char* sel = (unsigned char*)malloc((size_t)nb);
        double* logg = (double*)malloc(sizeof(double) * (size_t)nb);
        double* logits = (double*)malloc(sizeof(double) * (size_t)N);
        const float** vals = (const float**)malloc(sizeof(float*) * (size_t)N);
#pragma omp for schedule(dynamic, 4)
        for (int64_t n = 0; n < nrows; ++n) {
            const int64_t r = rows[n];
            const int64_t b = r / (Hq * N), h = (r / N) % Hq, t = r % N;
            const int64_t g = h / G, i = t / bs;
            const int32_t* list = idx + ((b * Hkv + g) * nb + i) * idx_stride;
            mark_blocks(list, idx_stride, nb, sel);
            if (gate_scores)
                gate_log_weights(gate_scores + ((b * Hkv + g) * nb + i) * nb, list, idx_stride, nb, logg);
            const float* qr = q + r * d;
            const float* kb = k + (b * Hkv + g) * N * d;
            const float* vb = v + (b * Hkv + g) * N * d;
            int64_t m = 0;
            for (int64_t u = 0; u < N; ++u) {
                if (!key_allowed(sel, bs, t, u)) continue;   /* M_u = -inf: weight exactly 0 */
                double l = dot64(qr, kb + u * d, d) * scale;
                if (gate_scores) {
                    const double bias = logg[u / bs];
                    if (bias == -INFINITY) continue;          /* g_j = 0 */
                    l += bias;
                }
                logits[m] = l;
                vals[m] = vb + u * d;
                ++m;
            }
            softmax_rows(logits, vals, m, d, out + n * d, lse + n);
        }
        free(sel); free(logg); free(logits); free(vals);
    }
}

/* Decode rows.  q [B,Hq,d] (one token per sequence), k/v [B,Hkv,Nk,d],
 * idx [B,Hkv,idx_stride].  Every cached token is history of the query.
 * rows[n] = b*Hq + h. */
void oracle_attend_decode_rows(const float* q, const float* k, const float* v,
                               int64_t B, int64_t Hq, int64_t Hkv, int64_t Nk, int64_t d,
                               int64_t bs, const int32_t* idx, int64_t idx_stride, double scale,
                               const int64_t* rows, int64_t nrows, double* out, double* lse)
{
    const int64_t nb = Nk / bs, G = Hq / Hkv;
    (void)B;
#pragma omp parallel
    {
        unsigned char* sel = (unsigned char*)malloc((size_t)nb);
        double* logits = (double*)malloc(sizeof(double) * (size_t)Nk);
        const float** vals = (const float**)malloc(sizeof(float*) * (size_t)Nk);
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < nrows; ++n) {
            const int64_t r = rows[n];
            const int64_t b = r / Hq, h = r % Hq, g = h / G;
            mark_blocks(idx + (b * Hkv + g) * idx_stride, idx_stride, nb, sel);
            const float* kb = k + (b * Hkv + g) * Nk * d;
            const float* vb = v + (b * Hkv + g) * Nk * d;
            int64_t m = 0;
            for (int64_t u = 0; u < Nk; ++u) {
                if (!sel[u / bs]) continue;
                logits[m] = dot64(q + r * d, kb + u * d, d) * scale;
                vals[m] = vb + u * d;
                ++m;
            }
            softmax_rows(logits, vals, m, d, out + n * d, lse + n);
        }
        free(sel); free(logits); free(vals);
    }
}

/* Gist rows.  q [B,Hq,d], token k/v [B,Hkv,Nk,d], gist gk/gv [B,Hkv,nc,d]
 * with nc = Nk/chunk, idx [B,Hq,idx_stride] = the expanded chunks of each
 * query head.  Keys: every token of an expanded chunk, and the gist of every
 * chunk that is not expanded.  rows[n] = b*Hq + h. */
void oracle_attend_gist_rows(const float* q, const float* k, const float* v,
                             const float* gk, const float* gv,
                             int64_t B, int64_t Hq, int64_t Hkv, int64_t Nk, int64_t d,
                             int64_t chunk, const int32_t* idx, int64_t idx_stride, double scale,
                             const int64_t* rows, int64_t nrows, double* out, double* lse)
{
    const int64_t nc = Nk / chunk, G = Hq / Hkv;
    (void)B;
#pragma omp parallel
    {
        unsigned char* sel = (unsigned char*)malloc((size_t)nc);
        double* logits = (double*)malloc(sizeof(double) * (size_t)(Nk + nc));
        const float** vals = (const float**)malloc(sizeof(float*) * (size_t)(Nk + nc));
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < nrows; ++n) {
            const int64_t r = rows[n];
            const int64_t b = r / Hq, h = r % Hq, g = h / G;
            mark_blocks(idx + r * idx_stride, idx_stride, nc, sel);
            const float* kb = k + (b * Hkv + g) * Nk * d;
            const float* vb = v + (b * Hkv + g) * Nk * d;
            const float* gkb = gk + (b * Hkv + g) * nc * d;
            const float* gvb = gv + (b * Hkv + g) * nc * d;
            int64_t m = 0;
            for (int64_t c = 0; c < nc; ++c) {
                if (sel[c]) {
                    for (int64_t u = c * chunk; u < (c + 1) * chunk; ++u) {
                        logits[m] = dot64(q + r * d, kb + u * d, d) * scale;
                        vals[m] = vb + u * d;
                        ++m;
                    }
                } else {
                    logits[m] = dot64(q + r * d, gkb + c * d, d) * scale;
                    vals[m] = gvb + c * d;
                    ++m;
                }
            }
            softmax_rows(logits, vals, m, d, out + n * d, lse + n);
        }
        free(sel); free(logits); free(vals);
    }
}

/* Threads the OpenMP runtime will use (for reporting the CPU baseline). */
/* ------------------------------------------------------------------------ */
/* 7. Fixed pattern + dynamic blocks (MInference block-sparse)              */
/* ------------------------------------------------------------------------ */

/* The Sparse Frontier review (§2.2.3, and its §3.2 method table: "局部 +
 * 首块 + 动态选择块") describes block-sparse prefill as a local window, the
 * first block(s) of the sequence (the attention sinks of StreamingLLM,
 * §2.2.3) and a set of dynamically selected blocks per query block.
 * Row r is query block i = r % ncols.  Forced: the first `sink` blocks
 * (j < sink, j <= i) and the `local` most recent blocks (i-local < j <= i,
 * the current block included).  Candidates: every other block j < i; the
 * min(kb, #candidates) best of them by the step-3 order are kept.  Output:
 * kept blocks ascending, then -1; count = their number. */
void oracle_topk_pattern(const float* s, int64_t rows, int64_t ncols, int64_t sink, int64_t local,
                         int64_t kb, int32_t* idx, int64_t idx_stride, int32_t* count)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t i = r % ncols;
        unsigned char* forced = (unsigned char*)calloc((size_t)(i + 1), 1);
        cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(i + 1));
        for (int64_t j = 0; j <= i; ++j)
            if (j < sink || j > i - local) forced[j] = 1;
        int64_t ncand = 0;
        for (int64_t j = 0; j < i; ++j)
            if (!forced[j]) { c[ncand].s = s[r * ncols + j]; c[ncand].j = (int32_t)j; ++ncand; }
        qsort(c, (size_t)ncand, sizeof(cand_t), cand_cmp);
        const int64_t take = (kb < ncand) ? kb : ncand;
        int32_t* out = idx + r * idx_stride;
        int64_t n = 0;
        for (int64_t t = 0; t < take; ++t) out[n++] = c[t].j;
        for (int64_t j = 0; j <= i; ++j) if (forced[j]) out[n++] = (int32_t)j;
        qsort(out, (size_t)n, sizeof(int32_t), int_cmp);
        for (int64_t t = n; t < idx_stride; ++t) out[t] = -1;
        if (count) count[r] = (int32_t)n;
        free(c); free(forced);
    }
}

/* ------------------------------------------------------------------------ */
/* 8. One budget shared by the heads of a group (Ada-KV)                    */
/* ------------------------------------------------------------------------ */

/* Ada-KV (Sparse Frontier review §2.3.2) keeps the top (k x h) units over
 * all h heads together, so that important heads keep more keys and others
 * fewer.  s [rows][G][ncols]: each query head's decode scores of one
 * (batch, KV group) row.  The candidates are the pairs (h, j), j < ncols-1
 * (decode: the last block is kept by every head); the min(kb_total,
 * G*(ncols-1)) best by score are kept, equal scores going to the lower flat
 * index h*(ncols-1) + j, NaN below every number.  idx [rows][G][idx_stride]:
 * each head's kept blocks ascending, the last block included, then -1;
 * count [rows][G]. */
void oracle_topk_joint_heads(const float* s, int64_t rows, int64_t G, int64_t ncols, int64_t kb_total,
                             int32_t* idx, int64_t idx_stride, int32_t* count)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t per = ncols - 1, ncand = G * per;
        cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(ncand > 0 ? ncand : 1));
        for (int64_t h = 0; h < G; ++h)
            for (int64_t j = 0; j < per; ++j) {
                c[h * per + j].s = s[(r * G + h) * ncols + j];
                c[h * per + j].j = (int32_t)(h * per + j);
            }
        qsort(c, (size_t)ncand, sizeof(cand_t), cand_cmp);
        const int64_t take = (kb_total < ncand) ? kb_total : ncand;
        for (int64_t h = 0; h < G; ++h) {
            int32_t* out = idx + (r * G + h) * idx_stride;
            int64_t n = 0;
            for (int64_t t = 0; t < take; ++t)
                if (c[t].j / per == h) out[n++] = (int32_t)(c[t].j % per);
            out[n++] = (int32_t)(ncols - 1);
            qsort(out, (size_t)n, sizeof(int32_t), int_cmp);
            for (int64_t t = n; t < idx_stride; ++t) out[t] = -1;
            if (count) count[r * G + h] = (int32_t)n;
        }
        free(c);
    }
}

/* Decode rows where every query head has its own kept blocks: as step 6's
 * decode, with idx [B,Hq,idx_stride] read per head.  rows[n] = b*Hq + h. */
void oracle_attend_decode_heads_rows(const float* q, const float* k, const float* v,
                                     int64_t B, int64_t Hq, int64_t Hkv, int64_t Nk, int64_t d,
                                     int64_t bs, const int32_t* idx, int64_t idx_stride, double scale,
                                     const int64_t* rows, int64_t nrows, double* out, double* lse)
{
    const int64_t nb = Nk / bs, G = Hq / Hkv;
    (void)B;
#pragma omp parallel
    {
        unsigned char* sel = (unsigned char*)malloc((size_t)nb);
        double* logits = (double*)malloc(sizeof(double) * (size_t)Nk);
        const float** vals = (const float**)malloc(sizeof(float*) * (size_t)Nk);
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < nrows; ++n) {
            const int64_t r = rows[n];
            const int64_t b = r / Hq, h = r % Hq, g = h / G;
            mark_blocks(idx + r * idx_stride, idx_stride, nb, sel);
            const float* kb = k + (b * Hkv + g) * Nk * d;
            const float* vb = v + (b * Hkv + g) * Nk * d;
            int64_t m = 0;
            for (int64_t u = 0; u < Nk; ++u) {
                if (!sel[u / bs]) continue;
                logits[m] = dot64(q + r * d, kb + u * d, d) * scale;
                vals[m] = vb + u * d;
                ++m;
            }
            softmax_rows(logits, vals, m, d, out + n * d, lse + n);
        }
        free(sel); free(logits); free(vals);
    }
}

/* ------------------------------------------------------------------------ */
/* 9. Paged KV cache                                                        */
/* ------------------------------------------------------------------------ */

/* PagedAttention (稀疏注意力 tutorial §7): the logically contiguous KV cache
 * of a sequence is mapped onto physical blocks that need not be contiguous.
 * pool [P][Hkv][bs][d] holds physical blocks; table [B][max_blocks] maps
 * sequence b's logical block j to physical block table[b][j].  Writes the
 * logical view out [B][Hkv][nb*bs][d] of the first nb blocks. */
void oracle_paged_gather(const float* pool, const int32_t* table, int64_t B, int64_t Hkv, int64_t nb,
                         int64_t bs, int64_t d, int64_t max_blocks, float* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t bg = 0; bg < B * Hkv; ++bg) {
        const int64_t b = bg / Hkv, g = bg % Hkv;
        for (int64_t j = 0; j < nb; ++j) {
            const int64_t p = table[b * max_blocks + j];
            memcpy(out + ((bg * nb + j) * bs) * d, pool + ((p * Hkv + g) * bs) * d, sizeof(float) * (size_t)(bs * d));
        }
    }
}

/* ------------------------------------------------------------------------ */
/* 10. Two-level gist routing (H-SSA)                                       */
/* ------------------------------------------------------------------------ */

/* SSA page, 层级扩展 H-SSA: meta-gist tokens ("gist-of-gist", one per group of
 * M consecutive chunks) make a coarse selection first; then, inside the
 * selected groups, the ordinary gists score the chunks finely and the best
 * are expanded.  Per query head h of row b:
 *   meta  -- score q_h against the nm = nc/M meta-gist keys (step 2's fixed
 *            order), keep the km best groups (step 3's order, nothing forced);
 *   fine  -- score q_h against the gists of the chunks in the kept groups,
 *            keep the k best of those chunks.
 * mk [B,Hkv,nm,d], gk [B,Hkv,nc,d].  meta_idx [B,Hq,km_stride] and chunk_idx
 * [B,Hq,k_stride]: ascending, -1 padded. */
void oracle_hssa_select(const float* q, const float* gk, const float* mk, int64_t B, int64_t Hq, int64_t Hkv,
                        int64_t nc, int64_t M, int64_t d, int64_t km, int64_t k, int32_t* meta_idx,
                        int64_t km_stride, int32_t* chunk_idx, int64_t k_stride)
{
    const int64_t nm = nc / M, G = Hq / Hkv;
    const float scale = score_scale(d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < B * Hq; ++r) {
        const int64_t b = r / Hq, h = r % Hq, g = h / G;
        const float* qr = q + r * d;
        cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(nc > nm ? nc : nm));
        for (int64_t m = 0; m < nm; ++m) {
            c[m].s = score_dot(qr, mk + ((b * Hkv + g) * nm + m) * d, d, scale);
            c[m].j = (int32_t)m;
        }
        qsort(c, (size_t)nm, sizeof(cand_t), cand_cmp);
        const int64_t tm = (km < nm) ? km : nm;
        int32_t* mo = meta_idx + r * km_stride;
        for (int64_t t = 0; t < tm; ++t) mo[t] = c[t].j;
        qsort(mo, (size_t)tm, sizeof(int32_t), int_cmp);
        for (int64_t t = tm; t < km_stride; ++t) mo[t] = -1;
        int64_t n = 0;
        for (int64_t t = 0; t < tm; ++t)
            for (int64_t x = 0; x < M; ++x) {
                const int64_t ch = (int64_t)mo[t] * M + x;
                c[n].s = score_dot(qr, gk + ((b * Hkv + g) * nc + ch) * d, d, scale);
                c[n].j = (int32_t)ch;
                ++n;
            }
        qsort(c, (size_t)n, sizeof(cand_t), cand_cmp);
        const int64_t tk = (k < n) ? k : n;
        int32_t* co = chunk_idx + r * k_stride;
        for (int64_t t = 0; t < tk; ++t) co[t] = c[t].j;
        qsort(co, (size_t)tk, sizeof(int32_t), int_cmp);
        for (int64_t t = tk; t < k_stride; ++t) co[t] = -1;
        free(c);
    }
}

/* H-SSA rows.  Keys of query head h (the reading of the page's coarse-to-
 * fine routing, as SSA's mixed attention one level up): every token of an
 * expanded chunk; the gist of every other chunk inside a kept group; the
 * meta-gist of every group not kept.  rows[n] = b*Hq + h. */
void oracle_attend_hssa_rows(const float* q, const float* k, const float* v, const float* gk, const float* gv,
                             const float* mk, const float* mv, int64_t B, int64_t Hq, int64_t Hkv, int64_t Nk,
                             int64_t d, int64_t chunk, int64_t M, const int32_t* meta_idx, int64_t km_stride,
                             const int32_t* chunk_idx, int64_t k_stride, double scale, const int64_t* rows,
                             int64_t nrows, double* out, double* lse)
{
    const int64_t nc = Nk / chunk, nm = nc / M, G = Hq / Hkv;
    (void)B;
#pragma omp parallel
    {
        unsigned char* kept = (unsigned char*)malloc((size_t)nm);
        unsigned char* exp_ = (unsigned char*)malloc((size_t)nc);
        double* logits = (double*)malloc(sizeof(double) * (size_t)(Nk + nc + nm));
        const float** vals = (const float**)malloc(sizeof(float*) * (size_t)(Nk + nc + nm));
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < nrows; ++n) {
            const int64_t r = rows[n];
            const int64_t b = r / Hq, g = (r % Hq) / G;
            mark_blocks(meta_idx + r * km_stride, km_stride, nm, kept);
            mark_blocks(chunk_idx + r * k_stride, k_stride, nc, exp_);
            const int64_t bg = b * Hkv + g;
            int64_t m = 0;
            for (int64_t gr = 0; gr < nm; ++gr) {
                if (!kept[gr]) {
                    logits[m] = dot64(q + r * d, mk + (bg * nm + gr) * d, d) * scale;
                    vals[m] = mv + (bg * nm + gr) * d;
                    ++m;
                    continue;
                }
                for (int64_t c = gr * M; c < (gr + 1) * M; ++c) {
                    if (exp_[c]) {
                        for (int64_t u = c * chunk; u < (c + 1) * chunk; ++u) {
                            logits[m] = dot64(q + r * d, k + (bg * Nk + u) * d, d) * scale;
                            vals[m] = v + (bg * Nk + u) * d;
                            ++m;
                        }
                    } else {
                        logits[m] = dot64(q + r * d, gk + (bg * nc + c) * d, d) * scale;
                        vals[m] = gv + (bg * nc + c) * d;
                        ++m;
                    }
                }
            }
            softmax_rows(logits, vals, m, d, out + n * d, lse + n);
        }
        free(kept); free(exp_); free(logits); free(vals);
    }
}

/* ------------------------------------------------------------------------ */
/* 11. Backward of the (gated) sparse prefill attention                      */
/* ------------------------------------------------------------------------ */

/* SAS page, 核心洞察 and 核心模块 2: because the selector's continuous score
 * enters the softmax logits in log form, the language-modelling loss reaches
 * the selector by ordinary back-propagation.  Given the upstream gradient dO
 * of the output of step 4/5 (prefill rows, the mask of step 4, the gate of
 * step 5), this computes by the definition, in fp64:
 *   P_{t,u} = softmax_u(l_{t,u}),  l_{t,u} = scale q_t.k_u + log g_{j(u)}
 *   dV_u  += sum_t P_{t,u} dO_t
 *   dl_{t,u} = P_{t,u} (dO_t.v_u - sum_w P_{t,w} dO_t.v_w)
 *   dQ_t   = scale sum_u dl_{t,u} k_u,   dK_u += scale sum_t dl_{t,u} q_t
 *   for the unit (b, g, i) of row t and its kept block l:
 *   ds_{b,g,i,l} = sum_j dlogg_j (delta_{jl} - g_l), dlogg_j = sum over the
 *   unit's rows t and block j's keys u of dl_{t,u}   (d log g_j / d s_l).
 * q/dq [B,Hq,N,d], k/v/dk/dv [B,Hkv,N,d], dO [B,Hq,N,d]; gate_scores NULL:
 * ungated (ds untouched); ds [B,Hkv,nb,nb] (zero where no block is kept).
 * Every output is written whole (zero where nothing contributes). */
void oracle_attend_prefill_bwd(const float* q, const float* k, const float* v, const float* dO, int64_t B,
                               int64_t Hq, int64_t Hkv, int64_t N, int64_t d, int64_t bs, const int32_t* idx,
                               int64_t idx_stride, const float* gate_scores, double scale, double* dq, double* dk,
                               double* dv, double* ds)
{
    const int64_t nb = N / bs, G = Hq / Hkv;
    memset(dq, 0, sizeof(double) * (size_t)(B * Hq * N * d));
    memset(dk, 0, sizeof(double) * (size_t)(B * Hkv * N * d));
    memset(dv, 0, sizeof(double) * (size_t)(B * Hkv * N * d));
    if (gate_scores) memset(ds, 0, sizeof(double) * (size_t)(B * Hkv * nb * nb));
    /* one (batch, group) at a time: its dk, dv and ds are written by it alone */
#pragma omp parallel
    {
        unsigned char* sel = (unsigned char*)malloc((size_t)nb);
        double* logg = (double*)malloc(sizeof(double) * (size_t)nb);
        double* dlogg = (double*)malloc(sizeof(double) * (size_t)nb);
        double* p = (double*)malloc(sizeof(double) * (size_t)N);
        double* dp = (double*)malloc(sizeof(double) * (size_t)N);
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t bg = 0; bg < B * Hkv; ++bg) {
            const int64_t b = bg / Hkv, g = bg % Hkv;
            const float* kb = k + bg * N * d;
            const float* vb = v + bg * N * d;
            for (int64_t i = 0; i < nb; ++i) {
                const int32_t* list = idx + (bg * nb + i) * idx_stride;
                mark_blocks(list, idx_stride, nb, sel);
                if (gate_scores) gate_log_weights(gate_scores + (bg * nb + i) * nb, list, idx_stride, nb, logg);
                for (int64_t j = 0; j < nb; ++j) dlogg[j] = 0.0;
                for (int64_t hh = 0; hh < G; ++hh) {
                    const int64_t h = g * G + hh;
                    for (int64_t t = i * bs; t < (i + 1) * bs; ++t) {
                        const int64_t r = (b * Hq + h) * N + t;
                        const float* qr = q + r * d;
                        const float* dor = dO + r * d;
                        int64_t m = 0;
                        double mx = -INFINITY;
                        for (int64_t u = 0; u < N; ++u) {
                            if (!key_allowed(sel, bs, t, u)) continue;
                            double l = dot64(qr, kb + u * d, d) * scale;
                            if (gate_scores) {
                                if (logg[u / bs] == -INFINITY) continue;
                                l += logg[u / bs];
                            }
                            keys[m] = u;
                            p[m] = l;
                            if (l > mx) mx = l;
                            ++m;
                        }
                        if (m == 0) continue;
                        double z = 0.0;
                        for (int64_t a = 0; a < m; ++a) { p[a] = exp(p[a] - mx); z += p[a]; }
                        double dsum = 0.0;
                        for (int64_t a = 0; a < m; ++a) {
                            p[a] /= z;
                            dp[a] = dot64(dor, vb + keys[a] * d, d);
                            dsum += p[a] * dp[a];
                        }
                        double* dqr = dq + r * d;
                        for (int64_t a = 0; a < m; ++a) {
                            const int64_t u = keys[a];
                            const double dl = p[a] * (dp[a] - dsum);
                            double* dkr = dk + (bg * N + u) * d;
                            double* dvr = dv + (bg * N + u) * d;
                            const float* kr = kb + u * d;
                            for (int64_t c = 0; c < d; ++c) {
                                dqr[c] += scale * dl * (double)kr[c];
                                dkr[c] += scale * dl * (double)qr[c];
                                dvr[c] += p[a] * (double)dor[c];
                            }
                            dlogg[u / bs] += dl;
                        }
                    }
                }
                if (gate_scores) {
                    /* chain through log g_j = s_j - log sum_l exp(s_l) over the kept blocks */
                    double tot = 0.0;
                    for (int64_t j = 0; j < nb; ++j) if (logg[j] != -INFINITY) tot += dlogg[j];
                    double* dsr = ds + (bg * nb + i) * nb;
                    for (int64_t l = 0; l < nb; ++l)
                        if (logg[l] != -INFINITY) dsr[l] = dlogg[l] - exp(logg[l]) * tot;
                }
            }
        }
        free(sel); free(logg); free(dlogg); free(p); free(dp); free(keys);
    }
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
