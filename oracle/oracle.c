/*
 * DSA region-sparse GQA: plain CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the slow, obviously-correct restatement of
 * what the CUDA library computes.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product path never does.  It
 * shares no code, header, table or constant generator with the CUDA library.
 *
 * Pages cited (title, site):
 *   [P1] Step-5-Preview 百万 token 长上下文: 滑窗 + DSA (kwkr.cn/news/601179)
 *   [P2] Step-5-Preview 如何实现1M长上下文？滑窗+DSA稀疏注意力混合机制完整揭秘 (yfxerp.com/news/376439)
 *   [P3] 100 万 token 上下文实测：Step 5 Preview 一次能吞下多大的工程 (kwkr.cn/news/593658)
 *
 * What the method computes, step by step (each function below cites its step):
 *   A1 region compression    [P1 §DSA ②], [P2 §区域压缩CSA]
 *   A2 indexer score         [P1 §DSA ③], [P2 §索引器打分]
 *   A3 top-k region select   [P2 §索引器打分], [P2 §第二招 sparse_config table]
 *   A4 sparse GQA attention  [P1 §DSA ④], [P2 §索引器打分], [P3 §一]
 *   sliding-window attention of the window layers [P1 §滑窗注意力], [P2 §第一招]
 *   indexer front end (projections, norm, partial RoPE, gates) [P2 §索引器打分]
 * The pages leave the arithmetic open; the fixed reading is:
 *   summary = mean of the 8 tokens' bf16 index_k, e4m3 with one fp32 absmax/448 scale;
 *   score(r,g) = sum_{h in group g} z_h * ReLU(q_h . s_{r,g}) / 16, heads 4g..4g+3;
 *   own region forced, ties to the lower region index;
 *   attention softmax(q K^T / sqrt(192)) V over the selected tokens t <= p.
 *
 * Precision: double everywhere except where the method fixes a precision (the fp32
 * mean handed to the quantiser, the fp32 scale, the fp32 quotient that is rounded to
 * e4m3).  Build with -ffp-contract=off and without fast-math.
 *
 * Parity pins live in tests/test_oracle_*.py; every function here is pinned there.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum {
    OR_REGION = 8,      /* tokens per region            [P1 §DSA ①] REGION_BLOCK_SIZE */
    OR_G = 4,           /* KV groups                    [P3 §一] num_attention_groups */
    OR_DI = 256,        /* summary / proxy dimension    [P2 §第二招] proxy_dim */
    OR_HI = 16,         /* indexer heads                [P1 §DSA ③] */
    OR_HQ = 64,         /* query heads                  [P3 §一] num_attention_heads */
    OR_D = 192,         /* attention head dim           [P3 §三] 2 x 4 x 192 */
    OR_PAGE = 64        /* tokens per K/V page (paged cache, [P3 §一] block_table) */
};

#define OR_Q_FP8 1u     /* flag: quantise index_q per (query, head) to e4m3 first */

/* ------------------------------------------------------------------ */
/* number formats                                                      */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32. */
static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

double oracle_bf16_to_f64(uint16_t b) { return (double)bf16_to_f32(b); }

/* Round a double to the nearest bf16, ties to even, in one step (no detour through
 * fp32, so no double rounding).  bf16: 8 exponent bits (bias 127), 7 stored mantissa
 * bits; normal range [2^-126, (2 - 2^-7) 2^127], subnormals in steps of 2^-133. */
uint16_t oracle_f64_to_bf16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (isnan(x)) return 0x7FC0u;
    if (isinf(x)) return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);               /* a = f * 2^e, f in [0.5, 1) -> a in [2^(e-1), 2^e) */
    int E = e - 1;              /* unbiased exponent of a */
    if (E < -126) E = -126;     /* subnormal binade shares the step of the lowest normal one */
    double step = ldexp(1.0, E - 7);
    double n = rint(a / step);  /* a/step is exact (power-of-two scaling); rint ties to even */
    double v = n * step;        /* may carry into the next binade: still exact */
    if (v > ldexp(255.0 / 128.0, 127)) {
        /* beyond the largest finite bf16 after rounding: infinity */
        return (uint16_t)(sign | 0x7F80u);
    }
    float f = (float)v;         /* exact: v has <= 8 significant bits within fp32 range */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFFu));
}

/* OCP 8-bit floating point, E4M3 ("fn": no infinities).  Layout s.eeee.mmm, exponent
 * bias 7.  Normal values (1 + m/8) 2^(e-7) for e = 1..15 except s.1111.111 (NaN);
 * subnormals (m/8) 2^-6 for e = 0.  Largest finite value 448 = 1.75 * 2^8. */
double oracle_e4m3_to_f64(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
    if (e == 0xF && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Nearest E4M3 value to a finite fp32, ties to even, magnitudes above 448 clamped to
 * 448 (saturating conversion).  NaN maps to the NaN code. */
uint8_t oracle_f32_to_e4m3(float xf)
{
    double x = (double)xf;
    uint8_t sign = signbit(x) ? 0x80u : 0u;
    double a = fabs(x);
    if (isnan(x)) return (uint8_t)(sign | 0x7Fu);
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);        /* saturate */
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    int E = e - 1;                                         /* a in [2^E, 2^(E+1)) */
    if (E < -6) E = -6;                                    /* subnormal step is 2^-9 */
    double step = ldexp(1.0, E - 3);                       /* 3 mantissa bits */
    double n = rint(a / step);                             /* exact quotient, ties to even */
    double v = n * step;
    if (v > 448.0) v = 448.0;                              /* 464 > a > 448 cannot reach here */
    /* encode v exactly */
    if (v < ldexp(1.0, -6)) {                              /* subnormal: v = k * 2^-9, k = 0..7 */
        int k = (int)ldexp(v, 9);
        return (uint8_t)(sign | (uint8_t)k);
    }
    int ev;
    double fv = frexp(v, &ev);                             /* v = fv * 2^ev, fv in [0.5, 1) */
    int eb = (ev - 1) + 7;                                 /* biased exponent, 1..15 */
    int mb = (int)((fv * 2.0 - 1.0) * 8.0);                /* exact: v has 4 significant bits */
    return (uint8_t)(sign | (uint8_t)(eb << 3) | (uint8_t)mb);
}

/* ------------------------------------------------------------------ */
/* A1: region compression                                              */
/* ------------------------------------------------------------------ */

/* One region summary for one KV group: rows[t] points at token t's 256 bf16 values.
 * [P1 §DSA ②] each complete region of 8 tokens becomes one 256-d FP8 summary;
 * [P2 §区域压缩CSA] only full regions are summarised.
 *   mean:  m_i = RN_fp32( (sum_{t=0..7} k_t,i) / 8 ), summed t = 0..7 in double
 *          (exact for any 8 bf16 values whose exponents span < 45 binades);
 *   scale: RN_fp32(absmax_i |m_i| / 448);
 *   code:  e4m3_RNE_satfinite( RN_fp32(m_i / scale) ); an all-zero region has scale 0
 *          and all codes 0. */
static void compress_one(const uint16_t *const rows[OR_REGION], uint8_t *code, float *scale_out)
{
    float m[OR_DI];
    float absmax = 0.0f;
    for (int i = 0; i < OR_DI; ++i) {
        double s = 0.0;
        for (int t = 0; t < OR_REGION; ++t) s += oracle_bf16_to_f64(rows[t][i]);
        m[i] = (float)(s * 0.125);
        float a = fabsf(m[i]);
        if (a > absmax) absmax = a;
    }
    float scale = absmax / 448.0f;
    *scale_out = scale;
    for (int i = 0; i < OR_DI; ++i) {
        if (scale == 0.0f) {
            code[i] = 0;
        } else {
            volatile float qv = m[i] / scale;   /* fp32 quotient, rounded once */
            code[i] = oracle_f32_to_e4m3(qv);
        }
    }
}

/* index_k: bf16 token rows, row t of group g at index_k[t*row_stride + g*256 + i].
 * Region i is made of rows src_row[i] .. src_row[i]+7 and is written to pool slot
 * dst_slot[i] of every group: the pool is group-major, summaries[(g*n_slots + slot)*256 + i],
 * scales[g*n_slots + slot]. */
void oracle_compress_regions(const uint16_t *index_k, int64_t row_stride,
                             const int64_t *src_row, const int64_t *dst_slot, int n_regions,
                             int64_t n_slots, uint8_t *summaries, float *scales)
{
#pragma omp parallel for schedule(static)
    for (int i = 0; i < n_regions; ++i) {
        for (int g = 0; g < OR_G; ++g) {
            const uint16_t *rows[OR_REGION];
            for (int t = 0; t < OR_REGION; ++t)
                rows[t] = index_k + (src_row[i] + t) * row_stride + (int64_t)g * OR_DI;
            int64_t slot = dst_slot[i];
            compress_one(rows, summaries + ((int64_t)g * n_slots + slot) * OR_DI,
                         scales + (int64_t)g * n_slots + slot);
        }
    }
}

/* ------------------------------------------------------------------ */
/* A2: indexer scores                                                  */
/* ------------------------------------------------------------------ */

/* Optional per-(query, head) quantisation of index_q to e4m3 (flag OR_Q_FP8), used by
 * the prefill path whose indexer is an FP8 x FP8 contraction.  Same codec as A1:
 * sq = RN_fp32(absmax/448), code = e4m3(RN_fp32(q/sq)); value = sq * e4m3 value. */
static void quantise_q_head(const uint16_t *qh, double *out)
{
    float absmax = 0.0f;
    for (int i = 0; i < OR_DI; ++i) {
        float a = fabsf(bf16_to_f32(qh[i]));
        if (a > absmax) absmax = a;
    }
    float sq = absmax / 448.0f;
    for (int i = 0; i < OR_DI; ++i) {
        if (sq == 0.0f) { out[i] = 0.0; continue; }
        volatile float qv = bf16_to_f32(qh[i]) / sq;
        out[i] = (double)sq * oracle_e4m3_to_f64(oracle_f32_to_e4m3(qv));
    }
}

/* scores[(qi*4 + g)*ld + r] for r = 0 .. own-1, own = q_pos[qi] / 8 (the regions
 * complete before the query's own region).  [P2 §索引器打分] score_regions scores a
 * query against all of its request's region summaries; the 4 KV groups map one to
 * one onto the regions' provider groups (num_provider_groups: 4), heads 4g..4g+3.
 *   score(r,g) = sum_{h=4g}^{4g+3} z_h * max(q_h . s_{r,g}, 0) / 16,
 *   s_{r,g,i} = e4m3 value of code i * scale_{r,g}.
 * Accumulated in double, rounded once to fp32.  Entries r >= own are not written. */
void oracle_indexer_scores(const uint16_t *index_q, const float *gate,
                           const int32_t *q_req, const int32_t *q_pos, int nq,
                           const uint8_t *summaries, const float *scales, const int64_t *sum_base,
                           int64_t n_slots, float *scores, int64_t ld, uint32_t flags)
{
    double *qd = (double *)malloc(sizeof(double) * (size_t)nq * OR_HI * OR_DI);
    for (int qi = 0; qi < nq; ++qi)
        for (int h = 0; h < OR_HI; ++h) {
            const uint16_t *qh = index_q + ((int64_t)qi * OR_HI + h) * OR_DI;
            double *dst = qd + ((int64_t)qi * OR_HI + h) * OR_DI;
            if (flags & OR_Q_FP8) quantise_q_head(qh, dst);
            else for (int i = 0; i < OR_DI; ++i) dst[i] = oracle_bf16_to_f64(qh[i]);
        }
    for (int qi = 0; qi < nq; ++qi) {
        int64_t own = q_pos[qi] / OR_REGION;
        int64_t base = sum_base[q_req[qi]];
        for (int g = 0; g < OR_G; ++g) {
#pragma omp parallel for schedule(static)
            for (int64_t r = 0; r < own; ++r) {
                int64_t slot = base + r;
                const uint8_t *s8 = summaries + ((int64_t)g * n_slots + slot) * OR_DI;
                double sc = (double)scales[(int64_t)g * n_slots + slot];
                double acc = 0.0;
                for (int h = OR_G * g; h < OR_G * g + OR_G; ++h) {
                    const double *qh = qd + ((int64_t)qi * OR_HI + h) * OR_DI;
                    double dot = 0.0;
                    for (int i = 0; i < OR_DI; ++i) dot += qh[i] * (oracle_e4m3_to_f64(s8[i]) * sc);
                    double relu = dot > 0.0 ? dot : 0.0;
                    acc += (double)gate[qi * OR_HI + h] * relu;
                }
                scores[((int64_t)qi * OR_G + g) * ld + r] = (float)(acc / 16.0);
            }
        }
    }
    free(qd);
}

/* ------------------------------------------------------------------ */
/* A3: top-k region selection                                          */
/* ------------------------------------------------------------------ */

typedef struct { double s; int32_t r; } cand_t;

/* higher score first; equal scores: lower region index first */
static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->r > y->r) - (x->r < y->r);
}

static int int_cmp(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Per (query, group): the own region own = q_pos/8 is always selected ([P2 §索引器打分]
 * "强制包含当前所在区域"); of the eligible regions r < own the k-1 best by (score desc,
 * index asc) join it.  Output: sel_idx[(qi*4+g)*k + j] ascending, count = min(k, own+1),
 * unused entries -1.  Scores equal as values (+0 and -0 included) tie. */
void oracle_topk_regions(const float *scores, int64_t ld, const int32_t *q_pos, int nq, int k,
                         int32_t *sel_idx, int32_t *sel_count)
{
#pragma omp parallel for schedule(dynamic)
    for (int qg = 0; qg < nq * OR_G; ++qg) {
        int qi = qg / OR_G;
        int64_t own = q_pos[qi] / OR_REGION;
        const float *row = scores + (int64_t)qg * ld;
        cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(own > 0 ? own : 1));
        for (int64_t r = 0; r < own; ++r) { c[r].s = (double)row[r]; c[r].r = (int32_t)r; }
        qsort(c, (size_t)own, sizeof(cand_t), cand_cmp);
        int64_t take = own < (int64_t)(k - 1) ? own : (int64_t)(k - 1);
        int32_t *out = sel_idx + (int64_t)qg * k;
        for (int64_t j = 0; j < take; ++j) out[j] = c[j].r;
        out[take] = (int32_t)own;
        int cnt = (int)(take + 1);
        qsort(out, (size_t)cnt, sizeof(int32_t), int_cmp);
        for (int j = cnt; j < k; ++j) out[j] = -1;
        sel_count[qg] = cnt;
        free(c);
    }
}

/* ------------------------------------------------------------------ */
/* A4: sparse GQA attention                                            */
/* ------------------------------------------------------------------ */

/* K/V cache: bf16 [num_pages][4][64][192]; token t of request b lives in page
 * block_table[b*max_pages + t/64], row t%64.  Query qi (request q_req, position p):
 * for head h in group g = h/16, T = union over selected regions r of {8r..8r+7},
 * restricted to t <= p (the causal mask only bites inside the own region).
 *   o_h = sum_t softmax_t(q_h . k_t / sqrt(192)) v_t,  lse_h = log sum_t exp(q_h . k_t / sqrt(192))
 * in double; out is rounded once to bf16, lse to fp32.  An empty T gives o = 0,
 * lse = -inf.  [P1 §DSA ④] attention runs on the real K/V of the selected regions only;
 * [P2 §索引器打分] _sparse_attention. */
void oracle_sparse_attention(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                             const int32_t *block_table, int max_pages,
                             const int32_t *q_req, const int32_t *q_pos, int nq,
                             const int32_t *sel_idx, const int32_t *sel_count, int k,
                             uint16_t *out, float *lse, double *out_f64)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)OR_D);
#pragma omp parallel for schedule(dynamic)
    for (int qh = 0; qh < nq * OR_HQ; ++qh) {
        int qi = qh / OR_HQ, h = qh % OR_HQ, g = h / (OR_HQ / OR_G);
        int b = q_req[qi], p = q_pos[qi];
        const int32_t *sel = sel_idx + ((int64_t)qi * OR_G + g) * k;
        int cnt = sel_count[qi * OR_G + g];
        const uint16_t *qv = q + ((int64_t)qi * OR_HQ + h) * OR_D;
        double qd[OR_D];
        for (int d = 0; d < OR_D; ++d) qd[d] = oracle_bf16_to_f64(qv[d]);
        /* collect logits */
        int ntok = 0;
        int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(cnt * OR_REGION + 1));
        double *lg = (double *)malloc(sizeof(double) * (size_t)(cnt * OR_REGION + 1));
        for (int j = 0; j < cnt; ++j) {
            int r = sel[j];
            for (int u = 0; u < OR_REGION; ++u) {
                int64_t t = (int64_t)r * OR_REGION + u;
                if (t > p) continue;
                int64_t page = block_table[(int64_t)b * max_pages + t / OR_PAGE];
                int64_t row = ((page * OR_G + g) * OR_PAGE + t % OR_PAGE) * OR_D;
                double dot = 0.0;
                for (int d = 0; d < OR_D; ++d) dot += qd[d] * oracle_bf16_to_f64(k_cache[row + d]);
                rows[ntok] = row;
                lg[ntok] = dot * inv_sqrt_d;
                ++ntok;
            }
        }
        double o[OR_D];
        for (int d = 0; d < OR_D; ++d) o[d] = 0.0;
        double l = -INFINITY;
        if (ntok > 0) {
            double mx = lg[0];
            for (int i = 1; i < ntok; ++i) if (lg[i] > mx) mx = lg[i];
            double den = 0.0;
            for (int i = 0; i < ntok; ++i) { lg[i] = exp(lg[i] - mx); den += lg[i]; }
            for (int i = 0; i < ntok; ++i) {
                double w = lg[i] / den;
                for (int d = 0; d < OR_D; ++d) o[d] += w * oracle_bf16_to_f64(v_cache[rows[i] + d]);
            }
            l = mx + log(den);
        }
        uint16_t *ov = out + ((int64_t)qi * OR_HQ + h) * OR_D;
        for (int d = 0; d < OR_D; ++d) ov[d] = oracle_f64_to_bf16(o[d]);
        if (out_f64) for (int d = 0; d < OR_D; ++d) out_f64[((int64_t)qi * OR_HQ + h) * OR_D + d] = o[d];
        if (lse) lse[(int64_t)qi * OR_HQ + h] = (float)l;
        free(rows);
        free(lg);
    }
}

/* ------------------------------------------------------------------ */
/* sliding-window attention (the 69 window layers)                      */
/* ------------------------------------------------------------------ */

/* Same cache layout as oracle_sparse_attention.  Query qi (request q_req, position p)
 * attends, for head h in group g = h/16, every token of the window
 *   T = { t : max(0, p - window + 1) <= t <= p },
 * the window's tokens read through the block table (a ring buffer is a block table
 * that maps the request's pages cyclically onto a few physical pages).
 *   o_h = sum_t softmax_t(q_h . k_t / sqrt(192)) v_t,  lse_h = log sum_t exp(...)
 * in double; out rounded once to bf16, lse to fp32.  [P1 §滑窗注意力]: the window layers
 * read only the most recent 512 tokens; [P2 §第一招]: sliding_window 512, a ring buffer
 * that keeps each request's last 512 tokens, attention inside the window. */
void oracle_window_attention(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                             const int32_t *block_table, int max_pages,
                             const int32_t *q_req, const int32_t *q_pos, int nq, int window,
                             uint16_t *out, float *lse, double *out_f64)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)OR_D);
#pragma omp parallel for schedule(dynamic)
    for (int qh = 0; qh < nq * OR_HQ; ++qh) {
        int qi = qh / OR_HQ, h = qh % OR_HQ, g = h / (OR_HQ / OR_G);
        int b = q_req[qi], p = q_pos[qi];
        int64_t lo = (int64_t)p - window + 1;
        if (lo < 0) lo = 0;
        int n = p >= 0 ? (int)(p - lo + 1) : 0;
        const uint16_t *qv = q + ((int64_t)qi * OR_HQ + h) * OR_D;
        double qd[OR_D];
        for (int d = 0; d < OR_D; ++d) qd[d] = oracle_bf16_to_f64(qv[d]);
        int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n + 1));
        double *lg = (double *)malloc(sizeof(double) * (size_t)(n + 1));
        for (int i = 0; i < n; ++i) {
            int64_t t = lo + i;
            int64_t page = block_table[(int64_t)b * max_pages + t / OR_PAGE];
            int64_t row = ((page * OR_G + g) * OR_PAGE + t % OR_PAGE) * OR_D;
            double dot = 0.0;
            for (int d = 0; d < OR_D; ++d) dot += qd[d] * oracle_bf16_to_f64(k_cache[row + d]);
            rows[i] = row;
            lg[i] = dot * inv_sqrt_d;
        }
        double o[OR_D];
        for (int d = 0; d < OR_D; ++d) o[d] = 0.0;
        double l = -INFINITY;
        if (n > 0) {
            double mx = lg[0];
            for (int i = 1; i < n; ++i) if (lg[i] > mx) mx = lg[i];
            double den = 0.0;
            for (int i = 0; i < n; ++i) { lg[i] = exp(lg[i] - mx); den += lg[i]; }
            for (int i = 0; i < n; ++i) {
                double w = lg[i] / den;
                for (int d = 0; d < OR_D; ++d) o[d] += w * oracle_bf16_to_f64(v_cache[rows[i] + d]);
            }
            l = mx + log(den);
        }
        uint16_t *ov = out + ((int64_t)qi * OR_HQ + h) * OR_D;
        for (int d = 0; d < OR_D; ++d) ov[d] = oracle_f64_to_bf16(o[d]);
        if (out_f64) for (int d = 0; d < OR_D; ++d) out_f64[((int64_t)qi * OR_HQ + h) * OR_D + d] = o[d];
        if (lse) lse[(int64_t)qi * OR_HQ + h] = (float)l;
        free(rows);
        free(lg);
    }
}

/* ------------------------------------------------------------------ */
/* indexer front end: hidden state -> index_q, index_k, z               */
/* ------------------------------------------------------------------ */

/* [P2 §索引器打分]: the indexer projects the hidden state to index_q / index_k / index_z,
 * then normalises and applies RoPE to part of the dimensions.  The pages give no constants;
 * the fixed reading, per token t at position pos[t] with hidden row h (bf16 [hid]):
 *   a_j   = sum_i W[j][i] h[i]                          (W bf16 [16*256 + 4*256 + 16][hid];
 *                                                         rows: q heads, k groups, gates)
 *   for each 256-d head vector x (16 q heads, 4 k groups, weights gamma_q / gamma_k [256]):
 *     y_d = x_d / sqrt(mean_d(x_d^2) + 1e-6) * gamma[d]                     (RMSNorm)
 *     for i < 32, theta = pos * 10000^(-2i/64):                            (RoPE on d < 64)
 *       y'_i      = y_i cos(theta) - y_{i+32} sin(theta)
 *       y'_{i+32} = y_{i+32} cos(theta) + y_i sin(theta)
 *   z_h = 1 / (1 + exp(-a_{gate h}))                                        (sigmoid gates)
 * in double; index_q/index_k rounded once to bf16, z to fp32. */
void oracle_indexer_frontend(const uint16_t *hidden, const uint16_t *w, const uint16_t *gamma_q,
                             const uint16_t *gamma_k, const int32_t *pos, int n_tok, int hid,
                             uint16_t *index_q, uint16_t *index_k, float *z)
{
    const int n_out = OR_HI * OR_DI + OR_G * OR_DI + OR_HI;
#pragma omp parallel for schedule(dynamic)
    for (int t = 0; t < n_tok; ++t) {
        double *a = (double *)malloc(sizeof(double) * (size_t)n_out);
        const uint16_t *h = hidden + (int64_t)t * hid;
        for (int j = 0; j < n_out; ++j) {
            const uint16_t *wr = w + (int64_t)j * hid;
            double s = 0.0;
            for (int i = 0; i < hid; ++i) s += oracle_bf16_to_f64(wr[i]) * oracle_bf16_to_f64(h[i]);
            a[j] = s;
        }
        for (int v = 0; v < OR_HI + OR_G; ++v) {
            const double *x = a + (int64_t)v * OR_DI;
            const uint16_t *gm = v < OR_HI ? gamma_q : gamma_k;
            double ms = 0.0;
            for (int d = 0; d < OR_DI; ++d) ms += x[d] * x[d];
            const double inv = 1.0 / sqrt(ms / OR_DI + 1e-6);
            double y[OR_DI];
            for (int d = 0; d < OR_DI; ++d) y[d] = x[d] * inv * oracle_bf16_to_f64(gm[d]);
            for (int i = 0; i < 32; ++i) {
                const double th = (double)pos[t] * pow(10000.0, -2.0 * i / 64.0);
                const double c = cos(th), sn = sin(th);
                const double u0 = y[i], u1 = y[i + 32];
                y[i] = u0 * c - u1 * sn;
                y[i + 32] = u1 * c + u0 * sn;
            }
            uint16_t *dst = v < OR_HI ? index_q + ((int64_t)t * OR_HI + v) * OR_DI
                                      : index_k + ((int64_t)t * OR_G + (v - OR_HI)) * OR_DI;
            for (int d = 0; d < OR_DI; ++d) dst[d] = oracle_f64_to_bf16(y[d]);
        }
        for (int hh = 0; hh < OR_HI; ++hh)
            z[(int64_t)t * OR_HI + hh] = (float)(1.0 / (1.0 + exp(-a[(OR_HI + OR_G) * OR_DI + hh])));
        free(a);
    }
}

/* ------------------------------------------------------------------ */
/* threads                                                             */
/* ------------------------------------------------------------------ */

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
