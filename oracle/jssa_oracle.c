/*
 * JSSA decode-step oracle: a plain, slow, obviously correct CPU restatement of
 * what the decode hot path of Joint Subspace Sparse Attention computes, in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, calls or
 * includes this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark load it.  It shares no code, header or constant with the
 * CUDA sources.
 *
 * Sources (web pages on the method; cited by title and section):
 *   [ABS]  "Joint Subspace Sparse Attention for Efficient Long-Context Decoding"
 *          (arXiv 2610.19026), Abstract.
 *   [NEWS] "JSSA makes token-level sparse decoding gather-free, reaching up to
 *          full-KV throughput at 128K context" (news item), sections Synopsis,
 *          Interpretation and Perspective.
 *
 * Step order (one decode step of one attention layer):
 *   1. append      Kt[b,h,t,:] = round( K[b,t,h,:] . P[h] )        [NEWS Synopsis; ABS]
 *   2. score       s_t = sum_g (P_h^T q_g) . Kt[b,h,t,:]  (or max_g)  [NEWS Synopsis, Interp. para 2]
 *   3. select      top-k_b of s over t < T_b, order (s desc, t asc),
 *                  one distinct set per (batch, KV head)            [NEWS Synopsis; ABS]
 *   4. attend      softmax attention of every query head of the KV head
 *                  over the selected tokens, full-width q.k and V   [NEWS Interp. para 3; ABS]
 *   5. dense       step 4 over all t < T_b (or the last W tokens)   [ABS: the full-KV baseline]
 * Variant (for measurement; the method shares one set per KV head [ABS]):
 *   2'. score_heads  s[b,g,t] = (P_h^T q_g) . Kt[b,h,t,:] per query head
 *   3'. select       top-k_b of s per (batch, query head), as in step 3
 *   4'. attend_heads attention of each query head over its own set
 *
 * Readings taken where the pages are silent:
 *   - the G = Hq/Hkv query heads of a KV head are h*G .. h*G+G-1;
 *   - the group score is the SUM over the group of the subspace logits
 *     (MAX is offered as a variant);
 *   - ties in the score are broken by the lower token index;
 *   - k_b = min(k, T_b); unused index slots hold -1;
 *   - no forced sink / recent tokens;
 *   - T_b = 0 gives a zero output and lse = -inf.
 *
 * Parity pins: every function here is pinned by tests/test_oracle_*.py against
 * special cases with a closed form or a library routine (P = I, k = T, one
 * token, equal logits, torch SDPA in fp64), brute force on tiny inputs, and the
 * hand-worked fixtures under tests/golden/.
 *
 * Dtype codes for raw buffers: 0 = bf16 (uint16 bit patterns), 1 = fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_BF16 0
#define OR_FP32 1

static double ld_elem(const void *base, int dtype, size_t i)
{
    if (dtype == OR_BF16) {
        uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float *)base)[i];
}

/* Round a double once, to nearest-even, onto the bf16 grid (8 significant
 * bits, exponent range of fp32, gradual underflow, overflow to inf).  A single
 * rounding straight from fp64: no detour through fp32. */
double oracle_round_bf16(double x)
{
    if (x == 0.0 || isnan(x) || isinf(x))
        return x;
    int e;
    (void)frexp(x, &e);            /* |x| in [2^(e-1), 2^e) */
    int q = e - 8;                 /* ulp exponent with 8 significant bits */
    if (q < -133)                  /* bf16 subnormal spacing is 2^-133 */
        q = -133;
    double y = nearbyint(ldexp(x, -q)); /* default rounding mode: ties to even */
    double r = ldexp(y, q);
    const double maxv = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
    if (fabs(r) > maxv)
        return x > 0 ? INFINITY : -INFINITY;
    return r;
}

static uint16_t bf16_bits_of(double x)
{
    float f = (float)oracle_round_bf16(x); /* exact: already on the bf16 grid */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(bits >> 16);
}

static void st_elem(void *base, int dtype, size_t i, double v)
{
    if (dtype == OR_BF16)
        ((uint16_t *)base)[i] = bf16_bits_of(v);
    else
        ((float *)base)[i] = (float)v;
}

static int clamp_len(int v, int cap)
{
    return v < 0 ? 0 : (v > cap ? cap : v);
}

/* ---------------------------------------------------------------- append ---
 * Low-rank key cache written on append [NEWS Synopsis: keys are scored in a
 * shared low-dimensional query-key subspace; ABS: shared subspace]:
 *   Kt[b,h,t,j] = round_to_kt_dtype( sum_i K[b,t,h,i] * P[h,i,j] )
 * for t in [pos_begin[b], pos_begin[b] + n_new).  K is [B,T_cap,Hkv,d],
 * P is [Hkv,d,r] fp32, Kt is [B,Hkv,T_cap,r].  Kt_exact (optional, fp64, same
 * shape as Kt) receives the unrounded sums. */
int oracle_append_lowrank(int B, int T_cap, int Hkv, int d, int r,
                          const void *K, int k_dtype, const float *P,
                          const int32_t *pos_begin, int n_new,
                          void *Kt, int kt_dtype, double *Kt_exact)
{
    if (B < 0 || T_cap < 0 || Hkv <= 0 || d <= 0 || r <= 0 || n_new < 0)
        return -1;
    for (int b = 0; b < B; ++b)
        if (pos_begin[b] < 0 || pos_begin[b] + n_new > T_cap)
            return -1;
    long nrow = (long)B * Hkv * n_new;
#pragma omp parallel for schedule(static)
    for (long row = 0; row < nrow; ++row) {
        int b = (int)(row / ((long)Hkv * n_new));
        int h = (int)((row / n_new) % Hkv);
        int t = pos_begin[b] + (int)(row % n_new);
        size_t krow = (((size_t)b * T_cap + t) * Hkv + h) * (size_t)d;
        size_t orow = (((size_t)b * Hkv + h) * T_cap + t) * (size_t)r;
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += ld_elem(K, k_dtype, krow + i) * (double)P[((size_t)h * d + i) * r + j];
            if (Kt_exact)
                Kt_exact[orow + j] = acc;
            st_elem(Kt, kt_dtype, orow + j, acc);
        }
    }
    return 0;
}

/* ----------------------------------------------------------------- score ---
 * Subspace scoring [NEWS Synopsis and Interpretation para 2: queries and keys
 * share one low-dimensional scoring space]:
 *   qt_g[j] = sum_i q[b,g,i] * P[h,i,j]                (each query head g of h)
 *   SUM:  s[b,h,t] = sum_g sum_j qt_g[j] * Kt[b,h,t,j]
 *   MAX:  s[b,h,t] = max_g sum_j qt_g[j] * Kt[b,h,t,j]
 * for t < T_b.  Entries t >= T_b are set to -inf.  bh_list (optional) restricts
 * the work to the listed flattened (b*Hkv + h) pairs. */
int oracle_score(int B, int Hq, int Hkv, int d, int r, int T_cap,
                 const void *q, int q_dtype, const float *P,
                 const void *Kt, int kt_dtype, const int32_t *seq_lens, int agg,
                 const int32_t *bh_list, int n_bh, double *scores)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || (agg != 0 && agg != 1))
        return -1;
    int G = Hq / Hkv;
    int n = bh_list ? n_bh : B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < n; ++w) {
        int bh = bh_list ? bh_list[w] : w;
        int b = bh / Hkv, h = bh % Hkv;
        int Tb = clamp_len(seq_lens[b], T_cap);
        double *qt = (double *)malloc(sizeof(double) * (size_t)G * r);
        for (int g = 0; g < G; ++g)
            for (int j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i)
                    acc += ld_elem(q, q_dtype, ((size_t)b * Hq + h * G + g) * d + i) *
                           (double)P[((size_t)h * d + i) * r + j];
                qt[(size_t)g * r + j] = acc;
            }
        double *srow = scores + (size_t)bh * T_cap;
        for (int t = 0; t < T_cap; ++t) {
            if (t >= Tb) {
                srow[t] = -INFINITY;
                continue;
            }
            size_t krow = ((size_t)bh * T_cap + t) * (size_t)r;
            double total = 0.0, best = -INFINITY;
            for (int g = 0; g < G; ++g) {
                double lg = 0.0;
                for (int j = 0; j < r; ++j)
                    lg += qt[(size_t)g * r + j] * ld_elem(Kt, kt_dtype, krow + j);
                total += lg;
                if (lg > best)
                    best = lg;
            }
            srow[t] = agg == 0 ? total : best;
        }
        free(qt);
    }
    return 0;
}

/* Per-query-head subspace scores [variant: ABS and NEWS Synopsis describe one
 * distinct set per KV head; giving every query head its own set measures what
 * that sharing costs]:
 *   qt_g[j] = sum_i q[b,g,i] * P[h,i,j],  s[b,g,t] = sum_j qt_g[j] * Kt[b,h,t,j]
 * with h = g / G, for t < T_b; -inf beyond.  scores is [B, Hq, T_cap];
 * bh_list (optional) lists flattened (b*Hq + g) rows.  With G = 1 this is
 * oracle_score; SUM and MAX over a group are the sum and max of these rows. */
int oracle_score_heads(int B, int Hq, int Hkv, int d, int r, int T_cap,
                       const void *q, int q_dtype, const float *P,
                       const void *Kt, int kt_dtype, const int32_t *seq_lens,
                       const int32_t *bh_list, int n_bh, double *scores)
{
    if (Hkv <= 0 || Hq % Hkv != 0)
        return -1;
    int G = Hq / Hkv;
    int n = bh_list ? n_bh : B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < n; ++w) {
        int bg = bh_list ? bh_list[w] : w;
        int b = bg / Hq, g = bg % Hq, h = g / G;
        int Tb = clamp_len(seq_lens[b], T_cap);
        double *qt = (double *)malloc(sizeof(double) * (size_t)r);
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += ld_elem(q, q_dtype, ((size_t)b * Hq + g) * d + i) * (double)P[((size_t)h * d + i) * r + j];
            qt[j] = acc;
        }
        double *srow = scores + (size_t)bg * T_cap;
        for (int t = 0; t < T_cap; ++t) {
            if (t >= Tb) {
                srow[t] = -INFINITY;
                continue;
            }
            size_t krow = (((size_t)b * Hkv + h) * T_cap + t) * (size_t)r;
            double lg = 0.0;
            for (int j = 0; j < r; ++j)
                lg += qt[j] * ld_elem(Kt, kt_dtype, krow + j);
            srow[t] = lg;
        }
        free(qt);
    }
    return 0;
}

/* ---------------------------------------------------------------- select ---
 * Per-(batch, KV head) token top-k [NEWS Synopsis: a distinct selected token
 * set for each KV head; ABS: distinct per-KV-head selections]:
 * sort t in [0, T_b) by (s desc, t asc), keep the first k_b = min(k, T_b),
 * emit them in ascending t, pad with -1.  Equal scores (including -0.0 vs
 * +0.0, which compare equal) fall to the lower index. */
typedef struct {
    double s;
    int32_t t;
} or_pair;

static int cmp_pair(const void *pa, const void *pb)
{
    const or_pair *a = (const or_pair *)pa, *b = (const or_pair *)pb;
    if (a->s > b->s)
        return -1;
    if (a->s < b->s)
        return 1;
    return (a->t > b->t) - (a->t < b->t);
}

static int cmp_i32(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

int oracle_topk(int B, int Hkv, int T_cap, const double *scores,
                const int32_t *seq_lens, int k, const int32_t *bh_list, int n_bh,
                int32_t *idx, int32_t *count)
{
    if (k < 1)
        return -1;
    int n = bh_list ? n_bh : B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < n; ++w) {
        int bh = bh_list ? bh_list[w] : w;
        int b = bh / Hkv;
        int Tb = clamp_len(seq_lens[b], T_cap);
        int kb = k < Tb ? k : Tb;
        or_pair *pr = (or_pair *)malloc(sizeof(or_pair) * (size_t)(Tb > 0 ? Tb : 1));
        for (int t = 0; t < Tb; ++t) {
            pr[t].s = scores[(size_t)bh * T_cap + t];
            pr[t].t = t;
        }
        qsort(pr, (size_t)Tb, sizeof(or_pair), cmp_pair);
        int32_t *out = idx + (size_t)bh * k;
        for (int j = 0; j < kb; ++j)
            out[j] = pr[j].t;
        qsort(out, (size_t)kb, sizeof(int32_t), cmp_i32);
        for (int j = kb; j < k; ++j)
            out[j] = -1;
        if (count)
            count[bh] = kb;
        free(pr);
    }
    return 0;
}

/* Top-k with forced tokens [selection variant; the pages are silent on it: a
 * reading of "sink" and "recent-window" tokens that sparse decoders keep].
 * F = {t < n_sink} U {t >= T_b - n_recent}, t in [0, T_b).  If |F| >= k_b
 * the selection is the k_b smallest indices of F; otherwise it is F plus the
 * k_b - |F| tokens outside F that come first under (s desc, t asc).  Emitted
 * in ascending t, -1 padded.  n_sink = n_recent = 0 is oracle_topk. */
int oracle_topk_forced(int B, int Hkv, int T_cap, const double *scores,
                       const int32_t *seq_lens, int k, int n_sink, int n_recent,
                       const int32_t *bh_list, int n_bh, int32_t *idx, int32_t *count)
{
    if (k < 1 || n_sink < 0 || n_recent < 0)
        return -1;
    int n = bh_list ? n_bh : B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < n; ++w) {
        int bh = bh_list ? bh_list[w] : w;
        int b = bh / Hkv;
        int Tb = clamp_len(seq_lens[b], T_cap);
        int kb = k < Tb ? k : Tb;
        int32_t *out = idx + (size_t)bh * k;
        int nf = 0;
        for (int t = 0; t < Tb; ++t) {
            int forced = t < n_sink || t >= Tb - n_recent;
            if (forced && nf < kb)
                out[nf++] = t; /* ascending, the smallest indices first */
        }
        int rest = kb - nf;
        if (rest > 0) {
            or_pair *pr = (or_pair *)malloc(sizeof(or_pair) * (size_t)(Tb > 0 ? Tb : 1));
            int m = 0;
            for (int t = 0; t < Tb; ++t) {
                if (t < n_sink || t >= Tb - n_recent)
                    continue;
                pr[m].s = scores[(size_t)bh * T_cap + t];
                pr[m].t = t;
                ++m;
            }
            qsort(pr, (size_t)m, sizeof(or_pair), cmp_pair);
            for (int j = 0; j < rest; ++j)
                out[nf + j] = pr[j].t;
            free(pr);
        }
        qsort(out, (size_t)kb, sizeof(int32_t), cmp_i32);
        for (int j = kb; j < k; ++j)
            out[j] = -1;
        if (count)
            count[bh] = kb;
    }
    return 0;
}

/* ---------------------------------------------------------------- attend ---
 * Attention over a given token list per (b, h) [NEWS Interpretation para 3:
 * the selected key-value entries are read in place and attended as usual;
 * ABS: indexed attention under the standard GQA cache layout].  For each
 * query head g of KV head h:
 *   l_t = scale * sum_i q[b,g,i] * K[b,t,h,i]           (t in the list)
 *   m   = max_t l_t,  Z = sum_t exp(l_t - m)
 *   o_g = sum_t exp(l_t - m) / Z * V[b,t,h,0:dv]
 *   lse = m + ln Z
 * An empty list gives o_g = 0 and lse = -inf.  V rows are v_ld elements apart
 * per (t, h) step: dv for a separate V cache, d when V aliases K (latent cache). */
static void attend_head(int b, int hq, int h, int Hq, int Hkv, int d, int dv, int T_cap,
                        const void *q, int q_dtype, const void *K, const void *V,
                        int kv_dtype, int v_ld, const int32_t *list, int n,
                        double scale, double *out, double *lse)
{
    double *o = out + ((size_t)b * Hq + hq) * dv;
    for (int c = 0; c < dv; ++c)
        o[c] = 0.0;
    if (n == 0) {
        if (lse)
            lse[(size_t)b * Hq + hq] = -INFINITY;
        return;
    }
    double *lg = (double *)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        int t = list[j];
        size_t krow = (((size_t)b * T_cap + t) * Hkv + h) * (size_t)d;
        double acc = 0.0;
        for (int i = 0; i < d; ++i)
            acc += ld_elem(q, q_dtype, ((size_t)b * Hq + hq) * d + i) * ld_elem(K, kv_dtype, krow + i);
        lg[j] = scale * acc;
        if (lg[j] > m)
            m = lg[j];
    }
    double Z = 0.0;
    for (int j = 0; j < n; ++j)
        Z += exp(lg[j] - m);
    for (int j = 0; j < n; ++j) {
        int t = list[j];
        double w = exp(lg[j] - m) / Z;
        size_t vrow = (((size_t)b * T_cap + t) * Hkv + h) * (size_t)v_ld;
        for (int c = 0; c < dv; ++c)
            o[c] += w * ld_elem(V, kv_dtype, vrow + c);
    }
    if (lse)
        lse[(size_t)b * Hq + hq] = m + log(Z);
    free(lg);
}

/* every query head g of KV head h over the one list of (b, h) */
static void attend_one(int b, int h, int Hq, int Hkv, int d, int dv, int T_cap,
                       const void *q, int q_dtype, const void *K, const void *V,
                       int kv_dtype, int v_ld, const int32_t *list, int n,
                       double scale, double *out, double *lse)
{
    int G = Hq / Hkv;
    for (int g = 0; g < G; ++g)
        attend_head(b, h * G + g, h, Hq, Hkv, d, dv, T_cap, q, q_dtype, K, V, kv_dtype, v_ld, list, n, scale, out,
                    lse);
}

/* Indexed attention over per-(b,h) lists idx[b,h,0:count[b,h]] (the rest of
 * the k slots is ignored).  Returns -2 if a listed index is outside [0, T_b). */
int oracle_attend(int B, int Hq, int Hkv, int d, int dv, int T_cap,
                  const void *q, int q_dtype, const void *K, const void *V,
                  int kv_dtype, int v_ld, const int32_t *idx, const int32_t *count,
                  int k, const int32_t *seq_lens, double scale,
                  const int32_t *bh_list, int n_bh, double *out, double *lse)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || dv > v_ld)
        return -1;
    int n = bh_list ? n_bh : B * Hkv;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int w = 0; w < n; ++w) {
        int bh = bh_list ? bh_list[w] : w;
        int b = bh / Hkv, h = bh % Hkv;
        int Tb = clamp_len(seq_lens[b], T_cap);
        int c = count[bh];
        if (c < 0 || c > k) {
            bad = 1;
            continue;
        }
        const int32_t *list = idx + (size_t)bh * k;
        int ok = 1;
        for (int j = 0; j < c; ++j)
            if (list[j] < 0 || list[j] >= Tb)
                ok = 0;
        if (!ok) {
            bad = 1;
            continue;
        }
        attend_one(b, h, Hq, Hkv, d, dv, T_cap, q, q_dtype, K, V, kv_dtype, v_ld,
                   list, c, scale, out, lse);
    }
    return bad ? -2 : 0;
}

/* Dense (full-KV) attention: the list is t in [lo, T_b) with lo = 0, or
 * lo = max(0, T_b - window) for a sliding window (window > 0). */
int oracle_dense(int B, int Hq, int Hkv, int d, int dv, int T_cap,
                 const void *q, int q_dtype, const void *K, const void *V,
                 int kv_dtype, int v_ld, const int32_t *seq_lens, int window,
                 double scale, const int32_t *bh_list, int n_bh, double *out,
                 double *lse)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || dv > v_ld || window < 0)
        return -1;
    int n = bh_list ? n_bh : B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < n; ++w) {
        int bh = bh_list ? bh_list[w] : w;
        int b = bh / Hkv, h = bh % Hkv;
        int Tb = clamp_len(seq_lens[b], T_cap);
        int lo = (window > 0 && Tb > window) ? Tb - window : 0;
        int cnt = Tb - lo;
        int32_t *list = (int32_t *)malloc(sizeof(int32_t) * (size_t)(cnt > 0 ? cnt : 1));
        for (int j = 0; j < cnt; ++j)
            list[j] = lo + j;
        attend_one(b, h, Hq, Hkv, d, dv, T_cap, q, q_dtype, K, V, kv_dtype, v_ld,
                   list, cnt, scale, out, lse);
        free(list);
    }
    return 0;
}

/* Attention of each query head over its own list idx[b,g,0:count[b,g]]
 * (idx [B, Hq, k], count [B, Hq]) [variant of step 4: per-query-head sets],
 * the same arithmetic as oracle_attend.  bh_list (optional) lists flattened
 * (b*Hq + g) rows.  Returns -2 if a listed index is outside [0, T_b). */
int oracle_attend_heads(int B, int Hq, int Hkv, int d, int dv, int T_cap,
                        const void *q, int q_dtype, const void *K, const void *V,
                        int kv_dtype, int v_ld, const int32_t *idx, const int32_t *count,
                        int k, const int32_t *seq_lens, double scale,
                        const int32_t *bh_list, int n_bh, double *out, double *lse)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || dv > v_ld)
        return -1;
    int G = Hq / Hkv;
    int n = bh_list ? n_bh : B * Hq;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int w = 0; w < n; ++w) {
        int bg = bh_list ? bh_list[w] : w;
        int b = bg / Hq, g = bg % Hq;
        int Tb = clamp_len(seq_lens[b], T_cap);
        int c = count[bg];
        if (c < 0 || c > k) {
            bad = 1;
            continue;
        }
        const int32_t *list = idx + (size_t)bg * k;
        int ok = 1;
        for (int j = 0; j < c; ++j)
            if (list[j] < 0 || list[j] >= Tb)
                ok = 0;
        if (!ok) {
            bad = 1;
            continue;
        }
        attend_head(b, g, g / G, Hq, Hkv, d, dv, T_cap, q, q_dtype, K, V, kv_dtype, v_ld, list, c, scale, out, lse);
    }
    return bad ? -2 : 0;
}
