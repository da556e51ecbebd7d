/*
 * jssa.h -- C ABI of libjssa.so, the B200 (sm_100a) decode hot path of
 * Joint Subspace Sparse Attention (JSSA).
 *
 * Method pages, cited by title and section:
 *   [ABS]  "Joint Subspace Sparse Attention for Efficient Long-Context
 *          Decoding" (arXiv 2610.19026), Abstract.
 *   [NEWS] "JSSA makes token-level sparse decoding gather-free, reaching up
 *          to full-KV throughput at 128K context" (news item), Synopsis,
 *          Interpretation, Perspective.
 *
 * One decode step of one attention layer is
 *   jssa_append_lowrank (n_new = 1)  ->  jssa_select (= jssa_score + jssa_topk)
 *   ->  jssa_indexed_decode,
 * or all three at once with jssa_decode_step.  jssa_dense_decode and
 * jssa_gather_then_dense are the comparison paths the pages measure against
 * (full-KV attention [ABS]; gather into a contiguous buffer, then a dense
 * kernel [NEWS Interpretation para 3]).
 *
 * ------------------------------------------------------------ conventions --
 * Notation: G = Hq / Hkv query heads share KV head h; query head g belongs to
 * KV head g / G (heads h*G .. h*G+G-1).  T_b = seq_lens[b] <= T_cap.
 * k_b = min(k, T_b).
 *
 * Layouts (row-major, contiguous, all device memory, all caller-owned):
 *   q      [B, Hq, d]            dtype kv_dtype
 *   K      [B, T_cap, Hkv, d]    dtype kv_dtype (standard GQA cache layout)
 *   V      [B, T_cap, Hkv, dv]   dtype kv_dtype; for a latent (MLA) cache pass
 *                                V == K, Hkv = 1, dv < d: the value of a token
 *                                is the first dv entries of its key row
 *   P      [Hkv, d, r]           fp32, the per-KV-head shared basis
 *   Kt     [B, Hkv, T_cap, r]    dtype kt_dtype, the low-rank key cache
 *   scores [B, Hkv, T_cap]       fp32
 *   idx    [B, Hkv, k]           int32, selected token indices, ascending,
 *                                slots >= count hold -1
 *   count  [B, Hkv]              int32, k_b
 *   out    [B, Hq, dv]           dtype kv_dtype
 *   lse    [B, Hq]               fp32, natural-log log-sum-exp of the scaled
 *                                logits (-inf for an empty token set); optional
 * Every pointer must be 16-byte aligned.  Supported shapes: d in {64, 128,
 * 256} with dv == d, or the latent form d = 576, dv = 512, Hkv = 1; r a
 * power of two in [8, 128] with r <= d; G <= 16 (any G for the latent form);
 * 1 <= k <= 2048.
 *
 * Status: every entry point returns JSSA_OK or a negative JSSA_ERR_* code.
 * Arguments are checked on the host, synchronously, before anything is
 * enqueued; on an error nothing is enqueued and jssa_last_error() returns a
 * thread-local message.  Work is enqueued asynchronously on `stream` (a
 * cudaStream_t; NULL = the legacy default stream).  The library never
 * synchronises, allocates device memory or traps.
 *
 * Workspace: each call takes caller-owned device scratch `ws` of at least
 * jssa_workspace_size(...) bytes.  Zero it once with jssa_workspace_init()
 * before first use; afterwards the library keeps it valid (its arrival
 * counters reset themselves).  Calls that share one workspace must be
 * ordered (same stream, or events); concurrent calls need separate ones.
 * Word 0 of the workspace is a sticky status word: kernels OR in
 * JSSA_DEV_* bits for bad data they meet (and skip that item); read it back
 * with a device-to-host copy of 4 bytes; jssa_workspace_init() clears it.
 *
 * Host state: launch plans of the selection pass are cached per device and
 * shape in host memory (mutex-protected).  The selection (jssa_topk,
 * jssa_select, jssa_decode_step) has three forms with identical results:
 * one thread-block cluster per (b, h) holding the keys of its rows in shared
 * memory, taken when all B*Hkv clusters fit on the GPU at once; otherwise a
 * persistent streaming pass with a segment merge, warp-specialised for SUM
 * over the low-rank cache, block-synchronous for the other cases.  The
 * decode step with k <= 256 (SUM, bf16 caches, not the latent form) tries
 * the streaming form first, since it then runs as one fused launch.  The
 * `form` field of jssa_select_opts forces one form where it has a kernel
 * (tests and measurement); jssa_workspace_size covers every form.  The
 * library reads no environment variables.
 */
#ifndef JSSA_H
#define JSSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define JSSA_VERSION 2

#if defined(__GNUC__)
#define JSSA_API __attribute__((visibility("default")))
#else
#define JSSA_API
#endif

typedef void *jssa_stream_t; /* a cudaStream_t */

enum {
    JSSA_OK = 0,
    JSSA_ERR_INVALID_ARG = -1, /* null pointer, bad dimension, k < 1, r > d, misaligned pointer */
    JSSA_ERR_UNSUPPORTED = -2, /* a shape / dtype combination without a kernel */
    JSSA_ERR_WORKSPACE = -3,   /* ws_bytes below jssa_workspace_size() */
    JSSA_ERR_CUDA = -4         /* a CUDA runtime call or launch failed */
};

/* Device status bits (workspace word 0). */
enum {
    JSSA_DEV_SEQLEN = 1u,  /* a seq_lens entry outside [0, T_cap] (clamped) */
    JSSA_DEV_INDEX = 2u,   /* an index outside [0, T_b) or a count outside [0, k] (skipped) */
    JSSA_DEV_POS = 4u,     /* an append position outside [0, T_cap - n_new] (row skipped) */
    JSSA_DEV_TIMEOUT = 8u  /* a bounded on-chip wait gave up (the kernel returned early) */
};

typedef enum { JSSA_BF16 = 0, JSSA_FP32 = 1 } jssa_dtype;

/* How the G query heads of one KV head combine into one token score.  The
 * pages do not say; SUM (the default, the timed path) adds the subspace
 * logits of the group, MAX takes their maximum. */
typedef enum { JSSA_AGG_SUM = 0, JSSA_AGG_MAX = 1 } jssa_agg;

typedef enum {
    JSSA_OP_APPEND = 0,
    JSSA_OP_SCORE = 1,
    JSSA_OP_TOPK = 2,
    JSSA_OP_SELECT = 3,
    JSSA_OP_INDEXED_DECODE = 4,
    JSSA_OP_DENSE_DECODE = 5,
    JSSA_OP_GATHER_THEN_DENSE = 6,
    JSSA_OP_DECODE_STEP = 7,
    JSSA_OP_SELECT_HEADS = 8,        /* jssa_select_heads */
    JSSA_OP_INDEXED_DECODE_HEADS = 9, /* jssa_indexed_decode_heads */
    JSSA_OP_CALIBRATE = 10            /* jssa_calibrate_basis (k ignored) */
} jssa_op;

typedef struct {
    int32_t B, Hq, Hkv, d, dv, r, T_cap;
    int32_t kv_dtype; /* jssa_dtype of q, K, V, out */
    int32_t kt_dtype; /* jssa_dtype of Kt */
} jssa_dims;

/* Library version (JSSA_VERSION). */
JSSA_API int jssa_version(void);

/* Text for a JSSA_OK / JSSA_ERR_* code (static storage). */
JSSA_API const char *jssa_status_string(int status);

/* Message of the last failing call on this host thread (static per thread). */
JSSA_API const char *jssa_last_error(void);

/* Bytes of workspace `op` needs for these dims and k (k is ignored by ops
 * without a selection).  The size covers either aggregation, any sliding
 * window and every selection form and option (jssa_select_opts), and depends
 * on the current device's SM count.  Writes *bytes; returns a status. */
JSSA_API int jssa_workspace_size(const jssa_dims *dims, int k, int op, size_t *bytes);

/* How one call of `op` (JSSA_OP_*) with these dims, k and aggregation is
 * carried out on the current device: *launches = the kernels it enqueues
 * (the decode step is a single launch when its fused streaming form applies,
 * else three or four), and, when desc is not NULL, a NUL-terminated
 * description of the forms chosen (at most desc_len bytes written).  Host
 * planning only: nothing is enqueued.  The pages have no counterpart; this
 * is a measurement aid (launch counts of a timed region). */
JSSA_API int jssa_plan_info(const jssa_dims *dims, int k, int op, int agg, int *launches, char *desc,
                            size_t desc_len);

/* Zero `ws_bytes` bytes of workspace on `stream` (clears the status word and
 * the arrival counters).  Needed once per workspace before first use. */
JSSA_API int jssa_workspace_init(void *ws, size_t ws_bytes, jssa_stream_t stream);

/* Low-rank key append [ABS: shared low-dimensional query-key subspace; NEWS
 * Synopsis: candidate tokens are scored in that subspace].
 *   Kt[b,h,t,:] = round(sum_i K[b,t,h,i] * P[h,i,:])   (fp32 accumulation,
 *   one round-to-nearest-even into kt_dtype)
 * for t in [pos_begin[b], pos_begin[b] + n_new), every b and h.  pos_begin is
 * device int32 [B].  A row whose range leaves [0, T_cap) is skipped and sets
 * JSSA_DEV_POS.  n_new = 1 is the per-step append; n_new = T builds a prefix. */
JSSA_API int jssa_append_lowrank(const jssa_dims *dims, const void *K, const float *P, void *Kt,
                        const int32_t *pos_begin, int n_new, void *ws, size_t ws_bytes,
                        jssa_stream_t stream);

/* Subspace scores [NEWS Synopsis and Interpretation para 2: queries and keys
 * share one scoring space].  With qt_g = P_h^T q_g (fp32):
 *   SUM: scores[b,h,t] = (sum_g qt_g) . Kt[b,h,t,:]
 *   MAX: scores[b,h,t] = max_g qt_g . Kt[b,h,t,:]
 * for t < T_b (entries t >= T_b are not written).  fp32 arithmetic. */
JSSA_API int jssa_score(const jssa_dims *dims, const void *q, const float *P, const void *Kt,
               const int32_t *seq_lens, int agg, float *scores, void *ws, size_t ws_bytes,
               jssa_stream_t stream);

/* Per-(b, h) top-k [ABS: distinct per-KV-head selections; NEWS Synopsis]:
 * the k_b tokens t < T_b that come first under (scores desc, t asc); -0.0 and
 * +0.0 are one value; written in ascending t, -1 padded.  count may be NULL. */
JSSA_API int jssa_topk(const jssa_dims *dims, const float *scores, const int32_t *seq_lens, int k,
              int32_t *idx, int32_t *count, void *ws, size_t ws_bytes, jssa_stream_t stream);

/* jssa_score followed by jssa_topk in one pass over Kt, without writing the
 * score array.  Results are bit-identical to the two-call path (same fp32
 * scores, same order): the global top-k of a strict total order is the top-k
 * of the union of the per-chunk top-k sets. */
JSSA_API int jssa_select(const jssa_dims *dims, const void *q, const float *P, const void *Kt,
                const int32_t *seq_lens, int agg, int k, int32_t *idx, int32_t *count,
                void *ws, size_t ws_bytes, jssa_stream_t stream);

/* Selection forms (jssa_select_opts.form).  All give identical results. */
typedef enum {
    JSSA_FORM_AUTO = 0,    /* the library's choice for the shape */
    JSSA_FORM_CLUSTER = 1, /* one thread-block cluster per (b, h) (several waves allowed) */
    JSSA_FORM_STREAM = 2,  /* the warp-specialised streaming pass (SUM over the low-rank cache) */
    JSSA_FORM_SCAN = 3     /* the block-synchronous streaming pass */
} jssa_select_form;

/* Selection options.
 *  - n_sink, n_recent: tokens that are always selected.  A variant the pages
 *    do not describe (their selection is a pure top-k); the reading is the
 *    usual one of sparse decoders that keep "sink" tokens and a recent
 *    window.  With F = {t < n_sink} U {t >= T_b - n_recent} (t < T_b): if
 *    |F| >= k_b the selection is the k_b smallest indices of F, otherwise F
 *    plus the k_b - |F| best other tokens under (score desc, t asc).
 *  - form: a jssa_select_form; a forced form without a kernel for the shape
 *    falls back to the next one (cluster -> stream -> scan).
 *  - unfused: for jssa_decode_step_ex, nonzero keeps the step in separate
 *    launches (prologue, selection, attention) even where the one-launch
 *    fused form applies.
 *  - block_norms: exact block screening (a lossless cut of the low-rank
 *    stream; the method pages on DoSA-style screening describe the bound).
 *    NULL: off.  Else [B, Hkv, ceil(T_cap / JSSA_NORM_BLOCK)] fp32 upper
 *    bounds of ||Kt[b,h,t,:]|| over each block of JSSA_NORM_BLOCK tokens (see
 *    jssa_block_norms).  The streaming form then skips reading a tile of the
 *    low-rank cache when ||qbar|| times its blocks' bound (inflated by 1e-4
 *    to cover fp32 rounding) cannot beat the k-th best key its segment has
 *    already seen; the selection is bit-identical either way (other forms
 *    ignore the bound).  Tiles holding forced tokens are never skipped.  The
 *    decode step keeps the bound of the block of the appended row current
 *    (raised with an atomic max); an append made with jssa_append_lowrank
 *    needs jssa_block_norms afterwards.  Skipped tiles are counted in word 1
 *    of the workspace (uint32, cumulative; jssa_workspace_init clears it).
 * NULL or all zeros: plain top-k, automatic form, no screening. */
typedef struct {
    int32_t n_sink;     /* >= 0 */
    int32_t n_recent;   /* >= 0 */
    int32_t form;       /* jssa_select_form */
    int32_t unfused;    /* 0 or 1 */
    float *block_norms; /* screening bounds, or NULL */
} jssa_select_opts;

#define JSSA_NORM_BLOCK 128

/* Block norm bounds of the low-rank cache for screening: norms[b,h,j] = the
 * largest ||Kt[b,h,t,:]|| (fp32, from the stored values) over t in
 * [j*JSSA_NORM_BLOCK, min(T_cap, (j+1)*JSSA_NORM_BLOCK)), every row b.
 * norms: [B, Hkv, ceil(T_cap / JSSA_NORM_BLOCK)] fp32 device memory.  Only
 * B, Hkv, T_cap, r and kt_dtype of dims are read.  The pages have no API for
 * it; it is the screening variant's bookkeeping. */
JSSA_API int jssa_block_norms(const jssa_dims *dims, const void *Kt, float *norms, jssa_stream_t stream);

/* jssa_topk, jssa_select and jssa_decode_step with selection options (NULL
 * = the plain calls).  jssa_select_ex stays bit-identical to jssa_score +
 * jssa_topk_ex with the same options.  Errors: JSSA_ERR_INVALID_ARG for a
 * negative count. */
JSSA_API int jssa_topk_ex(const jssa_dims *dims, const float *scores, const int32_t *seq_lens, int k,
                 const jssa_select_opts *opts, int32_t *idx, int32_t *count, void *ws, size_t ws_bytes,
                 jssa_stream_t stream);
JSSA_API int jssa_select_ex(const jssa_dims *dims, const void *q, const float *P, const void *Kt,
                   const int32_t *seq_lens, int agg, int k, const jssa_select_opts *opts, int32_t *idx,
                   int32_t *count, void *ws, size_t ws_bytes, jssa_stream_t stream);

/* Gather-free indexed attention [ABS: token-level indexed-attention kernel
 * with distinct per-KV-head selections under the standard GQA cache layout;
 * NEWS Interpretation para 3: selected tokens are read in place through their
 * indices].  For every query head g of KV head h, over t in
 * idx[b,h,0:count[b,h]]:
 *   l_t = softmax_scale * q[b,g,:] . K[b,t,h,:]
 *   out[b,g,:] = sum_t softmax(l)_t * V[b,t,h,:],  lse[b,g] = ln sum_t e^{l_t}
 * fp32 accumulation, split over the index list, log-sum-exp combine.
 * count may be NULL (then the count is the number of leading non-negative
 * slots).  An empty set gives out = 0, lse = -inf.  An index outside [0, T_b)
 * is skipped and sets JSSA_DEV_INDEX.  lse may be NULL.
 * Latent form: the 128-token splits of a batch row merge inside the attention
 * kernel when all B * ceil(k / 128) of its CTAs fit on the device at once
 * (one per SM), else in a second kernel.  The in-kernel merge waits, bounded,
 * for the other splits of the batch row: if concurrent work on another stream
 * keeps SMs from the kernel for longer than the limit, the call completes with
 * JSSA_DEV_TIMEOUT in the status word and the affected rows undefined. */
JSSA_API int jssa_indexed_decode(const jssa_dims *dims, const void *q, const void *K, const void *V,
                        const int32_t *idx, const int32_t *count, int k,
                        const int32_t *seq_lens, float softmax_scale, void *out, float *lse,
                        void *ws, size_t ws_bytes, jssa_stream_t stream);

/* Full-KV decode attention (window = 0: t < T_b) or sliding-window decode
 * (window = W > 0: t in [max(0, T_b - W), T_b)), same arithmetic as above. */
JSSA_API int jssa_dense_decode(const jssa_dims *dims, const void *q, const void *K, const void *V,
                      const int32_t *seq_lens, int window, float softmax_scale, void *out,
                      float *lse, void *ws, size_t ws_bytes, jssa_stream_t stream);

/* The gather-then-dense comparison path [NEWS Interpretation para 3]: copy the
 * selected K and V rows into gather_buf (laid out [2][B, Hkv, k, d]; needs
 * 2*B*Hkv*k*d*sizeof(kv_dtype) bytes, 16-byte aligned), then run dense decode
 * over the contiguous rows.  Same results as jssa_indexed_decode. */
JSSA_API int jssa_gather_then_dense(const jssa_dims *dims, const void *q, const void *K, const void *V,
                           const int32_t *idx, const int32_t *count, int k,
                           const int32_t *seq_lens, float softmax_scale, void *gather_buf,
                           size_t gather_bytes, void *out, float *lse, void *ws,
                           size_t ws_bytes, jssa_stream_t stream);

/* One whole decode step: append the row at pos_begin[b] (n_new = 1), select
 * (score + top-k, fused), then indexed decode.  Equal to the three calls in a
 * row; idx and count receive the selection. */
JSSA_API int jssa_decode_step(const jssa_dims *dims, const void *q, const void *K, const void *V,
                     const float *P, void *Kt, const int32_t *seq_lens,
                     const int32_t *pos_begin, int k, int agg, float softmax_scale,
                     int32_t *idx, int32_t *count, void *out, float *lse, void *ws,
                     size_t ws_bytes, jssa_stream_t stream);

/* jssa_decode_step with selection options (NULL = jssa_decode_step). */
JSSA_API int jssa_decode_step_ex(const jssa_dims *dims, const void *q, const void *K, const void *V,
                        const float *P, void *Kt, const int32_t *seq_lens, const int32_t *pos_begin, int k,
                        int agg, float softmax_scale, const jssa_select_opts *opts, int32_t *idx,
                        int32_t *count, void *out, float *lse, void *ws, size_t ws_bytes,
                        jssa_stream_t stream);

/* Bytes of host input (and of the device staging buffer) that
 * jssa_decode_step_host takes: the queries [B, Hq, d], then the new token's
 * K rows [B, Hkv, d], then its V rows [B, Hkv, dv] (none for a latent
 * cache), packed back to back in kv_dtype. */
JSSA_API int jssa_host_step_bytes(const jssa_dims *dims, size_t *bytes);

/* One decode step driven from host memory: the call a serving loop makes per
 * token.  Enqueued on `stream`, in order:
 *   1. one host-to-device copy of in_host (jssa_host_step_bytes bytes, layout
 *      above) into the device buffer `stage` (same size, 16-byte aligned);
 *   2. the new K / V rows written into the cache at position pos_begin[b]
 *      (K[b, pos, :, :], V[b, pos, :, :]); a position outside [0, T_cap) is
 *      skipped and sets JSSA_DEV_POS;
 *   3. jssa_decode_step_ex with q = the staged queries (append of the
 *      low-rank row at pos_begin, selection, indexed attention) into the
 *      device buffers idx, count, out, lse;
 *   4. one device-to-host copy of out into out_host ([B, Hq, dv] kv_dtype).
 * in_host and out_host should be pinned (page-locked) host memory for the
 * copies to run asynchronously; the host must synchronise the stream before
 * reading out_host.  Other arguments and errors as jssa_decode_step_ex. */
JSSA_API int jssa_decode_step_host(const jssa_dims *dims, const void *in_host, void *stage, void *K, void *V,
                                   const float *P, void *Kt, const int32_t *seq_lens, const int32_t *pos_begin,
                                   int k, int agg, float softmax_scale, const jssa_select_opts *opts,
                                   int32_t *idx, int32_t *count, void *out, float *lse, void *out_host, void *ws,
                                   size_t ws_bytes, jssa_stream_t stream);

/* Calibration of the shared basis P from sampled queries and keys: the step
 * before the decode path [ABS: a spectral solution for the shared query-key
 * subspace; NEWS Interpretation para 2: queries and keys preserved jointly].
 * The pages give no objective or formula; the reading computed is, per KV
 * head h,
 *   S_q = sum of q q^T over the rows of q_cal [n_q, Hq, d] of the head's G
 *         query heads,   S_k = sum of k k^T over n_keys sampled tokens per
 *         batch row (t_j = floor(j * T_b / n_keys), j < n_keys; all t < T_b
 *         when T_b <= n_keys),
 *   M = S_q / tr(S_q) + S_k / tr(S_k)  (fp32),
 *   P_out[h] = an orthonormal basis of the dominant r-dimensional
 *              eigen-subspace of M, by `iters` rounds of subspace iteration
 *              X <- orth(M X) from P_init[h] (Gram-Schmidt applied twice).
 * P_init, P_out: [Hkv, d, r] fp32 (may not alias).  r <= 64; d in {64, 128,
 * 256}; GQA shapes.  Workspace: jssa_workspace_size(.., JSSA_OP_CALIBRATE). */
JSSA_API int jssa_calibrate_basis(const jssa_dims *dims, const void *q_cal, int n_q, const void *K,
                                  const int32_t *seq_lens, int n_keys, int iters, const float *P_init,
                                  float *P_out, void *ws, size_t ws_bytes, jssa_stream_t stream);

/* Per-query-head selection: a variant for measurement.  The method selects
 * one distinct token set per (batch, KV head), shared by the G query heads of
 * the KV head [ABS: distinct per-KV-head selections; NEWS Synopsis]; this
 * call gives every query head g its own set, so the two can be compared
 * (bytes of selected rows read, recall, output error):
 *   s[b,g,t] = (P_h^T q_g) . Kt[b,h,t,:]   (h = g / G, fp32, t < T_b)
 *   idx[b,g,:] = the k_b tokens that come first under (s desc, t asc),
 *                ascending, -1 padded;  count[b,g] = k_b   (count may be NULL)
 * idx is [B, Hq, k], count [B, Hq].  The selection runs in the cluster or the
 * block-synchronous form (opts->form JSSA_FORM_STREAM is taken as automatic).
 * GQA shapes only (not the latent form); G <= 16. */
JSSA_API int jssa_select_heads(const jssa_dims *dims, const void *q, const float *P, const void *Kt,
                               const int32_t *seq_lens, int k, const jssa_select_opts *opts, int32_t *idx,
                               int32_t *count, void *ws, size_t ws_bytes, jssa_stream_t stream);

/* Attention of each query head over its own token list (the companion of
 * jssa_select_heads): for query head g of KV head h = g / G, over t in
 * idx[b,g,0:count[b,g]] (idx [B, Hq, k], count [B, Hq] or NULL), the same
 * arithmetic as jssa_indexed_decode: rows read in place from the standard GQA
 * cache, fp32 online softmax, log-sum-exp combine of the splits.  Every
 * query head reads its own rows, so a KV head's rows are read up to G times.
 * GQA shapes only. */
JSSA_API int jssa_indexed_decode_heads(const jssa_dims *dims, const void *q, const void *K, const void *V,
                                       const int32_t *idx, const int32_t *count, int k,
                                       const int32_t *seq_lens, float softmax_scale, void *out, float *lse,
                                       void *ws, size_t ws_bytes, jssa_stream_t stream);

/* jssa_plan_info with selection options (NULL = jssa_plan_info): the forms
 * and launch count of a call made with these options. */
JSSA_API int jssa_plan_info_ex(const jssa_dims *dims, int k, int op, int agg, const jssa_select_opts *opts,
                               int *launches, char *desc, size_t desc_len);

/* Failure-detection self-check of the bounded on-chip waits.  The method
 * pages have no counterpart.  Every wait inside the library's kernels (on an
 * mbarrier phase, or on a device word other CTAs raise) is bounded: after a
 * wall-time limit (2 s in the path's kernels) it gives up, the kernel sets
 * JSSA_DEV_TIMEOUT in the status word, and it returns instead of trapping or
 * hanging.  This call runs those same wait routines, with limit_ns, in one
 * small kernel on a barrier and a word that nothing completes, so every wait
 * expires: afterwards the status word (word 0 of ws) holds JSSA_DEV_TIMEOUT
 * and the 32-bit word at byte 128 of ws holds 3, the number of waits that
 * gave up.  ws: device memory of at least 256 bytes, 16-byte aligned (bytes
 * 64..255 are cleared on `stream` first).  limit_ns in [1000, 1000000000].
 * The context stays usable. */
JSSA_API int jssa_check_wait_expiry(void *ws, size_t ws_bytes, uint64_t limit_ns, jssa_stream_t stream);

/* Allocation-free variant of jssa_indexed_decode.  The method pages have no
 * counterpart: this is an integration entry point of this library.
 *
 * Some callers cannot hand the library device scratch memory, because they
 * cannot allocate at call time: a serving engine whose allocator has already
 * reserved the GPU's memory for its KV-cache pool, a real-time decode loop
 * that cannot afford the implicit device synchronisation of cudaMalloc /
 * cudaFree, or a plugin host that forbids allocation inside its hooks.  This
 * entry point takes the same inputs and outputs as jssa_indexed_decode but no
 * workspace: its scratch (split partials, arrival counters, status word) is a
 * fixed 8 MiB array of device memory inside the library, which every GPU that
 * loads the library holds until the process exits.  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 *  - Shapes whose scratch would exceed 8 MiB are rejected with
 *    JSSA_ERR_WORKSPACE and a message (use jssa_indexed_decode then).
 *  - The first call on each device looks up the array's device address with
 *    that device current; make that first call before any stream capture.
 *    The address stays cached for the process: after cudaDeviceReset() on a
 *    device, unload and reload the library before calling this again.
 *  - Latent-cache shapes (d = 576, dv = 512, Hkv = 1, 128 heads) are served
 *    too, with their split partials in the same array.
 *  - Every call on a device shares the one array, which keeps the last call's
 *    contents.  The call clears the counters and the status word on `stream`
 *    before its kernel; calls whose execution overlaps on the GPU (other
 *    streams, concurrent threads) race on the array and must be serialised
 *    by the caller.
 *  - The device status word is not readable by the caller here; bad indices
 *    are still skipped as in jssa_indexed_decode.
 * Results equal those of jssa_indexed_decode on the same inputs. */
JSSA_API int jssa_indexed_decode_noalloc(const jssa_dims *dims, const void *q, const void *K,
                                         const void *V, const int32_t *idx, const int32_t *count,
                                         int k, const int32_t *seq_lens, float softmax_scale,
                                         void *out, float *lse, jssa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* JSSA_H */
