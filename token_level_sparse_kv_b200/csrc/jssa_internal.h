// Host-side plans, kernel argument blocks and launcher declarations shared
// by the translation units of libjssa.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/jssa.h"

namespace jssa {

constexpr int kMaxK = 2048;
constexpr int kMaxG = 16;
constexpr int kScanThreads = 256;
constexpr int kScanStageBytes = 16384;
constexpr int kScoreTileTokens = 2048;  // tokens per tile when the source is a score array
constexpr int kAttnThreads = 128;

// ------------------------------------------------------------------ scan ---
// One persistent pass over per-(b,h) token streams.  Source: the low-rank key
// cache (scores computed on the fly) or a score array.  Mode: write the scores,
// or keep a per-segment top-k and merge segments into the final selection.
enum ScanSrc { SRC_KT_BF16 = 0, SRC_KT_FP32 = 1, SRC_SCORES = 2 };
enum ScanMode { MODE_WRITE = 0, MODE_SELECT = 1 };

struct ScanArgs {
    const void *src;          // Kt [B,Hkv,T_cap,r] or scores [B,Hkv,T_cap]
    const float *qproj;       // [B*Hkv, nq, r] projected (folded) queries
    const int32_t *seq_lens;  // [B]
    float *scores_out;        // MODE_WRITE
    uint32_t *cand_key;       // [BH, max_seg, k]
    int32_t *cand_idx;        // [BH, max_seg, k]
    int32_t *cand_cnt;        // [BH, max_seg]
    uint32_t *counters;       // [BH] arrival tickets (self-resetting)
    int32_t *idx_out;         // [BH, k]
    int32_t *count_out;       // [BH] or null
    uint32_t *status;
    int B, Hkv, T_cap, r, nq, k;
    int tile_tokens, tiles_per_bh;
    long long total_tiles;
    int grid, max_seg, cap, nstages;
    int n_sink, n_recent;  // always-selected tokens (0, 0: plain top-k)
    int src_div;           // selection row bh reads source row bh / src_div (0 or 1: the same row)
    float *norms;          // screening: [BH, norm_blocks] block norm bounds, or null (streaming form)
    int norm_blocks;       // blocks of JSSA_NORM_BLOCK tokens per row
    int nb_cap;            // streaming form: tile bounds staged in shared memory per CTA (plan)
    uint32_t *skip_count;  // screening: tiles skipped (cumulative)
};

struct ScanPlan {
    int src, mode, tile_tokens, tiles_per_bh, grid, max_seg, cap, nstages;
    int nb_cap;  // streaming form: tile bounds a CTA stages in shared memory for screening
    long long total_tiles;
    size_t smem;
};

struct ProjArgs {
    const void *q;   // [B, Hq, d] kv dtype
    const float *P;  // [Hkv, d, r]
    float *qproj;    // [B*Hkv, nq, r]
    int B, Hq, Hkv, d, r, agg;
};

struct AppendArgs {
    const void *K;  // [B, T_cap, Hkv, d]
    const float *P;
    void *Kt;       // [B, Hkv, T_cap, r]
    const int32_t *pos_begin;
    uint32_t *status;
    int B, T_cap, Hkv, d, r, n_new, rows_per_cta;
};

// ---------------------------------------------------------------- attend ---
enum AttnSrc { ATT_INDEXED = 0, ATT_RANGE = 1, ATT_RANGE_BH = 2 };

struct AttnArgs {
    const void *q;  // [B, Hq, d]
    const void *K;
    const void *V;
    long long k_sb, k_st, k_sh;  // element strides of K: batch, token, head
    long long v_sb, v_st, v_sh;
    const int32_t *idx;      // ATT_INDEXED: [BH, k]
    const int32_t *count;    // ATT_INDEXED / ATT_RANGE_BH: [BH] (indexed: may be null)
    const int32_t *seq_lens; // [B]
    int k, window;
    int B, Hq, Hkv, G, T_cap;
    float scale_log2;        // softmax_scale * log2(e)
    int splits, pos_per_split;
    float *part_o;           // [BH, splits, G, D]
    float *part_ml;          // [BH, splits, G, 2]
    uint32_t *counters;      // [BH]
    void *out;               // [B, Hq, D]
    float *lse;              // [B, Hq] or null
    uint32_t *status;
    int head_div;            // row head h reads K/V head h / head_div (0 or 1: head h)
};

struct AttnPlan {
    int nt, splits, pos_per_split, stages;
    size_t smem;
};

struct GatherArgs {
    const void *K;
    const void *V;
    const int32_t *idx;
    const int32_t *count;
    const int32_t *seq_lens;
    void *gK;  // [B, Hkv, k, d]
    void *gV;  // null with V null (latent cache: the rows are gathered once)
    int32_t *gcount;  // [BH] rows actually gathered
    uint32_t *status;
    int B, Hkv, T_cap, d, k;
};

// ----------------------------------------------------- dense (tensor core) ---
// Dense attention of bf16 rows over a contiguous token range per (b, h): the
// cache ([B, T_cap, Hkv, d], rows [max(0, T_b - window), T_b) or [0, T_b))
// or a gathered buffer ([B*Hkv, k, d], rows [0, count[bh])).
struct DenseArgs {
    const void *q;            // [B, Hq, d] bf16
    const int32_t *seq_lens;  // [B]
    const int32_t *count;     // gathered source: rows per (b,h); null for the cache
    int B, Hq, Hkv, G, T_cap, window, k;
    int row_tiles;            // plan: 64-token tiles per row
    long long total_tiles;    // plan: rows * row_tiles
    int grid, part_stride;    // plan: persistent CTAs; partial slots per row
    int row_split;            // plan: > 0 = each row split into row_split parts, one CTA each (short problems)
    float scale_log2;         // softmax_scale * log2(e)
    float *part_o;            // [BH, part_stride, G, d]
    float *part_ml;           // [BH, part_stride, G, 2]
    uint32_t *counters;       // [BH] arrival tickets (self-resetting)
    void *out;                // [B, Hq, d] bf16
    float *lse;               // [B, Hq] or null
    uint32_t *status;
};
struct DensePlan {
    int row_tiles, grid, part_stride, row_split;
    long long total_tiles;
    size_t smem;
};
int dense_part_stride(int B, int Hkv);
// cudaErrorNotSupported where it has no kernel (d outside {64, 128, 256}).
cudaError_t plan_dense(int d, int B, int Hkv, int row_len, DensePlan *p);
cudaError_t launch_dense(const DensePlan &p, const DenseArgs &a, const void *K, const void *V, int d,
                         cudaStream_t s, bool pdl);

// ----------------------------------------------------------- calibration ---
struct CalibArgs {
    const void *q;            // [Nq, Hq, d] calibration queries (kv dtype)
    const void *K;            // [B, T_cap, Hkv, d]
    const int32_t *seq_lens;  // [B]
    int B, Hq, Hkv, T_cap, Nq, n_keys, chunks, r, iters;
    const float *P_init;      // [Hkv, d, r] start of the subspace iteration
    float *P_out;             // [Hkv, d, r]
    float *Sk;                // [Hkv, chunks, d, d] partial key sums
    float *Sq;                // [Hkv, d, d] query sums
    float *M;                 // [Hkv, d, d] the joint matrix
    uint32_t *status;
};
int calib_chunks(int Hkv);
cudaError_t launch_calib(const CalibArgs &a, int kv_dtype, int d, cudaStream_t s);

// ------------------------------------------- latent cache, token range ---
// Attention of the 128 heads of a latent cache over [0, T_b) of the cache
// ([B, T_cap, 1, 576]) or [0, count[b]) of a gathered buffer ([B, k, 576]).
struct MlaRangeArgs {
    const void *q;            // [B, 128, 576] bf16
    const int32_t *seq_lens;  // [B]
    const int32_t *count;     // gathered source: rows per batch row; null for the cache
    int B, T_cap, k;
    int row_tiles, splits;    // plan: 128-token tiles per row; CTAs (x 2 head halves) per row
    float scale_log2;
    __nv_bfloat16 *part_o;    // [B, splits, 128, 512] bf16 (unnormalised O of each split)
    float *part_ml;           // [B, splits, 128, 2]
    void *out;                // [B, 128, 512] bf16
    float *lse;               // [B, 128] or null
    uint32_t *status;
};
struct MlaRangePlan {
    int row_tiles, splits;
    size_t smem;
};
cudaError_t plan_mla_range(int B, int row_len, MlaRangePlan *p);
cudaError_t launch_mla_range(const MlaRangePlan &p, const MlaRangeArgs &a, const void *K, cudaStream_t s, bool pdl);

// --------------------------------------------------------- cluster select ---
// Top-k of one (b,h) by a cluster of CTAs holding the keys in shared memory.
struct CSelArgs {
    const void *src;          // Kt [B,Hkv,T_cap,r] or scores [B,Hkv,T_cap]
    const float *qproj;       // [B*Hkv, nq, r]
    const int32_t *seq_lens;  // [B]
    int32_t *idx_out;         // [BH, k]
    int32_t *count_out;       // [BH] or null
    uint32_t *status;
    int B, Hkv, T_cap, r, nq, k, csize, slice, nstages;
    int n_sink, n_recent;  // always-selected tokens (0, 0: plain top-k)
    int src_div;           // selection row bh reads source row bh / src_div (0 or 1: the same row)
};
struct CSelPlan {
    int csize, slice, grid_y, nstages;
    size_t smem;
};
// form: jssa_select_form (JSSA_FORM_CLUSTER relaxes the one-wave condition;
// JSSA_FORM_STREAM / JSSA_FORM_SCAN give cudaErrorNotSupported).
cudaError_t plan_csel(int form, int src, int agg, int B, int Hkv, int T_cap, int r, int nq, int k, CSelPlan *p);
cudaError_t launch_csel(const CSelPlan &p, const CSelArgs &a, int src, int agg, cudaStream_t s, bool pdl);

// ------------------------------------------------------------------- MLA ---
// Latent-cache attention: 128 query heads, 576-wide latent rows, the value is
// the first 512 columns of the row.
struct MlaArgs {
    const void *q;            // [B, 128, 576] bf16
    const void *K;            // [B, T_cap, 1, 576] bf16 (also the values)
    const int32_t *idx;       // [B, k] selected tokens (indexed form)
    const int32_t *count;     // [B] or null
    const int32_t *seq_lens;  // [B]
    int k, T_cap, B;
    float scale_log2;
    int splits;               // CTAs per batch row (128 tokens each)
    __nv_bfloat16 *part_o;    // [B, splits, 128, 512] bf16 (unnormalised O of each split)
    float *part_ml;           // [B, splits, 128, 2]
    void *out;                // [B, 128, 512] bf16
    float *lse;               // [B, 128] or null
    uint32_t *status;
    uint32_t *ctr;            // [2 B] arrival / done counters of the in-kernel merge (self-resetting, start at 0)
    int inline_combine;       // set by launch_mla: the splits merge inside the kernel
};
int mla_splits(int npos);
// true when the splits of a latent-cache indexed decode merge inside its kernel
// (every CTA of the grid resident at once) rather than in a second kernel
bool mla_inline_combine(int splits, int B);
cudaError_t launch_mla(const MlaArgs &a, bool indexed, cudaStream_t s, bool pdl);
// Log-sum-exp merge of a.splits latent-cache partials into out / lse.
cudaError_t launch_mla_combine(const MlaArgs &a, cudaStream_t s, bool pdl);

// --------------------------------------------------------------- helpers ---
// A TMA tensor map over bf16 data (cuTensorMapEncodeTiled, looked up once
// through the runtime: no link-time dependency on the driver library): rank
// dims (innermost first), rank-1 byte strides, box extents; 128-byte
// swizzle, 256-byte L2 promotion, zero fill outside the tensor.
// cudaErrorNotSupported when the driver offers no encoder.
cudaError_t encode_tiled_bf16(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                              const cuuint64_t *strides, const cuuint32_t *box);
bool tensor_maps_available();
int device_sm_count();
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and device
// (launch paths call it on every launch; the runtime call is made only when
// the requested size grows).
cudaError_t ensure_smem(const void *kern, size_t smem);
cudaError_t launch_project(const ProjArgs &a, cudaStream_t s, bool pdl, int kv_dtype);
// Block norm bounds of the low-rank cache (jssa_block_norms), and the raise of
// the bound of the block holding each row's appended row at pos[b].
cudaError_t launch_block_norms(const void *Kt, int kt_dtype, float *norms, int BH, int T_cap, int r,
                               cudaStream_t s, bool pdl);
cudaError_t launch_norm_raise(const void *Kt, int kt_dtype, float *norms, const int32_t *pos, int B, int Hkv,
                              int T_cap, int r, cudaStream_t s, bool pdl);
// Write each batch row's new K row (row_k_bytes, all KV heads) and V row into
// the cache at position pos[b]; v_new / V null for a latent cache.
cudaError_t launch_place_rows(const void *k_new, const void *v_new, void *K, void *V, const int32_t *pos, int B,
                              int T_cap, size_t row_k_bytes, size_t row_v_bytes, uint32_t *status, cudaStream_t s,
                              bool pdl);
cudaError_t launch_append(const AppendArgs &a, cudaStream_t s, bool pdl, int kv_dtype, int kt_dtype);
cudaError_t launch_prep(const AppendArgs &ap, const ProjArgs &pj, cudaStream_t s, bool pdl, int kv_dtype,
                        int kt_dtype);
cudaError_t plan_scan(int src, int mode, int agg, int B, int Hkv, int T_cap, int r, int nq, int k, ScanPlan *p);
cudaError_t launch_scan(const ScanPlan &p, const ScanArgs &a, int agg, cudaStream_t s, bool pdl);
// Warp-specialised streaming select (SUM over the low-rank key cache):
// cudaErrorNotSupported where it has no kernel.
cudaError_t plan_stream(int src, int agg, int B, int Hkv, int T_cap, int r, int k, ScanPlan *p);
cudaError_t launch_stream(const ScanPlan &p, const ScanArgs &a, cudaStream_t s, bool pdl);

// The whole decode step in the streaming kernel: the new row of the low-rank
// cache and the folded query are computed in its prologue, the attention of
// each (b,h) by the CTA that completes its selection, in its epilogue.
struct StepExtra {
    const void *q;            // [B, Hq, d] bf16
    const float *P;           // [Hkv, d, r]
    const void *K;            // [B, T_cap, Hkv, d] bf16
    const void *V;            // [B, T_cap, Hkv, d] bf16
    const int32_t *pos_begin; // [B] position of the appended token
    void *out;                // [B, Hq, d] bf16
    float *lse;               // [B, Hq] or null
    float scale_log2;         // softmax_scale * log2(e)
    int Hq, G, d;
};
// Fused plan for this shape (bf16 K/V and low-rank cache, SUM, d in {128, 256},
// r in {32, 64}, G a power of two <= 16); cudaErrorNotSupported otherwise.
cudaError_t plan_step_fused(int B, int Hkv, int Hq, int d, int T_cap, int r, int k, ScanPlan *p);
cudaError_t launch_step_fused(const ScanPlan &p, const ScanArgs &a, const StepExtra &x, cudaStream_t s, bool pdl);
cudaError_t plan_attend(int src, int kv_dtype, int d, int G, int B, int Hkv, int npos, AttnPlan *p);
cudaError_t launch_attend(const AttnPlan &p, int src, const AttnArgs &a, int kv_dtype, int d, cudaStream_t s,
                          bool pdl);
cudaError_t launch_gather(const GatherArgs &a, int kv_dtype, cudaStream_t s, bool pdl);

// Failure-detection self-check (jssa_check_wait_expiry): the bounded waits on
// a barrier and a flag that nothing completes; ws holds the status word at
// byte 0, the flag at byte 64 and the count of expired waits at byte 128.
cudaError_t launch_wait_expiry(void *ws, uint64_t limit_ns, cudaStream_t s);

// Launch with the programmatic-stream-serialisation attribute (PDL) if asked.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                          Args &&...args) {
    // planning of other shapes may have set the attribute for this kernel;
    // it only ever grows, so one check per launch keeps it sufficient
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace jssa
