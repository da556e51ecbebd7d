// Low-rank key append and query projection.
//
// Append ("Joint Subspace Sparse Attention for Efficient Long-Context
// Decoding", Abstract: a shared low-dimensional query-key subspace; news item
// "JSSA makes token-level sparse decoding gather-free", Synopsis: candidate
// tokens are scored in that subspace):
//   Kt[b,h,t,:] = round(K[b,t,h,:] . P[h])   for t in [pos_b, pos_b + n_new).
// Projection (same pages, Interpretation para 2: queries and keys share the
// scoring space): qt_g = P_h^T q_g; the SUM score folds the group first,
// qbar_h = P_h^T (sum_g q_g), which is the same linear map applied once.
//
// Every dot product over d is evaluated in one fixed order, independent of
// the launch shape: partial sums over consecutive chunks of kChunk inputs
// (fma chains from 0), then the chunk partials added left to right.  So the
// per-step append, the prefix append and the fused decode-step prologue give
// bit-identical rows, and the score and select paths see the same qbar.
#include <cooperative_groups.h>

#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace cg = cooperative_groups;

namespace jssa {

namespace {

constexpr int kPrepThreads = 256;
constexpr int kPrepThreadsWide = 1024;  // latent rows: 128-head folds and 576-wide dot products

// Threads per CTA for a head width: wide rows get four times the threads.
inline int prep_threads(int d) { return d > 256 ? kPrepThreadsWide : kPrepThreads; }
constexpr int kChunk = 16;  // d is a multiple of 16 for every supported shape

// out[o] for o < n_out, with out[o] = sum_i x[row(o)][i] * P[i][col(o)], x in
// shared memory (fp32, rows of d), P global [d][r].  `part` is shared scratch
// of n_out * (d / kChunk) floats.
__device__ __forceinline__ void chunked_dots(const float *x, const float *__restrict__ P, int d, int r, int n_out,
                                             float *part) {
    const int nch = d / kChunk;
    // consecutive threads take consecutive outputs (columns of P): coalesced P reads
    for (int p = threadIdx.x; p < n_out * nch; p += blockDim.x) {
        const int c = p / n_out, o = p - c * n_out;
        const int row = o / r, j = o - row * r;
        const float *xr = x + (size_t)row * d + c * kChunk;
        const float *pc = P + (size_t)(c * kChunk) * r + j;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < kChunk; ++i) acc = fmaf(xr[i], __ldg(pc + (size_t)i * r), acc);
        part[(size_t)o * nch + c] = acc;
    }
    __syncthreads();
}

__device__ __forceinline__ float sum_chunks(const float *part, int o, int nch) {
    float s = part[(size_t)o * nch];
    for (int c = 1; c < nch; ++c) s += part[(size_t)o * nch + c];
    return s;
}

// Append rows [row0, row0 + nrows) of KV head bh's new range.
template <typename KV, typename KT>
__device__ void append_rows(const AppendArgs &a, int bh, int row0, int nrows, float *xs, float *part) {
    const int b = bh / a.Hkv, h = bh - b * a.Hkv;
    const int pos = a.pos_begin[b];
    if (pos < 0 || pos > a.T_cap - a.n_new) {
        if (threadIdx.x == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_POS);
        return;
    }
    const int d = a.d, r = a.r;
    const KV *K = static_cast<const KV *>(a.K);
    for (int p = threadIdx.x; p < nrows * d; p += blockDim.x) {
        const int rr = p / d, i = p - rr * d;
        const size_t t = (size_t)pos + row0 + rr;
        xs[p] = to_f32(K[(((size_t)b * a.T_cap + t) * a.Hkv + h) * d + i]);
    }
    __syncthreads();
    const float *P = a.P + (size_t)h * d * r;
    chunked_dots(xs, P, d, r, nrows * r, part);
    KT *Kt = static_cast<KT *>(a.Kt);
    const int nch = d / kChunk;
    for (int o = threadIdx.x; o < nrows * r; o += blockDim.x) {
        const int rr = o / r, j = o - rr * r;
        const size_t t = (size_t)pos + row0 + rr;
        store_elem(Kt + (((size_t)b * a.Hkv + h) * a.T_cap + t) * r + j, sum_chunks(part, o, nch));
    }
}

// Projected queries of KV head bh: SUM -> qproj[bh][0][:] = P_h^T sum_g q_g;
// MAX -> qproj[bh][g][:] = P_h^T q_g.
template <typename KV>
__device__ void project_bh(const ProjArgs &a, int bh, float *xs, float *part) {
    const int b = bh / a.Hkv, h = bh - b * a.Hkv;
    const int G = a.Hq / a.Hkv, d = a.d, r = a.r;
    const KV *q = static_cast<const KV *>(a.q) + ((size_t)b * a.Hq + (size_t)h * G) * d;
    const int nrow = a.agg == JSSA_AGG_SUM ? 1 : G;
    if (a.agg == JSSA_AGG_SUM) {
        // stage the group's queries in shared memory (every load in flight at
        // once), then sum over the group in head order
        KV *qsm = reinterpret_cast<KV *>(part + (size_t)r * (d / kChunk));
        const int nvec = G * d * (int)sizeof(KV) / 16;
        for (int v = threadIdx.x; v < nvec; v += blockDim.x) cp_async16(qsm + (size_t)v * (16 / sizeof(KV)), q + (size_t)v * (16 / sizeof(KV)), 16);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        for (int i = threadIdx.x; i < d; i += blockDim.x) {
            // head order kept; the loads of eight heads are issued together
            float s = 0.f;
            int g = 0;
            for (; g + 8 <= G; g += 8) {
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = to_f32(qsm[(size_t)(g + u) * d + i]);
#pragma unroll
                for (int u = 0; u < 8; ++u) s += v[u];
            }
            for (; g < G; ++g) s += to_f32(qsm[(size_t)g * d + i]);
            xs[i] = s;
        }
        __syncthreads();
    } else {
        for (int p = threadIdx.x; p < G * d; p += blockDim.x) xs[p] = to_f32(q[p]);
    }
    __syncthreads();
    chunked_dots(xs, a.P + (size_t)h * d * r, d, r, nrow * r, part);
    const int nch = d / kChunk;
    for (int o = threadIdx.x; o < nrow * r; o += blockDim.x)
        a.qproj[(size_t)bh * nrow * r + o] = sum_chunks(part, o, nch);
}

template <typename KV, typename KT>
__global__ void __launch_bounds__(kPrepThreadsWide) append_kernel(AppendArgs a) {
    extern __shared__ __align__(16) float sm_prep[];
    pdl_trigger();
    pdl_wait();
    const int bh = blockIdx.y;
    const int row0 = blockIdx.x * a.rows_per_cta;
    const int nrows = min(a.rows_per_cta, a.n_new - row0);
    if (nrows <= 0) return;
    append_rows<KV, KT>(a, bh, row0, nrows, sm_prep, sm_prep + (size_t)a.rows_per_cta * a.d);
}

template <typename KV>
__global__ void __launch_bounds__(kPrepThreadsWide) project_kernel(ProjArgs a) {
    extern __shared__ __align__(16) float sm_prep[];
    pdl_trigger();
    pdl_wait();
    const int G = a.Hq / a.Hkv;
    const int xrows = a.agg == JSSA_AGG_SUM ? 1 : G;
    project_bh<KV>(a, blockIdx.x, sm_prep, sm_prep + (size_t)xrows * a.d);
}

// Decode-step prologue: one CTA per (b, h) appends the new row and projects
// the queries; equal to append_kernel (n_new = 1) followed by project_kernel.
template <typename KV, typename KT>
__global__ void __launch_bounds__(kPrepThreadsWide) prep_kernel(AppendArgs ap, ProjArgs pj) {
    extern __shared__ __align__(16) float sm_prep[];
    pdl_trigger();
    pdl_wait();
    const int G = pj.Hq / pj.Hkv;
    const int xrows = pj.agg == JSSA_AGG_SUM ? 1 : G;
    float *xs = sm_prep;
    float *part = sm_prep + (size_t)xrows * pj.d;
    append_rows<KV, KT>(ap, blockIdx.x, 0, 1, xs, part);
    __syncthreads();
    project_bh<KV>(pj, blockIdx.x, xs, part);
}

// The same prologue (SUM aggregation) split over a cluster of kPrepCluster
// CTAs per (b, h): rank s takes the d-chunks s, s + C, ...; it stages its
// chunks of the group's queries and of P, folds the queries, and stores the
// chunk partials of the projection and of the new key row into rank 0's
// shared memory; rank 0 adds them in chunk order.  Every value is formed in
// the order prep_kernel uses, so the two give the same bits; the split puts
// many more loads in flight for wide rows (576-d latent rows, 128 heads).
constexpr int kPrepCluster = 8;
constexpr int kPrepClThreads = 256;

template <typename KV, typename KT>
__global__ void __launch_bounds__(kPrepClThreads) prep_cluster_kernel(AppendArgs ap, ProjArgs pj) {
    extern __shared__ __align__(16) float sm_pc[];
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
    const int bh = blockIdx.x / C;
    const int b = bh / pj.Hkv, h = bh - b * pj.Hkv;
    const int G = pj.Hq / pj.Hkv, d = pj.d, r = pj.r, nch = d / kChunk;
    const int cpr = (nch + C - 1) / C;                          // chunk slots per rank
    const int mine = rank < nch ? (nch - 1 - rank) / C + 1 : 0;  // chunks rank, rank + C, ...
    constexpr int EV = 16 / (int)sizeof(KV);                   // elements per 16-byte vector
    float *part_all = sm_pc;                                    // [2][nch][r]: projection, key row
    KV *qs = reinterpret_cast<KV *>(part_all + (size_t)2 * nch * r);  // [G][cpr * kChunk]
    float *ps = reinterpret_cast<float *>(qs + (size_t)G * cpr * kChunk);  // [cpr * kChunk][r]
    float *xq = ps + (size_t)cpr * kChunk * r;                  // folded query chunks
    float *xk = xq + cpr * kChunk;                              // new key row chunks
    pdl_trigger();
    pdl_wait();
    const int pos = ap.pos_begin[b];
    const bool app = pos >= 0 && pos <= ap.T_cap - 1;
    if (!app && rank == 0 && threadIdx.x == 0 && ap.status) atomicOr(ap.status, (uint32_t)JSSA_DEV_POS);
    // stage this rank's chunks of every head's query and of P_h
    const KV *q = static_cast<const KV *>(pj.q) + ((size_t)b * pj.Hq + (size_t)h * G) * d;
    constexpr int VPC = kChunk / EV;  // vectors per query chunk
    for (int v = threadIdx.x; v < G * mine * VPC; v += blockDim.x) {
        const int g = v / (mine * VPC), rem = v - g * mine * VPC, cl = rem / VPC, e = rem - cl * VPC;
        const int c = rank + cl * C;
        cp_async16(qs + ((size_t)g * cpr + cl) * kChunk + e * EV, q + (size_t)g * d + c * kChunk + e * EV, 16);
    }
    const float *Ph = pj.P + (size_t)h * d * r;
    const int pvr = r / 4;  // vectors per P row
    for (int v = threadIdx.x; v < mine * kChunk * pvr; v += blockDim.x) {
        const int row = v / pvr, e = v - row * pvr;
        const int cl = row / kChunk, i = row - cl * kChunk;
        cp_async16(ps + (size_t)row * r + e * 4, Ph + (size_t)((rank + cl * C) * kChunk + i) * r + e * 4, 16);
    }
    cp_async_commit();
    const KV *K = static_cast<const KV *>(ap.K);
    for (int i = threadIdx.x; i < mine * kChunk; i += blockDim.x) {
        const int cl = i / kChunk, c = rank + cl * C;
        xk[i] = app ? to_f32(K[(((size_t)b * ap.T_cap + pos) * ap.Hkv + h) * d + c * kChunk + (i - cl * kChunk)]) : 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();
    // fold over the group in head order (eight loads in flight at a time)
    for (int i = threadIdx.x; i < mine * kChunk; i += blockDim.x) {
        float sum = 0.f;
        int g = 0;
        for (; g + 8 <= G; g += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = to_f32(qs[(size_t)(g + u) * cpr * kChunk + i]);
#pragma unroll
            for (int u = 0; u < 8; ++u) sum += v[u];
        }
        for (; g < G; ++g) sum += to_f32(qs[(size_t)g * cpr * kChunk + i]);
        xq[i] = sum;
    }
    __syncthreads();
    // chunk partials (fma chain from 0 over the chunk) into rank 0's copy
    float *dst = cluster.map_shared_rank(part_all, 0);
    for (int p = threadIdx.x; p < 2 * mine * r; p += blockDim.x) {
        const int o = p / (mine * r), rem = p - o * mine * r, cl = rem / r, j = rem - cl * r;
        const float *x = (o ? xk : xq) + cl * kChunk;
        const float *pc = ps + (size_t)cl * kChunk * r + j;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < kChunk; ++i) acc = fmaf(x[i], pc[(size_t)i * r], acc);
        dst[((size_t)o * nch + rank + cl * C) * r + j] = acc;
    }
    cluster.sync();
    if (rank != 0) return;
    KT *Kt = static_cast<KT *>(ap.Kt);
    for (int t = threadIdx.x; t < 2 * r; t += blockDim.x) {
        const int o = t / r, j = t - o * r;
        const float *pp = part_all + (size_t)o * nch * r + j;
        float sum = pp[0];
        for (int c = 1; c < nch; ++c) sum += pp[(size_t)c * r];
        if (o == 0)
            pj.qproj[(size_t)bh * r + j] = sum;
        else if (app)
            store_elem(Kt + ((size_t)bh * ap.T_cap + pos) * r + j, sum);
    }
}

// The new token's K and V rows of each batch row, staged contiguously
// ([B, Hkv, d] then [B, Hkv, dv]), written into the cache at pos[b] (the
// host-buffer decode step).  A position outside [0, T_cap) is skipped and
// flagged.  16-byte copies; one CTA per batch row.
__global__ void __launch_bounds__(128) place_rows_kernel(const uint4 *k_new, const uint4 *v_new, uint4 *K, uint4 *V,
                                                         const int32_t *pos, int T_cap, int row_k16, int row_v16,
                                                         uint32_t *status) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x;
    const int p = pos[b];
    if (p < 0 || p >= T_cap) {
        if (threadIdx.x == 0 && status) atomicOr(status, (uint32_t)JSSA_DEV_POS);
        return;
    }
    for (int c = threadIdx.x; c < row_k16; c += blockDim.x)
        K[((size_t)b * T_cap + p) * row_k16 + c] = k_new[(size_t)b * row_k16 + c];
    if (V)
        for (int c = threadIdx.x; c < row_v16; c += blockDim.x)
            V[((size_t)b * T_cap + p) * row_v16 + c] = v_new[(size_t)b * row_v16 + c];
}

// ||row|| of r stored values (fp32 sum of squares of the exact stored values)
template <typename KT>
__device__ __forceinline__ float row_norm(const KT *row, int r, int lane) {
    float s = 0.f;
    for (int j = lane; j < r; j += 32) {
        const float v = to_f32(row[j]);
        s = fmaf(v, v, s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return sqrtf(s);
}

// One warp per block of JSSA_NORM_BLOCK tokens of a row.
template <typename KT>
__global__ void __launch_bounds__(256) block_norms_kernel(const KT *Kt, float *norms, int BH, int T_cap, int r,
                                                          int nblk) {
    pdl_trigger();
    pdl_wait();
    const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= (long long)BH * nblk) return;
    const int bh = (int)(w / nblk), j = (int)(w - (long long)bh * nblk);
    const int t1 = min(T_cap, (j + 1) * JSSA_NORM_BLOCK);
    float m = 0.f;
    for (int t = j * JSSA_NORM_BLOCK; t < t1; ++t) m = fmaxf(m, row_norm(Kt + ((size_t)bh * T_cap + t) * r, r, lane));
    if (lane == 0) norms[w] = m;
}

// One warp per (b,h): the bound of the block holding the row at pos[b] is
// raised to cover the row (an atomic max on the non-negative float's bits).
template <typename KT>
__global__ void __launch_bounds__(256) norm_raise_kernel(const KT *Kt, float *norms, const int32_t *pos, int B,
                                                         int Hkv, int T_cap, int r, int nblk) {
    pdl_trigger();
    pdl_wait();
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (w >= B * Hkv) return;
    const int p = pos[w / Hkv];
    if (p < 0 || p >= T_cap) return;
    const float n = row_norm(Kt + ((size_t)w * T_cap + p) * r, r, lane);
    if (lane == 0) atomicMax(reinterpret_cast<int *>(norms + (size_t)w * nblk + p / JSSA_NORM_BLOCK), __float_as_int(n));
}

size_t prep_smem(int rows, int d, int r) {
    return ((size_t)rows * d + (size_t)rows * r * (d / kChunk)) * sizeof(float);
}

template <typename Kern>
cudaError_t allow_smem(Kern k, size_t smem) {
    return ensure_smem(reinterpret_cast<const void *>(k), smem);
}

}  // namespace

cudaError_t launch_append(const AppendArgs &a0, cudaStream_t s, bool pdl, int kv_dtype, int kt_dtype) {
    AppendArgs a = a0;
    // rows per CTA: as many as keep the staging under ~96 KiB
    int rows = 32;
    while (rows > 1 && prep_smem(rows, a.d, a.r) > 96 * 1024) rows >>= 1;
    if (rows > a.n_new) rows = a.n_new;
    a.rows_per_cta = rows;
    const size_t smem = prep_smem(rows, a.d, a.r);
    dim3 grid((a.n_new + rows - 1) / rows, a.B * a.Hkv);
    void (*k)(AppendArgs);
    if (kv_dtype == JSSA_BF16)
        k = kt_dtype == JSSA_BF16 ? append_kernel<__nv_bfloat16, __nv_bfloat16> : append_kernel<__nv_bfloat16, float>;
    else
        k = kt_dtype == JSSA_BF16 ? append_kernel<float, __nv_bfloat16> : append_kernel<float, float>;
    cudaError_t e = allow_smem(k, smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(k, grid, dim3(prep_threads(a.d)), smem, s, pdl, a);
}

cudaError_t launch_block_norms(const void *Kt, int kt_dtype, float *norms, int BH, int T_cap, int r,
                               cudaStream_t s, bool pdl) {
    const int nblk = (T_cap + JSSA_NORM_BLOCK - 1) / JSSA_NORM_BLOCK;
    const long long warps = (long long)BH * nblk;
    const dim3 grid((unsigned)((warps + 7) / 8));
    if (kt_dtype == JSSA_BF16)
        return launch_kernel(block_norms_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, pdl,
                             static_cast<const __nv_bfloat16 *>(Kt), norms, BH, T_cap, r, nblk);
    return launch_kernel(block_norms_kernel<float>, grid, dim3(256), 0, s, pdl, static_cast<const float *>(Kt), norms,
                         BH, T_cap, r, nblk);
}

cudaError_t launch_norm_raise(const void *Kt, int kt_dtype, float *norms, const int32_t *pos, int B, int Hkv,
                              int T_cap, int r, cudaStream_t s, bool pdl) {
    const int nblk = (T_cap + JSSA_NORM_BLOCK - 1) / JSSA_NORM_BLOCK;
    const dim3 grid((unsigned)((B * Hkv + 7) / 8));
    if (kt_dtype == JSSA_BF16)
        return launch_kernel(norm_raise_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, pdl,
                             static_cast<const __nv_bfloat16 *>(Kt), norms, pos, B, Hkv, T_cap, r, nblk);
    return launch_kernel(norm_raise_kernel<float>, grid, dim3(256), 0, s, pdl, static_cast<const float *>(Kt), norms,
                         pos, B, Hkv, T_cap, r, nblk);
}

cudaError_t launch_place_rows(const void *k_new, const void *v_new, void *K, void *V, const int32_t *pos, int B,
                              int T_cap, size_t row_k_bytes, size_t row_v_bytes, uint32_t *status, cudaStream_t s,
                              bool pdl) {
    return launch_kernel(place_rows_kernel, dim3(B), dim3(128), 0, s, pdl, static_cast<const uint4 *>(k_new),
                         static_cast<const uint4 *>(v_new), static_cast<uint4 *>(K), static_cast<uint4 *>(V), pos,
                         T_cap, (int)(row_k_bytes / 16), (int)(row_v_bytes / 16), status);
}

cudaError_t launch_project(const ProjArgs &a, cudaStream_t s, bool pdl, int kv_dtype) {
    const int G = a.Hq / a.Hkv;
    const int nrow = a.agg == JSSA_AGG_SUM ? 1 : G;
    const size_t es = kv_dtype == JSSA_BF16 ? 2 : 4;
    const size_t stage = a.agg == JSSA_AGG_SUM ? (size_t)G * a.d * es : 0;
    const size_t smem = ((size_t)nrow * a.d + (size_t)nrow * a.r * (a.d / kChunk)) * sizeof(float) + stage;
    void (*k)(ProjArgs) = kv_dtype == JSSA_BF16 ? project_kernel<__nv_bfloat16> : project_kernel<float>;
    cudaError_t e = allow_smem(k, smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(k, dim3(a.B * a.Hkv), dim3(prep_threads(a.d)), smem, s, pdl, a);
}

cudaError_t launch_prep(const AppendArgs &ap0, const ProjArgs &pj, cudaStream_t s, bool pdl, int kv_dtype,
                        int kt_dtype) {
    AppendArgs ap = ap0;
    ap.n_new = 1;
    ap.rows_per_cta = 1;
    if (pj.agg == JSSA_AGG_SUM && pj.r % 4 == 0) {
        const int G = pj.Hq / pj.Hkv, nch = pj.d / kChunk, cpr = (nch + kPrepCluster - 1) / kPrepCluster;
        const size_t es = kv_dtype == JSSA_BF16 ? 2 : 4;
        const size_t smem = (size_t)2 * nch * pj.r * 4 + (size_t)G * cpr * kChunk * es +
                            (size_t)cpr * kChunk * pj.r * 4 + (size_t)2 * cpr * kChunk * 4;
        void (*k)(AppendArgs, ProjArgs);
        if (kv_dtype == JSSA_BF16)
            k = kt_dtype == JSSA_BF16 ? prep_cluster_kernel<__nv_bfloat16, __nv_bfloat16>
                                      : prep_cluster_kernel<__nv_bfloat16, float>;
        else
            k = kt_dtype == JSSA_BF16 ? prep_cluster_kernel<float, __nv_bfloat16> : prep_cluster_kernel<float, float>;
        cudaError_t e = allow_smem(k, smem);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(pj.B * pj.Hkv * kPrepCluster);
        cfg.blockDim = dim3(kPrepClThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[2];
        int na = 0;
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = kPrepCluster;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
        if (pdl) {
            attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[na].val.programmaticStreamSerializationAllowed = 1;
            ++na;
        }
        cfg.attrs = attr;
        cfg.numAttrs = na;
        {
            cudaError_t es = ensure_smem(reinterpret_cast<const void *>(k), cfg.dynamicSmemBytes);
            if (es != cudaSuccess) return es;
        }
        return cudaLaunchKernelEx(&cfg, k, ap, pj);
    }
    const int G = pj.Hq / pj.Hkv;
    const int nrow = pj.agg == JSSA_AGG_SUM ? 1 : G;
    size_t xs = (size_t)nrow * pj.d;
    size_t part = (size_t)(nrow > 1 ? nrow : 1) * pj.r * (pj.d / kChunk);
    const size_t es = kv_dtype == JSSA_BF16 ? 2 : 4;
    const size_t stage = pj.agg == JSSA_AGG_SUM ? (size_t)G * pj.d * es : 0;
    const size_t smem = (xs + part) * sizeof(float) + stage;
    void (*k)(AppendArgs, ProjArgs);
    if (kv_dtype == JSSA_BF16)
        k = kt_dtype == JSSA_BF16 ? prep_kernel<__nv_bfloat16, __nv_bfloat16> : prep_kernel<__nv_bfloat16, float>;
    else
        k = kt_dtype == JSSA_BF16 ? prep_kernel<float, __nv_bfloat16> : prep_kernel<float, float>;
    cudaError_t e = allow_smem(k, smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(k, dim3(pj.B * pj.Hkv), dim3(prep_threads(pj.d)), smem, s, pdl, ap, pj);
}

}  // namespace jssa
