// Subspace scoring and per-(batch, KV head) top-k selection.
//
// Method: news item "JSSA makes token-level sparse decoding gather-free",
// Synopsis (tokens scored in a shared low-dimensional query-key subspace, a
// distinct selected token set per KV head) and Interpretation para 2; "Joint
// Subspace Sparse Attention for Efficient Long-Context Decoding", Abstract
// (distinct per-KV-head selections).
//
// One persistent kernel streams token tiles of every (b, h):
//  * work = the flattened list of (b,h, tile) tiles; CTA i takes the
//    contiguous range [i*N/grid, (i+1)*N/grid), so the load is balanced to
//    one tile whatever B*Hkv is.  A range crosses at most a few (b,h)
//    boundaries; each (b,h) piece of it is a "segment".
//  * low-rank key tiles (16 KiB) arrive through a ring of bulk asynchronous
//    copies (TMA engine, mbarrier completion, evict-first L2 hint); lanes
//    groups of r*es/16 threads reduce one token's dot product with warp
//    shuffles.  The score array source (jssa_topk) is read with plain loads.
//  * MODE_WRITE stores the fp32 scores.  MODE_SELECT keeps a running top-k
//    of the segment in shared memory: a token survives only if its key beats
//    the current k-th key, survivors are appended in token order, and when
//    the buffer fills a radix select (4 passes of 8 bits over order-
//    preserving uint32 keys) keeps the best k, ties to the lower index.  The
//    segment's k candidates go to the workspace; the last CTA to finish a
//    (b,h) (arrival ticket, no waiting) merges its segments with the same
//    machinery and writes the ascending index list.
// Because the order (score desc, index asc) is a strict total order, the top-k
// of the union of per-segment top-k sets is the global top-k: the fused path
// returns exactly what jssa_score + jssa_topk return.
#include <type_traits>

#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace jssa {

namespace {

constexpr int NT = kScanThreads;

struct ScanSmem {
    size_t stages, bars, tkey, tidx, qs, buf_key, buf_idx, res_key, res_idx, hist, tmp, misc, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline ScanSmem scan_smem(int src, int mode, int r, int nstages, int cap, int k,
                                              int tile) {
    ScanSmem L;
    size_t o = 0;
    const bool from_kt = src != SRC_SCORES;
    L.stages = o;
    o += from_kt ? (size_t)nstages * kScanStageBytes : 0;
    L.bars = o;
    o = align_up(o + (from_kt ? (size_t)nstages * 8 : 0), 16);
    L.tkey = o;
    o = align_up(o + (size_t)tile * 4, 16);
    L.tidx = o;
    o = align_up(o + (mode == MODE_SELECT ? (size_t)tile * 4 : 0), 16);
    L.qs = o;
    o = align_up(o + (from_kt ? (size_t)kMaxG * r * 4 : 0), 16);
    const bool sel = mode == MODE_SELECT;
    L.buf_key = o;
    o = align_up(o + (sel ? (size_t)cap * 4 : 0), 16);
    L.buf_idx = o;
    o = align_up(o + (sel ? (size_t)cap * 4 : 0), 16);
    L.res_key = o;
    o = align_up(o + (sel ? (size_t)k * 4 : 0), 16);
    L.res_idx = o;
    o = align_up(o + (sel ? (size_t)k * 4 : 0), 16);
    L.hist = o;
    o = align_up(o + 256 * 4, 16);
    L.tmp = o;
    o = align_up(o + 32 * 4, 16);
    L.misc = o;
    o = align_up(o + 16 * 4, 128);
    L.total = o;
    return L;
}

// Shared state of the running top-k buffer (all values uniform across the block).
struct TopK {
    uint32_t *key;
    int32_t *idx;
    uint32_t *res_key;
    int32_t *res_idx;
    uint32_t *hist;
    int *tmp;
    int *misc;
    int n;          // entries in the buffer
    bool valid;     // thresh holds the k-th best key of a full reduction
    uint32_t thresh;
};

// kk-th largest key among keys[0..n) (1 <= kk <= n): returns the key value and
// how many entries equal to it belong to the top kk.
__device__ void radix_select(const uint32_t *keys, int n, int kk, TopK &tk, uint32_t &tau, int &need) {
    const int tid = threadIdx.x;
    uint32_t prefix = 0u, mask = 0u;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        tk.hist[tid] = 0u;
        __syncthreads();
        for (int j = tid; j < n; j += NT) {
            const uint32_t u = keys[j];
            if ((u & mask) == prefix) atomicAdd(&tk.hist[(u >> shift) & 0xffu], 1u);
        }
        __syncthreads();
        const int c = (int)tk.hist[255 - tid];
        int tot;
        const int ex = block_excl_scan<NT>(c, tk.tmp, tot);
        if (ex < kk && ex + c >= kk) {
            tk.misc[0] = 255 - tid;
            tk.misc[1] = ex;
        }
        __syncthreads();
        prefix |= (uint32_t)tk.misc[0] << shift;
        mask |= 0xffu << shift;
        kk -= tk.misc[1];
        __syncthreads();
    }
    tau = prefix;
    need = kk;
}

// Keep the best k of the buffer (requires tk.n > k), stable in buffer order.
__device__ void reduce_topk(TopK &tk, int k) {
    const int tid = threadIdx.x;
    uint32_t tau;
    int need;
    radix_select(tk.key, tk.n, k, tk, tau, need);
    const int per = (tk.n + NT - 1) / NT;
    const int j0 = min(tid * per, tk.n), j1 = min(j0 + per, tk.n);
    int ceq = 0;
    for (int j = j0; j < j1; ++j) ceq += tk.key[j] == tau;
    int tot;
    const int eq0 = block_excl_scan<NT>(ceq, tk.tmp, tot);
    int ckeep = 0;
    {
        int e = eq0;
        for (int j = j0; j < j1; ++j) {
            const uint32_t u = tk.key[j];
            if (u > tau) {
                ++ckeep;
            } else if (u == tau) {
                ckeep += e < need;
                ++e;
            }
        }
    }
    int w = block_excl_scan<NT>(ckeep, tk.tmp, tot);
    {
        int e = eq0;
        for (int j = j0; j < j1; ++j) {
            const uint32_t u = tk.key[j];
            bool keep = u > tau;
            if (u == tau) {
                keep = e < need;
                ++e;
            }
            if (keep && w < k) {
                tk.res_key[w] = u;
                tk.res_idx[w] = tk.idx[j];
                ++w;
            }
        }
    }
    __syncthreads();
    for (int j = tid; j < k; j += NT) {
        tk.key[j] = tk.res_key[j];
        tk.idx[j] = tk.res_idx[j];
    }
    __syncthreads();
    tk.n = k;
    tk.valid = true;
    tk.thresh = tau;
}

// Append the survivors among keys[0..n) (indices t0 + j, or ids[j]) in order,
// then shrink the buffer if the next chunk of `chunk` entries might not fit.
template <int CHUNK>
__device__ void append_chunk(TopK &tk, const uint32_t *keys, const int32_t *ids, int t0, int n, int k, int cap) {
    constexpr int PER = (CHUNK + NT - 1) / NT;
    const int tid = threadIdx.x;
    const int j0 = min(tid * PER, n), j1 = min(j0 + PER, n);
    const bool all = !tk.valid;
    const uint32_t th = tk.thresh;
    int c = 0;
    for (int j = j0; j < j1; ++j) c += all || keys[j] > th;
    int tot;
    int w = tk.n + block_excl_scan<NT>(c, tk.tmp, tot);
    for (int j = j0; j < j1; ++j) {
        const uint32_t u = keys[j];
        if ((all || u > th) && w < cap) {
            tk.key[w] = u;
            tk.idx[w] = ids ? ids[j] : t0 + j;
            ++w;
        }
    }
    tk.n += tot;
    __syncthreads();
    if (tk.n > cap - CHUNK) reduce_topk(tk, k);
}

template <int SRC, int MODE, int R, int AGG>
__global__ void __launch_bounds__(NT) scan_kernel(ScanArgs a) {
    constexpr bool FROM_KT = SRC != SRC_SCORES;
    using KT = typename std::conditional<SRC == SRC_KT_FP32, float, __nv_bfloat16>::type;
    constexpr int ES = SRC == SRC_KT_FP32 ? 4 : 2;
    constexpr int ROWB = FROM_KT ? R * ES : 4;
    constexpr int LPT = FROM_KT ? ROWB / 16 : 1;  // lanes per token
    constexpr int EPL = 16 / ES;                  // elements per lane
    constexpr int TILE = FROM_KT ? kScanStageBytes / ROWB : kScoreTileTokens;
    static_assert(!FROM_KT || (LPT >= 1 && LPT <= 32 && (LPT & (LPT - 1)) == 0), "bad lanes per token");

    extern __shared__ __align__(128) unsigned char smem[];
    const ScanSmem L = scan_smem(SRC, MODE, FROM_KT ? R : 0, a.nstages, a.cap, a.k, TILE);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint32_t *tkey = reinterpret_cast<uint32_t *>(smem + L.tkey);
    int32_t *tidx = reinterpret_cast<int32_t *>(smem + L.tidx);
    float *qs = reinterpret_cast<float *>(smem + L.qs);

    TopK tk;
    tk.key = reinterpret_cast<uint32_t *>(smem + L.buf_key);
    tk.idx = reinterpret_cast<int32_t *>(smem + L.buf_idx);
    tk.res_key = reinterpret_cast<uint32_t *>(smem + L.res_key);
    tk.res_idx = reinterpret_cast<int32_t *>(smem + L.res_idx);
    tk.hist = reinterpret_cast<uint32_t *>(smem + L.hist);
    tk.tmp = reinterpret_cast<int *>(smem + L.tmp);
    tk.misc = reinterpret_cast<int *>(smem + L.misc);
    tk.n = 0;
    tk.valid = false;
    tk.thresh = 0u;

    const int tid = threadIdx.x;
    const long long cta = blockIdx.x;
    const long long x_begin = cta * a.total_tiles / a.grid;
    const long long x_end = (cta + 1) * a.total_tiles / a.grid;
    const int ntiles = (int)(x_end - x_begin);
    const int tpb = a.tiles_per_bh;

    if (FROM_KT && tid == 0) {
        for (int s = 0; s < a.nstages; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();

    auto tile_info = [&](long long x, int &bh, int &t0, int &n) {
        bh = (int)(x / tpb);
        t0 = (int)(x - (long long)bh * tpb) * TILE;
        const int b = bh / a.Hkv;
        const int Tb = clamp_seq(__ldg(a.seq_lens + b), a.T_cap, a.status);
        n = min(TILE, Tb - t0);
        if (n < 0) n = 0;
    };

    uint64_t pol = 0;
    auto issue = [&](int i) {  // thread 0 only
        int bh, t0, n;
        tile_info(x_begin + i, bh, t0, n);
        const int s = i % a.nstages;
        if (n > 0) {
            const uint32_t bytes = (uint32_t)n * ROWB;
            mbar_arrive_expect_tx(&bars[s], bytes);
            const char *src = static_cast<const char *>(a.src) + ((size_t)bh * a.T_cap + t0) * ROWB;
            bulk_g2s(smem + L.stages + (size_t)s * kScanStageBytes, src, bytes, &bars[s], pol);
        } else {
            mbar_arrive(&bars[s]);
        }
    };

    int issued = 0;
    if (FROM_KT && tid == 0) {
        pol = policy_evict_first();
        issued = min(a.nstages, ntiles);
        for (int i = 0; i < issued; ++i) issue(i);
    }

    // per-thread query slice (SUM: one folded query kept in registers)
    const int chunk = tid % LPT;
    float qreg[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) qreg[e] = 0.f;

    auto begin_segment = [&](int bh) {
        if (FROM_KT) {
            const int nq = a.nq;
            for (int p = tid; p < nq * R; p += NT) qs[p] = a.qproj[(size_t)bh * nq * R + p];
        }
        tk.n = 0;
        tk.valid = false;
        __syncthreads();
        if (FROM_KT && AGG == JSSA_AGG_SUM) {
#pragma unroll
            for (int e = 0; e < EPL; ++e) qreg[e] = qs[chunk * EPL + e];
        }
    };

    auto cta_of = [&](long long x) -> long long { return ((x + 1) * a.grid - 1) / a.total_tiles; };

    auto finish_segment = [&](int bh) {
        if (tk.n > a.k) reduce_topk(tk, a.k);
        const long long first = (long long)bh * tpb;
        const long long c_first = cta_of(first), c_last = cta_of(first + tpb - 1);
        const int slot = (int)(cta - c_first), nseg = (int)(c_last - c_first + 1);
        const size_t cb = ((size_t)bh * a.max_seg + slot) * a.k;
        for (int j = tid; j < tk.n; j += NT) {
            a.cand_key[cb + j] = tk.key[j];
            a.cand_idx[cb + j] = tk.idx[j];
        }
        if (tid == 0) a.cand_cnt[(size_t)bh * a.max_seg + slot] = tk.n;
        __threadfence();
        __syncthreads();
        if (tid == 0) tk.misc[2] = atomicAdd(&a.counters[bh], 1u) == (unsigned)(nseg - 1);
        __syncthreads();
        const bool last = tk.misc[2] != 0;
        __syncthreads();
        if (!last) return;
        __threadfence();
        tk.n = 0;
        tk.valid = false;
        for (int s = 0; s < nseg; ++s) {
            const int cnt = __ldcg(a.cand_cnt + (size_t)bh * a.max_seg + s);
            const size_t base = ((size_t)bh * a.max_seg + s) * a.k;
            for (int off = 0; off < cnt; off += TILE) {
                const int m = min(TILE, cnt - off);
                for (int j = tid; j < m; j += NT) {
                    tkey[j] = __ldcg(a.cand_key + base + off + j);
                    tidx[j] = __ldcg(a.cand_idx + base + off + j);
                }
                __syncthreads();
                append_chunk<TILE>(tk, tkey, tidx, 0, m, a.k, a.cap);
                __syncthreads();
            }
        }
        if (tk.n > a.k) reduce_topk(tk, a.k);
        for (int j = tid; j < a.k; j += NT) a.idx_out[(size_t)bh * a.k + j] = j < tk.n ? tk.idx[j] : -1;
        if (tid == 0) {
            if (a.count_out) a.count_out[bh] = tk.n;
            a.counters[bh] = 0u;
        }
        __syncthreads();
    };

    int cur_bh = -1;
    bool timed_out = false;
    int consumed = 0;
    for (int i = 0; i < ntiles; ++i) {
        int bh, t0, n;
        tile_info(x_begin + i, bh, t0, n);
        if (bh != cur_bh) {
            if (MODE == MODE_SELECT && cur_bh >= 0) finish_segment(cur_bh);
            cur_bh = bh;
            begin_segment(bh);
        }
        if constexpr (FROM_KT) {
            const int s = i % a.nstages;
            const uint32_t par = (uint32_t)(i / a.nstages) & 1u;
            const bool ok = __syncthreads_and(mbar_wait_bounded(&bars[s], par) ? 1 : 0) != 0;
            if (!ok) {
                timed_out = true;
                break;
            }
            consumed = i + 1;
            if (n > 0) {
                const uint4 *sv = reinterpret_cast<const uint4 *>(smem + L.stages + (size_t)s * kScanStageBytes);
#pragma unroll
                for (int tt = tid / LPT; tt < TILE; tt += NT / LPT) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (tt < n) v = sv[tt * LPT + chunk];
                    float kf[EPL];
                    Vec16<KT>::unpack(v, kf);
                    float sc;
                    if (AGG == JSSA_AGG_SUM) {
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < EPL; ++e) acc = fmaf(kf[e], qreg[e], acc);
#pragma unroll
                        for (int off = 1; off < LPT; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                        sc = acc;
                    } else {
                        float best = -INFINITY;
                        for (int g = 0; g < a.nq; ++g) {
                            const float *qg = qs + g * R + chunk * EPL;
                            float acc = 0.f;
#pragma unroll
                            for (int e = 0; e < EPL; ++e) acc = fmaf(kf[e], qg[e], acc);
#pragma unroll
                            for (int off = 1; off < LPT; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                            best = fmaxf(best, acc);
                        }
                        sc = best;
                    }
                    if (chunk == 0 && tt < n) tkey[tt] = MODE == MODE_WRITE ? __float_as_uint(sc) : score_key(sc);
                }
            }
            __syncthreads();  // stage s consumed; tkey complete
            if (tid == 0 && issued < ntiles) {
                issue(issued);
                ++issued;
            }
        } else {
            if (n > 0) {
                constexpr int PERT = (TILE + NT - 1) / NT;
                const float *srow = static_cast<const float *>(a.src) + (size_t)bh * a.T_cap + t0;
                float v[PERT];
#pragma unroll
                for (int u = 0; u < PERT; ++u) {
                    const int j = tid + u * NT;
                    v[u] = j < n ? __ldcs(srow + j) : 0.f;
                }
#pragma unroll
                for (int u = 0; u < PERT; ++u) {
                    const int j = tid + u * NT;
                    if (j < n) tkey[j] = score_key(v[u]);
                }
            }
            __syncthreads();
        }
        if (n > 0) {
            if (MODE == MODE_WRITE) {
                float *dst = a.scores_out + (size_t)bh * a.T_cap + t0;
                for (int j = tid; j < n; j += NT) dst[j] = __uint_as_float(tkey[j]);
            } else {
                append_chunk<TILE>(tk, tkey, nullptr, t0, n, a.k, a.cap);
            }
        }
        __syncthreads();
    }

    if (timed_out) {
        if (tid == 0) {
            if (a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_TIMEOUT);
            // let the copies already in flight land before the CTA exits
            for (int i = consumed; i < issued; ++i)
                (void)mbar_wait_bounded(&bars[i % a.nstages], (uint32_t)(i / a.nstages) & 1u);
        }
        __syncthreads();
        return;
    }
    if (MODE == MODE_SELECT && cur_bh >= 0) finish_segment(cur_bh);
}

template <int SRC, int MODE, int R, int AGG>
void (*pick3())(ScanArgs) {
    return scan_kernel<SRC, MODE, R, AGG>;
}

template <int SRC, int MODE>
void (*pick_r(int r, int agg))(ScanArgs) {
    switch (r) {
        case 8: return agg ? pick3<SRC, MODE, 8, 1>() : pick3<SRC, MODE, 8, 0>();
        case 16: return agg ? pick3<SRC, MODE, 16, 1>() : pick3<SRC, MODE, 16, 0>();
        case 32: return agg ? pick3<SRC, MODE, 32, 1>() : pick3<SRC, MODE, 32, 0>();
        case 64: return agg ? pick3<SRC, MODE, 64, 1>() : pick3<SRC, MODE, 64, 0>();
        case 128: return agg ? pick3<SRC, MODE, 128, 1>() : pick3<SRC, MODE, 128, 0>();
        default: return nullptr;
    }
}

void (*pick_scan(int src, int mode, int r, int agg))(ScanArgs) {
    if (src == SRC_SCORES) return mode == MODE_SELECT ? scan_kernel<SRC_SCORES, MODE_SELECT, 8, 0> : nullptr;
    if (src == SRC_KT_BF16)
        return mode == MODE_SELECT ? pick_r<SRC_KT_BF16, MODE_SELECT>(r, agg) : pick_r<SRC_KT_BF16, MODE_WRITE>(r, agg);
    return mode == MODE_SELECT ? pick_r<SRC_KT_FP32, MODE_SELECT>(r, agg) : pick_r<SRC_KT_FP32, MODE_WRITE>(r, agg);
}

int scan_tile_tokens(int src, int r) {
    if (src == SRC_SCORES) return kScoreTileTokens;
    return kScanStageBytes / (r * (src == SRC_KT_FP32 ? 4 : 2));
}

}  // namespace

cudaError_t plan_scan(int src, int mode, int agg, int B, int Hkv, int T_cap, int r, int nq, int k, ScanPlan *p) {
    (void)nq;
    auto kern = pick_scan(src, mode, r, agg);
    if (!kern) return cudaErrorInvalidValue;
    ScanPlan P;
    P.src = src;
    P.mode = mode;
    P.tile_tokens = scan_tile_tokens(src, r);
    P.tiles_per_bh = (T_cap + P.tile_tokens - 1) / P.tile_tokens;
    P.total_tiles = (long long)B * Hkv * P.tiles_per_bh;
    P.nstages = src == SRC_SCORES ? 0 : 3;
    P.cap = mode == MODE_SELECT ? k + (P.tile_tokens > 1024 ? P.tile_tokens : 1024) : 0;
    P.smem = scan_smem(src, mode, src == SRC_SCORES ? 0 : r, P.nstages, P.cap, mode == MODE_SELECT ? k : 0,
                       P.tile_tokens)
                 .total;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, NT, P.smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    long long g = (long long)device_sm_count() * occ;
    if (g > P.total_tiles) g = P.total_tiles;
    if (g < 1) g = 1;
    P.grid = (int)g;
    // exact maximum number of segments a (b,h) is split into
    int ms = 1;
    if (mode == MODE_SELECT) {
        const long long BH = (long long)B * Hkv;
        for (long long bh = 0; bh < BH; ++bh) {
            const long long f = bh * P.tiles_per_bh, l = f + P.tiles_per_bh - 1;
            const long long cf = ((f + 1) * P.grid - 1) / P.total_tiles;
            const long long cl = ((l + 1) * P.grid - 1) / P.total_tiles;
            if (cl - cf + 1 > ms) ms = (int)(cl - cf + 1);
        }
    }
    P.max_seg = ms;
    *p = P;
    return cudaSuccess;
}

cudaError_t launch_scan(const ScanPlan &p, const ScanArgs &a0, int agg, cudaStream_t s, bool pdl) {
    auto kern = pick_scan(p.src, p.mode, a0.r, agg);
    if (!kern) return cudaErrorInvalidValue;
    if (p.total_tiles <= 0) return cudaSuccess;
    ScanArgs a = a0;
    a.tile_tokens = p.tile_tokens;
    a.tiles_per_bh = p.tiles_per_bh;
    a.total_tiles = p.total_tiles;
    a.grid = p.grid;
    a.max_seg = p.max_seg;
    a.cap = p.cap;
    a.nstages = p.nstages;
    return launch_kernel(kern, dim3(p.grid), dim3(NT), p.smem, s, pdl, a);
}

}  // namespace jssa
