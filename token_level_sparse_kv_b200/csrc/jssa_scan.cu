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
//    contiguous range [i*N/grid, (i+1)*N/grid), so the load is balanced to one
//    tile whatever B*Hkv is.  A range crosses at most a few (b,h) boundaries;
//    each (b,h) piece of it is a "segment".
//  * 32 KiB tiles of the low-rank key cache arrive through a 3-deep ring of
//    bulk asynchronous copies (TMA engine, mbarrier completion, evict-first L2
//    hint).  A thread scores whole tokens (up to 64 bytes of a row; wider
//    rows are split over 2..8 lanes and reduced with shuffles), reading its
//    16-byte chunks in a lane-rotated order so that every quarter-warp hits 8
//    distinct bank groups.  The score-array source (jssa_topk) is read with
//    plain coalesced loads.
//  * MODE_WRITE stores fp32 scores.  MODE_SELECT keeps a running top-k of the
//    segment in shared memory: a token survives only if its key beats the
//    k-th key kept so far (tokens arrive in ascending index order within a
//    segment, so an equal key always loses to the kept one); survivors are
//    appended with one warp-aggregated shared atomic; when the buffer may not
//    absorb another tile, a radix select (4 passes of 8 bits over
//    order-preserving uint32 keys, then over inverted indices for the tie
//    group) keeps the best k.  The segment's candidates go to the workspace;
//    the last CTA to finish a (b,h) (arrival ticket, no waiting) merges the
//    segments the same way and writes the selection sorted by index.
// The order (score desc, index asc) is a strict total order, so the top-k of
// the union of per-segment top-k sets is the global top-k: the fused path
// returns exactly what jssa_score + jssa_topk return.
#include <type_traits>

#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace jssa {

namespace {

// Tile size, ring depth and block size of the streaming pass (compile-time;
// the defaults are the measured best on B200 for r*2 = 64-byte rows).
#ifndef JSSA_SCAN_TILE_BYTES
#define JSSA_SCAN_TILE_BYTES 32768
#endif
#ifndef JSSA_SCAN_STAGES
#define JSSA_SCAN_STAGES 3
#endif
#ifndef JSSA_SCAN_THREADS
#define JSSA_SCAN_THREADS 256
#endif
constexpr int NT = JSSA_SCAN_THREADS;
constexpr int kTileBytes = JSSA_SCAN_TILE_BYTES;
constexpr int kStages = JSSA_SCAN_STAGES;
static_assert(NT >= 256 && NT % 256 == 0, "the radix select uses one thread per digit");
constexpr int kHistBins = 2048;  // 11-bit digits of the one-pass select
constexpr int kBoundaryMax = 64;  // boundary-group entries resolved by exact ranking

__host__ __device__ inline int next_pow2(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

struct ScanSmem {
    size_t stages, bars, qs, buf_key, buf_idx, res_key, res_idx, hist, tmp, misc, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline ScanSmem scan_smem(int src, int mode, int r, int nq, int nstages, int cap, int k) {
    ScanSmem L;
    size_t o = 0;
    const bool from_kt = src != SRC_SCORES;
    const bool sel = mode == MODE_SELECT;
    L.stages = o;
    o += from_kt ? (size_t)nstages * kTileBytes : 0;
    L.bars = o;
    o = align_up(o + (from_kt ? (size_t)nstages * 8 : 0), 16);
    L.qs = o;
    o = align_up(o + (from_kt ? (size_t)nq * r * 4 : 0), 16);
    L.buf_key = o;
    o = align_up(o + (sel ? (size_t)cap * 4 : 0), 16);
    L.buf_idx = o;
    o = align_up(o + (sel ? (size_t)cap * 4 : 0), 16);
    L.res_key = o;
    o = align_up(o + (sel ? (size_t)k * 4 : 0), 16);
    L.res_idx = o;
    o = align_up(o + (sel ? (size_t)next_pow2(k) * 4 : 0), 16);
    L.hist = o;
    o = align_up(o + (size_t)kHistBins * 4, 16);
    L.tmp = o;
    o = align_up(o + 32 * 4, 16);
    L.misc = o;
    o = align_up(o + 16 * 4, 128);
    L.total = o;
    return L;
}

// Running top-k buffer in shared memory (pointers only; passed by value so that
// nothing of the hot loop lives in local memory).  Entries are unordered; the
// count lives in shared memory (misc[4]) because warps append with atomics.
struct TopK {
    uint32_t *key;
    int32_t *idx;
    uint32_t *res_key;
    int32_t *res_idx;
    uint32_t *hist;
    int *tmp;
    int *misc;  // [0..1], [5] select scratch, [2] ticket flag, [3] keep counter, [4] count,
                // [6] timeout flag, [8..9] shrink decisions
};

// Sum of the per-chunk partials of one thread, independent of the lane's
// rotation of the visiting order: a rotation by one swaps the pairs {0,2} and
// {1,3} as wholes, and each pair sum is commutative, so every lane adds the
// same two pair sums.  Identical rows therefore score bit-identically.
template <int CPT>
__device__ __forceinline__ float chunk_sum(const float (&p)[CPT]) {
    if constexpr (CPT == 4) return (p[0] + p[2]) + (p[1] + p[3]);
    if constexpr (CPT == 2) return p[0] + p[1];
    return p[0];
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Histogram increment (measured: aggregating equal bins across a warp with
// match.any costs more than the shared-memory atomic contention it saves).
__device__ __forceinline__ void hist_add(uint32_t *hist, uint32_t bin, bool active) {
    if (active) atomicAdd(&hist[bin], 1u);
}

// Warp-aggregated append of one candidate per lane (all 32 lanes call it).
__device__ __forceinline__ void offer(uint32_t *bkey, int32_t *bidx, int *count, bool take, uint32_t key,
                                      int32_t idx, int cap) {
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (m == 0u) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(m) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(count, __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (take) {
        const int pos = base + __popc(m & lanemask_lt());
        if (pos < cap) {
            bkey[pos] = key;
            bidx[pos] = idx;
        }
    }
}

// kk-th largest value of val(j) over the entries with use(j) (1 <= kk <= their
// count).  Returns the value, how many entries equal to it are in the top kk,
// and (eq_total) how many used entries equal it.
template <typename Use, typename Val>
__device__ __forceinline__ void radix_select(int n, int kk, const TopK tk, Use use, Val val, uint32_t &tau,
                                             int &need, int &eq_total) {
    const int tid = threadIdx.x;
    uint32_t prefix = 0u, mask = 0u;
    int last_count = 0;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        if (tid < 256) tk.hist[tid] = 0u;
        __syncthreads();
        for (int j0 = 0; j0 < n; j0 += NT) {
            const int j = j0 + tid;
            bool on = false;
            uint32_t u = 0u;
            if (j < n && use(j)) {
                u = val(j);
                on = (u & mask) == prefix;
            }
            hist_add(tk.hist, (u >> shift) & 0xffu, on);
        }
        __syncthreads();
        const int c = tid < 256 ? (int)tk.hist[255 - tid] : 0;
        int tot;
        const int ex = block_excl_scan<NT>(c, tk.tmp, tot);
        if (ex < kk && ex + c >= kk) {
            tk.misc[0] = 255 - tid;
            tk.misc[1] = ex;
            tk.misc[5] = c;
        }
        __syncthreads();
        prefix |= (uint32_t)tk.misc[0] << shift;
        mask |= 0xffu << shift;
        kk -= tk.misc[1];
        last_count = tk.misc[5];
        __syncthreads();
    }
    tau = prefix;
    need = kk;
    eq_total = last_count;
}

// Keep the best k of the n > k buffered entries under (key desc, idx asc);
// returns the key of the k-th kept entry (the new survival threshold).
// General form: 8-bit radix passes, then the same over inverted indices for
// the tie group.  Used when the one-pass form below cannot separate the keys.
__device__ __noinline__ uint32_t reduce_topk_radix(const TopK tk, int n, int k) {
    const int tid = threadIdx.x;
    uint32_t tau, tau2 = 0u;
    int need, m;
    radix_select(
        n, k, tk, [&](int) { return true; }, [&](int j) { return tk.key[j]; }, tau, need, m);
    const bool all_ties = need == m;
    if (!all_ties) {
        // among the entries equal to tau, the `need` lowest indices
        int need2, m2;
        radix_select(
            n, need, tk, [&](int j) { return tk.key[j] == tau; },
            [&](int j) { return ~(uint32_t)tk.idx[j]; }, tau2, need2, m2);
    }
    if (tid == 0) tk.misc[3] = 0;
    __syncthreads();
    const int lane = tid & 31;
    for (int j0 = 0; j0 < n; j0 += NT) {
        const int j = j0 + tid;
        bool keep = false;
        uint32_t u = 0u;
        int32_t ix = 0;
        if (j < n) {
            u = tk.key[j];
            ix = tk.idx[j];
            keep = u > tau || (u == tau && (all_ties || ~(uint32_t)ix >= tau2));
        }
        const unsigned msk = __ballot_sync(0xffffffffu, keep);
        int base = 0;
        if (msk) {
            const int leader = __ffs(msk) - 1;
            if (lane == leader) base = atomicAdd(&tk.misc[3], __popc(msk));
            base = __shfl_sync(0xffffffffu, base, leader);
        }
        if (keep) {
            const int pos = base + __popc(msk & lanemask_lt());
            if (pos < k) {
                tk.res_key[pos] = u;
                tk.res_idx[pos] = ix;
            }
        }
    }
    __syncthreads();
    for (int j = tid; j < k; j += NT) {
        tk.key[j] = tk.res_key[j];
        tk.idx[j] = tk.res_idx[j];
    }
    if (tid == 0) tk.misc[4] = k;
    __syncthreads();
    return tau;
}

__device__ __forceinline__ bool ranks_before(uint32_t ka, int32_t ia, uint32_t kb, int32_t ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// Adaptive-digit form of the same reduction.  The keys of the buffer share all
// bits above the highest bit where its minimum and maximum differ, so the 11
// bits below that point give a monotone 2048-bin histogram; one scan finds
// the bin of the k-th key.  While that bin is large, the next 11 bits of its
// keys are histogrammed the same way; its last few entries are then ranked
// exactly by (key desc, index asc).  Usually one or two levels instead of the
// four fixed 8-bit passes of the radix form.
__device__ __noinline__ uint32_t reduce_topk(const TopK tk, int n, int k) {
    const int tid = threadIdx.x, lane = tid & 31;
    unsigned *um = reinterpret_cast<unsigned *>(tk.misc);
    if (tid == 0) {
        um[10] = 0u;           // max key
        um[11] = 0xffffffffu;  // min key
    }
    __syncthreads();
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int j = tid; j < n; j += NT) {
        const uint32_t u = tk.key[j];
        lo = min(lo, u);
        hi = max(hi, u);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
        atomicMin(&um[11], lo);
        atomicMax(&um[10], hi);
    }
    __syncthreads();
    hi = um[10];
    lo = um[11];
    if (hi == lo) return reduce_topk_radix(tk, n, k);  // every key equal: order by index alone
    int top = 31 - __clz((int)(hi ^ lo));           // highest bit where keys differ
    uint32_t pmask = top == 31 ? 0u : ~((2u << top) - 1u), pval = hi & pmask;
    int kk = k, mb = 0;
    for (;;) {
        const int width = top + 1 < 11 ? top + 1 : 11;
        const int shift = top + 1 - width;
        const uint32_t dmask = (1u << width) - 1u;
        for (int d = tid; d < kHistBins; d += NT) tk.hist[d] = 0u;
        __syncthreads();
        for (int j0 = 0; j0 < n; j0 += NT) {
            const int j = j0 + tid;
            const uint32_t u = j < n ? tk.key[j] : 0u;
            hist_add(tk.hist, (u >> shift) & dmask, j < n && (u & pmask) == pval);
        }
        __syncthreads();
        // descending scan: thread t owns bins [kHistBins - BPT (t+1), kHistBins - BPT t)
        constexpr int BPT = kHistBins / NT;
        const int base_bin = kHistBins - BPT * (tid + 1);
        int cnt[BPT];
        int sum = 0;
#pragma unroll
        for (int q = 0; q < BPT; ++q) {
            cnt[q] = (int)tk.hist[base_bin + BPT - 1 - q];
            sum += cnt[q];
        }
        int tot;
        int ex = block_excl_scan<NT>(sum, tk.tmp, tot);
#pragma unroll
        for (int q = 0; q < BPT; ++q) {
            if (ex < kk && ex + cnt[q] >= kk) {
                tk.misc[0] = base_bin + BPT - 1 - q;
                tk.misc[1] = ex;
                tk.misc[5] = cnt[q];
            }
            ex += cnt[q];
        }
        __syncthreads();
        const uint32_t D = (uint32_t)tk.misc[0];
        kk -= tk.misc[1];
        mb = tk.misc[5];
        pmask |= dmask << shift;
        pval |= D << shift;
        __syncthreads();
        if (kk == mb || mb <= kBoundaryMax || shift == 0) break;
        top = shift - 1;
    }
    // kk entries of the boundary group (keys matching pval under pmask) are kept
    uint32_t kstar = 0u;
    int32_t istar = 0x7fffffff;
    const bool whole = kk == mb;
    if (!whole) {
        if (mb > kBoundaryMax) return reduce_topk_radix(tk, n, k);  // a large group of equal keys
        if (tid == 0) tk.misc[3] = 0;
        __syncthreads();
        uint32_t *bk = tk.hist;
        int32_t *bi = reinterpret_cast<int32_t *>(tk.hist + kBoundaryMax);
        for (int j = tid; j < n; j += NT) {
            const uint32_t u = tk.key[j];
            if ((u & pmask) == pval) {
                const int p = atomicAdd(&tk.misc[3], 1);
                bk[p] = u;
                bi[p] = tk.idx[j];
            }
        }
        __syncthreads();
        for (int i = tid; i < mb; i += NT) {
            const uint32_t ki = bk[i];
            const int32_t ii = bi[i];
            int r = 0;
            for (int j = 0; j < mb; ++j) r += ranks_before(bk[j], bi[j], ki, ii);
            if (r == kk - 1) {
                um[12] = ki;
                tk.misc[13] = ii;
            }
        }
        __syncthreads();
        kstar = um[12];
        istar = tk.misc[13];
    }
    if (tid == 0) {
        tk.misc[3] = 0;
        um[14] = 0xffffffffu;
    }
    __syncthreads();
    uint32_t kept_min = 0xffffffffu;
    for (int j0 = 0; j0 < n; j0 += NT) {
        const int j = j0 + tid;
        bool keep = false;
        uint32_t u = 0u;
        int32_t ix = 0;
        if (j < n) {
            u = tk.key[j];
            ix = tk.idx[j];
            const uint32_t um_ = u & pmask;
            keep = um_ > pval || (um_ == pval && (whole || !ranks_before(kstar, istar, u, ix)));
        }
        if (keep) kept_min = min(kept_min, u);
        const unsigned msk = __ballot_sync(0xffffffffu, keep);
        int base = 0;
        if (msk) {
            const int leader = __ffs(msk) - 1;
            if (lane == leader) base = atomicAdd(&tk.misc[3], __popc(msk));
            base = __shfl_sync(0xffffffffu, base, leader);
        }
        if (keep) {
            const int pos = base + __popc(msk & lanemask_lt());
            if (pos < k) {
                tk.res_key[pos] = u;
                tk.res_idx[pos] = ix;
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kept_min = min(kept_min, __shfl_xor_sync(0xffffffffu, kept_min, off));
    if (lane == 0) atomicMin(&um[14], kept_min);
    __syncthreads();
    for (int j = tid; j < k; j += NT) {
        tk.key[j] = tk.res_key[j];
        tk.idx[j] = tk.res_idx[j];
    }
    const uint32_t tau = um[14];
    if (tid == 0) tk.misc[4] = k;
    __syncthreads();
    return tau;
}

// Sort a[0..n) ascending in place (bitonic network over the next power of two,
// padded with INT_MAX; a has room for next_pow2(n) entries).
__device__ void sort_ascending(int32_t *a, int n) {
    const int tid = threadIdx.x;
    const int P = next_pow2(n < 1 ? 1 : n);
    for (int j = n + tid; j < P; j += NT) a[j] = 0x7fffffff;
    __syncthreads();
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < P / 2; i += NT) {
                const int lo = 2 * stride * (i / stride) + (i % stride);
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const int32_t x = a[lo], y = a[hi];
                if ((x > y) == up) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
            __syncthreads();
        }
    }
}

// End of a segment: publish its candidates; the last CTA of the (b,h) merges
// all segments (ascending token order; inside one segment the order is
// arbitrary, so keys equal to the threshold stay candidates) and writes the
// selection sorted by index.
template <int MCH>
__device__ __noinline__ void finish_segment(const ScanArgs &a, const TopK tk, int bh, long long cta) {
    const int tid = threadIdx.x;
    int n = tk.misc[4];
    __syncthreads();
    if (n > a.k) {
        reduce_topk(tk, n, a.k);
        n = a.k;
    }
    const int tpb = a.tiles_per_bh;
    const long long first = (long long)bh * tpb;
    const long long c_first = ((first + 1) * a.grid - 1) / a.total_tiles;
    const long long c_last = ((first + tpb) * a.grid - 1) / a.total_tiles;
    const int slot = (int)(cta - c_first), nseg = (int)(c_last - c_first + 1);
    const size_t cb = ((size_t)bh * a.max_seg + slot) * a.k;
    for (int j = tid; j < n; j += NT) {
        a.cand_key[cb + j] = tk.key[j];
        a.cand_idx[cb + j] = tk.idx[j];
    }
    if (tid == 0) a.cand_cnt[(size_t)bh * a.max_seg + slot] = n;
    __threadfence();
    __syncthreads();
    if (tid == 0) tk.misc[2] = atomicAdd(&a.counters[bh], 1u) == (unsigned)(nseg - 1);
    __syncthreads();
    const bool last = tk.misc[2] != 0;
    if (!last) return;
    __threadfence();
    if (tid == 0) tk.misc[4] = 0;
    __syncthreads();
    bool valid = false;
    uint32_t thresh = 0u;
    for (int s = 0; s < nseg; ++s) {
        const int cnt = __ldcg(a.cand_cnt + (size_t)bh * a.max_seg + s);
        const size_t base = ((size_t)bh * a.max_seg + s) * a.k;
        for (int off = 0; off < cnt; off += MCH) {
            const int m = min(MCH, cnt - off);
            for (int j0 = 0; j0 < m; j0 += NT) {
                const int j = j0 + tid;
                uint32_t u = 0u;
                int32_t ix = 0;
                if (j < m) {
                    u = __ldcg(a.cand_key + base + off + j);
                    ix = __ldcg(a.cand_idx + base + off + j);
                }
                offer(tk.key, tk.idx, &tk.misc[4], j < m && (!valid || u >= thresh), u, ix, a.cap);
            }
            __syncthreads();
            const int nb = tk.misc[4];
            __syncthreads();
            if (nb > a.cap - MCH) {
                thresh = reduce_topk(tk, nb, a.k);
                valid = true;
            }
        }
    }
    n = tk.misc[4];
    __syncthreads();
    if (n > a.k) {
        reduce_topk(tk, n, a.k);
        n = a.k;
    }
    int32_t *srt = tk.res_idx;
    for (int j = tid; j < n; j += NT) srt[j] = tk.idx[j];
    __syncthreads();
    sort_ascending(srt, n);
    for (int j = tid; j < a.k; j += NT) a.idx_out[(size_t)bh * a.k + j] = j < n ? srt[j] : -1;
    if (tid == 0) {
        if (a.count_out) a.count_out[bh] = n;
        a.counters[bh] = 0u;
    }
    __syncthreads();
}

template <int SRC, int MODE, int R, int AGG>
__global__ void __launch_bounds__(NT, 2) scan_kernel(ScanArgs a) {
    constexpr bool FROM_KT = SRC != SRC_SCORES;
    using KT = typename std::conditional<SRC == SRC_KT_FP32, float, __nv_bfloat16>::type;
    constexpr int ES = SRC == SRC_KT_FP32 ? 4 : 2;
    constexpr int ROWB = FROM_KT ? R * ES : 4;   // bytes per token
    constexpr int TPB = ROWB > 64 ? 64 : ROWB;   // bytes of a token per thread
    constexpr int LPT = ROWB / TPB;              // lanes per token
    constexpr int CPT = FROM_KT ? TPB / 16 : 1;  // 16-byte chunks per thread
    constexpr int EPL = 16 / ES;                 // elements per chunk
    constexpr int TILE = FROM_KT ? kTileBytes / ROWB : kScoreTileTokens;
    constexpr int TPP = NT / LPT;  // tokens per pass
    constexpr int PASSES = FROM_KT ? TILE / TPP : TILE / NT;
    constexpr int QN = FROM_KT ? CPT * EPL : 1;
    constexpr int MCH = FROM_KT ? (TILE > 1024 ? TILE : 1024) : TILE;  // merge chunk; cap >= k + MCH
    static_assert(!FROM_KT || (LPT >= 1 && LPT <= 32 && (LPT & (LPT - 1)) == 0), "lanes per token");
    static_assert(!FROM_KT || (CPT >= 1 && CPT <= 4), "chunks per thread");
    static_assert(!FROM_KT || TILE % TPP == 0, "tile / pass");

    extern __shared__ __align__(128) unsigned char smem[];
    const int nstages = a.nstages;  // ring depth chosen by the planner (<= kStages)
    const ScanSmem L = scan_smem(SRC, MODE, FROM_KT ? R : 0, a.nq, nstages, a.cap, a.k);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
    float *qs = reinterpret_cast<float *>(smem + L.qs);
    TopK tk;
    tk.key = reinterpret_cast<uint32_t *>(smem + L.buf_key);
    tk.idx = reinterpret_cast<int32_t *>(smem + L.buf_idx);
    tk.res_key = reinterpret_cast<uint32_t *>(smem + L.res_key);
    tk.res_idx = reinterpret_cast<int32_t *>(smem + L.res_idx);
    tk.hist = reinterpret_cast<uint32_t *>(smem + L.hist);
    tk.tmp = reinterpret_cast<int *>(smem + L.tmp);
    tk.misc = reinterpret_cast<int *>(smem + L.misc);
    uint32_t *const bkey = tk.key;
    int32_t *const bidx = tk.idx;
    int *const bcount = tk.misc + 4;
    volatile int *const flags = tk.misc;

    const int tid = threadIdx.x, lane = tid & 31;
    const long long cta = blockIdx.x;
    const long long x_begin = cta * a.total_tiles / a.grid;
    const long long x_end = (cta + 1) * a.total_tiles / a.grid;
    const int ntiles = (int)(x_end - x_begin);
    const int tpb = a.tiles_per_bh;

    if (FROM_KT && tid == 0) {
        for (int s = 0; s < nstages; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
    }
    if (tid == 0) {
        tk.misc[4] = 0;
        tk.misc[6] = 0;
        tk.misc[8] = 0;
        tk.misc[9] = 0;
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();

    // producer state (thread 0): next tile to copy and its ring slot
    int p_bh = (int)(x_begin / tpb), p_t = (int)(x_begin - (long long)p_bh * tpb), p_s = 0, issued = 0;
    uint64_t pol = 0;
    const char *const src_base = static_cast<const char *>(a.src);
    if (FROM_KT && tid == 0) {
        pol = policy_evict_first();
        const int first = min(nstages, ntiles);
        for (; issued < first; ++issued) {
            const int Tb_p = clamp_seq(__ldg(a.seq_lens + p_bh / a.Hkv), a.T_cap, a.status);
            const int t0 = p_t * TILE, n = min(TILE, Tb_p - t0);
            if (n > 0) {
                mbar_arrive_expect_tx(&bars[p_s], (uint32_t)n * ROWB);
                bulk_g2s(smem + L.stages + (size_t)p_s * kTileBytes, src_base + ((size_t)(a.src_div > 1 ? p_bh / a.src_div : p_bh) * a.T_cap + t0) * ROWB,
                         (uint32_t)n * ROWB, &bars[p_s], pol);
            } else {
                mbar_arrive(&bars[p_s]);
            }
            if (++p_t == tpb) {
                p_t = 0;
                ++p_bh;
            }
            if (++p_s == nstages) p_s = 0;
        }
    }

    // lane-rotated chunk order: each quarter-warp reads 8 distinct 16-byte bank groups
    const int sub = tid % LPT;
    const int rot = CPT == 4 ? (lane >> 1) & 3 : (CPT == 2 ? (lane >> 2) & 1 : 0);
    float qreg[QN];  // SUM: this thread's slice of the folded query, in chunk-visit order
#pragma unroll
    for (int e = 0; e < QN; ++e) qreg[e] = 0.f;

    int c_bh = (int)(x_begin / tpb), c_t = (int)(x_begin - (long long)c_bh * tpb), c_s = 0;
    uint32_t c_par = 0u;
    int cur_bh = -1, Tb = 0, consumed = 0;
    bool valid = false, timed_out = false;
    uint32_t thresh = 0u;
    for (int i = 0; i < ntiles; ++i) {
        const int bh = c_bh, t0 = c_t * TILE;
        if (++c_t == tpb) {
            c_t = 0;
            ++c_bh;
        }
        if (bh != cur_bh) {
            if (MODE == MODE_SELECT && cur_bh >= 0) finish_segment<MCH>(a, tk, cur_bh, cta);
            cur_bh = bh;
            Tb = clamp_seq(__ldg(a.seq_lens + bh / a.Hkv), a.T_cap, a.status);
            if (FROM_KT) {
                for (int p = tid; p < a.nq * R; p += NT) qs[p] = a.qproj[(size_t)bh * a.nq * R + p];
            }
            if (tid == 0) {
                tk.misc[4] = 0;
                tk.misc[8] = 0;
                tk.misc[9] = 0;
            }
            valid = false;
            __syncthreads();
            if (FROM_KT && AGG == JSSA_AGG_SUM) {
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    const int ch = sub * CPT + ((c + rot) % CPT);
#pragma unroll
                    for (int e = 0; e < EPL; ++e) qreg[(c * EPL + e) % QN] = qs[ch * EPL + e];
                }
            }
        }
        const int n = max(0, min(TILE, Tb - t0));
        if constexpr (FROM_KT) {
            if (!mbar_wait_bounded(&bars[c_s], c_par)) flags[6] = 1;  // seen by all after the tile barrier
            if (n > 0) {
                const unsigned char *st = smem + L.stages + (size_t)c_s * kTileBytes;
#pragma unroll
                for (int ps = 0; ps < PASSES; ++ps) {
                    const int tt = ps * TPP + tid / LPT;
                    const bool live = tt < n;
                    const unsigned char *row = st + (size_t)tt * ROWB + sub * TPB;
                    float sc;
                    if constexpr (AGG == JSSA_AGG_SUM) {
                        float pc[CPT];
#pragma unroll
                        for (int c = 0; c < CPT; ++c) {
                            uint4 v = make_uint4(0u, 0u, 0u, 0u);
                            if (live) v = *reinterpret_cast<const uint4 *>(row + ((c + rot) % CPT) * 16);
                            float kf[EPL];
                            Vec16<KT>::unpack(v, kf);
                            float acc = 0.f;
#pragma unroll
                            for (int e = 0; e < EPL; ++e) acc = fmaf(kf[e], qreg[c * EPL + e], acc);
                            pc[c] = acc;
                        }
                        float acc = chunk_sum<CPT>(pc);
#pragma unroll
                        for (int off = 1; off < LPT; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                        sc = acc;
                    } else {
                        float kf[CPT][EPL];
#pragma unroll
                        for (int c = 0; c < CPT; ++c) {
                            uint4 v = make_uint4(0u, 0u, 0u, 0u);
                            if (live) v = *reinterpret_cast<const uint4 *>(row + ((c + rot) % CPT) * 16);
                            Vec16<KT>::unpack(v, kf[c]);
                        }
                        float best = -INFINITY;
                        for (int g = 0; g < a.nq; ++g) {
                            float pc[CPT];
#pragma unroll
                            for (int c = 0; c < CPT; ++c) {
                                const int ch = sub * CPT + ((c + rot) % CPT);
                                const float *qg = qs + g * R + ch * EPL;
                                float acc = 0.f;
#pragma unroll
                                for (int e = 0; e < EPL; ++e) acc = fmaf(kf[c][e], qg[e], acc);
                                pc[c] = acc;
                            }
                            float acc = chunk_sum<CPT>(pc);
#pragma unroll
                            for (int off = 1; off < LPT; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                            best = fmaxf(best, acc);
                        }
                        sc = best;
                    }
                    if constexpr (MODE == MODE_WRITE) {
                        if (live && sub == 0) a.scores_out[(size_t)bh * a.T_cap + t0 + tt] = sc;
                    } else {
                        const uint32_t u = forced_key(score_key(sc), t0 + tt, Tb, a.n_sink, a.n_recent);
                        offer(bkey, bidx, bcount, live && sub == 0 && (!valid || u > thresh), u, t0 + tt, a.cap);
                    }
                }
            }
            if (++c_s == nstages) {
                c_s = 0;
                c_par ^= 1u;
            }
            __syncthreads();  // this stage is consumed; every append of the tile is done
            if (flags[6]) {   // a copy never landed: stop (uniform after the barrier)
                timed_out = true;
                break;
            }
            consumed = i + 1;
            if (tid == 0 && issued < ntiles) {
                const int Tb_p = clamp_seq(__ldg(a.seq_lens + p_bh / a.Hkv), a.T_cap, a.status);
                const int tp0 = p_t * TILE, np = min(TILE, Tb_p - tp0);
                if (np > 0) {
                    mbar_arrive_expect_tx(&bars[p_s], (uint32_t)np * ROWB);
                    bulk_g2s(smem + L.stages + (size_t)p_s * kTileBytes,
                             src_base + ((size_t)(a.src_div > 1 ? p_bh / a.src_div : p_bh) * a.T_cap + tp0) * ROWB,
                             (uint32_t)np * ROWB, &bars[p_s], pol);
                } else {
                    mbar_arrive(&bars[p_s]);
                }
                if (++p_t == tpb) {
                    p_t = 0;
                    ++p_bh;
                }
                if (++p_s == nstages) p_s = 0;
                ++issued;
            }
        } else {
            if (n > 0) {
                const float *srow = reinterpret_cast<const float *>(src_base) + (size_t)bh * a.T_cap + t0;
                float v[PASSES];
#pragma unroll
                for (int u = 0; u < PASSES; ++u) {
                    const int j = tid + u * NT;
                    v[u] = j < n ? __ldcs(srow + j) : 0.f;
                }
#pragma unroll
                for (int u = 0; u < PASSES; ++u) {
                    const int j = tid + u * NT;
                    const uint32_t key = forced_key(score_key(v[u]), t0 + j, Tb, a.n_sink, a.n_recent);
                    offer(bkey, bidx, bcount, j < n && (!valid || key > thresh), key, t0 + j, a.cap);
                }
            }
            __syncthreads();
        }
        if constexpr (MODE == MODE_SELECT) {
            // The buffer is shrunk one tile late, on a decision that thread 0 took
            // after the previous tile's barrier, so that no second barrier per tile
            // is needed; the capacity holds k + slack + two tiles.
            if (flags[8 + ((i + 1) & 1)]) {
                __syncthreads();
                const int nb = tk.misc[4];
                __syncthreads();
                if (nb > a.k) {
                    thresh = reduce_topk(tk, nb, a.k);
                    valid = true;
                }
            }
            if (tid == 0) flags[8 + (i & 1)] = tk.misc[4] > a.cap - 2 * TILE;
        }
    }

    if (timed_out) {
        if (tid == 0) {
            if (a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_TIMEOUT);
            // let the copies already in flight land before the CTA exits
            for (int i = consumed; i < issued; ++i)
                (void)mbar_wait_bounded(&bars[i % nstages], (uint32_t)(i / nstages) & 1u);
        }
        __syncthreads();
        return;
    }
    if (MODE == MODE_SELECT && cur_bh >= 0) finish_segment<MCH>(a, tk, cur_bh, cta);
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
    return kTileBytes / (r * (src == SRC_KT_FP32 ? 4 : 2));
}

}  // namespace

cudaError_t plan_scan(int src, int mode, int agg, int B, int Hkv, int T_cap, int r, int nq, int k, ScanPlan *p) {
    auto kern = pick_scan(src, mode, r, agg);
    if (!kern) return cudaErrorInvalidValue;
    ScanPlan P;
    P.nb_cap = 0;
    P.src = src;
    P.mode = mode;
    P.tile_tokens = scan_tile_tokens(src, r);
    P.tiles_per_bh = (T_cap + P.tile_tokens - 1) / P.tile_tokens;
    P.total_tiles = (long long)B * Hkv * P.tiles_per_bh;
    // two 32 KiB stages keep the copy engine saturated (measured: the pure
    // stream reaches the copy-bandwidth peak with 2 or 3 stages)
    P.nstages = src == SRC_SCORES ? 0 : (kStages < 2 ? kStages : 2);
    // capacity: k kept entries, two tiles (or one merge chunk) of new survivors,
    // and slack so that the buffer is shrunk only every few tiles; the slack is
    // the largest that still leaves two CTAs per SM
    const int tiles2 = 2 * P.tile_tokens;
    const int chunk = src == SRC_SCORES ? P.tile_tokens : (P.tile_tokens > 1024 ? P.tile_tokens : 1024);
    int occ = 0;
    const int slacks[4] = {1024, 512, 256, 0};
    for (int si = 0; si < 4; ++si) {
        const int slack = src == SRC_SCORES ? (si == 0 ? P.tile_tokens : slacks[si]) : slacks[si];
        P.cap = mode == MODE_SELECT ? k + (tiles2 > chunk ? tiles2 : chunk) + slack : 0;
        P.smem = scan_smem(src, mode, src == SRC_SCORES ? 0 : r, nq, P.nstages, P.cap, mode == MODE_SELECT ? k : 0)
                     .total;
        cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), P.smem);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, NT, P.smem);
        if (e != cudaSuccess) return e;
        if (occ >= 2 || mode != MODE_SELECT) break;
    }
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
