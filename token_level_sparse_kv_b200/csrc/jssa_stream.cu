// Per-(batch, KV head) top-k selection fused with subspace scoring: the
// warp-specialised persistent streaming form.
//
// Method: news item "JSSA makes token-level sparse decoding gather-free",
// Synopsis (tokens scored in a shared low-dimensional query-key subspace, a
// distinct selected token set per KV head) and Interpretation para 2; "Joint
// Subspace Sparse Attention for Efficient Long-Context Decoding", Abstract
// (distinct per-KV-head selections).
//
// One CTA per SM streams a contiguous range of the flattened (b,h, tile) list
// of the low-rank key cache.  Three roles share the CTA:
//  * a producer thread keeps a ring of 32 KiB bulk asynchronous copies in
//    flight (full / empty mbarriers per stage, evict-first L2 hint);
//  * 16 consumer warps score every token of a tile (the same fp32 arithmetic,
//    lane rotation and chunk order as the score pass, so scores are
//    bit-identical) and append the tokens whose order-preserving key beats the
//    current threshold to an epoch buffer (three buffers, rotating epochs of
//    >= 2048 tokens);
//  * 4 selector warps fold each finished epoch into the running candidate set
//    of the segment, cut it back to the best k with a radix select when it
//    fills, and publish the k-th key (tagged with the segment) as the new
//    threshold.  At the end of a segment they write its candidates to the
//    workspace; the last CTA of a (b,h) to finish (arrival ticket, no waiting)
//    merges the segments and writes the selection sorted by token index.
// The consumers never wait for a selection: only for data, and for an epoch
// buffer two epochs back.  Tokens of a segment arrive in ascending index order
// and a threshold is only ever computed from finished epochs, so a token whose
// key equals the threshold always loses to the kept entry (strict filter).
// The order (score desc, index asc) is strict and total, so the top-k of the
// union of per-segment top-k sets is the global top-k: the result is exactly
// that of the score pass followed by the top-k pass.
#include <cstring>
#include <type_traits>

#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace jssa {

namespace {

constexpr int kConsWarps = 16;
constexpr int kCons = kConsWarps * 32;            // consumer threads
constexpr int kSelWarps = 8;
constexpr int kSelT = kSelWarps * 32;             // selector threads
// Warp roles, selector first: the schedulers favour lower warp ids when
// several warps are ready, and the selector's latency-bound steps are the
// ones that must not wait behind the consumers' streaming work.
constexpr int kSelBase = 0;                       // first selector thread
constexpr int kProdBase = kSelT;                  // producer warp
constexpr int kConsBase = kSelT + 32;             // first consumer thread
constexpr int kThreads = kConsBase + kCons;       // 800
constexpr int kEB = 3;                            // epoch buffers
static_assert(kEB <= 4, "epoch buffer counts live in misc[40..43]");
constexpr int kTile = 32768;                      // bytes per ring stage
constexpr int kMaxStages = 8;
constexpr int kBins = 2048;                       // 11-bit digits
constexpr int kBoundary = 64;                     // boundary group ranked exactly
constexpr int kEpochTokens = 2048;                // minimum tokens per epoch
constexpr int kMaxRows = 8;                       // (b,h) rows per CTA range on the fused step
constexpr int kMinSegTiles = 16;                  // shortest row segment a CTA streams
constexpr int kChunkD = 16;                       // inputs per partial sum of a projection

__host__ __device__ inline int npow2(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}
__host__ __device__ inline size_t al(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct StreamSmem {
    size_t ring, bars, ek, ei, rk, ri, sk, si, hist, misc, qb, xs, nb, total;
};

// misc words (int): [0] abort, [3] candidate count, [4..6] select results,
// [7] boundary counter, [8] selector go/stop, [9] ticket, [10..15] select
// scratch, [16..23] scan partials, [24] copies issued, [32..33] threshold
// (u64), [40..42] epoch buffer counts, [44..45] smallest / largest key
// appended to the segment's candidates, [48..63] reduction scratch.
// misc words, fused step: [46] rows to attend, [64..71] their (b,h), [72..79]
// their token counts.  [80..87]: stage s holds a tile skipped by screening.  qb: folded queries of the range's rows [kMaxRows][r];
// xs: one input row of a projection [256].  nb: screening bounds of the CTA's
// first nb_cap tiles (the space left over by the ring, never a stage of it).
__host__ __device__ inline StreamSmem stream_smem(int nstages, int ept, int cap, int k, int fused_r = 0,
                                                  int nb_cap = 0) {
    StreamSmem L;
    size_t o = 0;
    // the ring and the epoch buffers first: one contiguous region that the
    // fused step's attention epilogue reuses once the stream is done
    L.ring = o;
    o += (size_t)nstages * kTile;
    L.ek = o;
    o = al(o + (size_t)kEB * ept * 4, 16);
    L.ei = o;
    o = al(o + (size_t)kEB * ept * 4, 16);
    L.bars = o;
    o = al(o + (size_t)(2 * nstages + 2 * kEB + kMaxRows + 2) * 8, 16);
    L.rk = o;
    o = al(o + (size_t)cap * 4, 16);
    L.ri = o;
    o = al(o + (size_t)cap * 4, 16);
    L.sk = o;
    o = al(o + (size_t)k * 4, 16);
    L.si = o;
    o = al(o + (size_t)npow2(k) * 4, 16);
    L.hist = o;
    o = al(o + (size_t)kBins * 4, 16);
    L.misc = o;
    o = al(o + 96 * 4, 16);
    L.qb = o;
    o = al(o + (size_t)kMaxRows * fused_r * 4, 16);
    L.xs = o;
    o = al(o + (fused_r ? 256 * 4 : 0), 16);
    L.nb = o;
    o = al(o + (size_t)nb_cap * 4, 128);
    L.total = o;
    return L;
}

// ------------------------------------------------------------- selector ---
__device__ __forceinline__ void sel_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kSelT) : "memory"); }

__device__ __forceinline__ unsigned lane_lt() {
    unsigned m;
    asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exclusive scan over the selector threads (two selector barriers).
__device__ __forceinline__ int sel_scan(int v, int *tmp, int st, int &total) {
    const int lane = st & 31, w = st >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) tmp[w] = x;
    sel_sync();
    int pre = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < kSelWarps; ++i) {
        const int t = tmp[i];
        pre += i < w ? t : 0;
        tot += t;
    }
    sel_sync();
    total = tot;
    return pre + x - v;
}

// Candidate set and scratch of the selector, in shared memory.
struct Sel {
    uint32_t *rk;  // candidate keys [cap]
    int32_t *ri;   // candidate token indices [cap]
    uint32_t *sk;  // kept keys [k]
    int32_t *si;   // kept indices / sort scratch [npow2(k)]
    uint32_t *hist;
    int *misc;
    int st;
};

__device__ __forceinline__ bool before(uint32_t ka, int32_t ia, uint32_t kb, int32_t ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// kk-th largest of val(j) over the entries with use(j), by 8-bit radix
// passes: returns the value, the number of entries equal to it inside the
// top kk, and how many used entries equal it.
template <typename Use, typename Val>
__device__ void sel_radix(const Sel &S, int n, int kk, Use use, Val val, uint32_t &tau, int &need, int &eq) {
    uint32_t prefix = 0u, mask = 0u;
    int last = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int d = S.st; d < 256; d += kSelT) S.hist[d] = 0u;
        sel_sync();
        for (int j = S.st; j < n; j += kSelT) {
            if (!use(j)) continue;
            const uint32_t u = val(j);
            if ((u & mask) == prefix) atomicAdd(&S.hist[(u >> shift) & 0xffu], 1u);
        }
        sel_sync();
        // thread st owns bin 255 - st (descending)
        static_assert(kSelT == 256, "one radix bin per selector thread");
        const int c0 = (int)S.hist[255 - S.st];
        int tot;
        const int ex = sel_scan(c0, S.misc + 16, S.st, tot);
        if (ex < kk && ex + c0 >= kk) {
            S.misc[4] = 255 - S.st;
            S.misc[5] = ex;
            S.misc[6] = c0;
        }
        sel_sync();
        prefix |= (uint32_t)S.misc[4] << shift;
        mask |= 0xffu << shift;
        kk -= S.misc[5];
        last = S.misc[6];
        sel_sync();
    }
    tau = prefix;
    need = kk;
    eq = last;
}

// Compact the kept entries (keep(j)) of rk/ri[0..n) into rk/ri[0..k) through
// sk/si; returns the smallest kept key.
template <typename Keep>
__device__ uint32_t sel_compact(const Sel &S, int n, int k, Keep keep) {
    unsigned *um = reinterpret_cast<unsigned *>(S.misc);
    if (S.st == 0) {
        S.misc[10] = 0;
        um[11] = 0xffffffffu;
    }
    sel_sync();
    const int lane = S.st & 31;
    uint32_t kmin = 0xffffffffu;
    for (int j0 = 0; j0 < n; j0 += kSelT) {
        const int j = j0 + S.st;
        uint32_t u = 0u;
        int32_t ix = 0;
        bool kp = false;
        if (j < n) {
            u = S.rk[j];
            ix = S.ri[j];
            kp = keep(u, ix);
        }
        if (kp) kmin = min(kmin, u);
        const unsigned m = __ballot_sync(0xffffffffu, kp);
        int base = 0;
        if (m) {
            const int ld = __ffs(m) - 1;
            if (lane == ld) base = atomicAdd(&S.misc[10], __popc(m));
            base = __shfl_sync(0xffffffffu, base, ld);
        }
        if (kp) {
            const int p = base + __popc(m & lane_lt());
            if (p < k) {
                S.sk[p] = u;
                S.si[p] = ix;
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
    if (lane == 0) atomicMin(&um[11], kmin);
    sel_sync();
    for (int j = S.st; j < k; j += kSelT) {
        S.rk[j] = S.sk[j];
        S.ri[j] = S.si[j];
    }
    const uint32_t t = um[11];
    sel_sync();
    return t;
}

// Keep the best k of the n > k candidates under (key desc, index asc), with
// the candidates read from shared memory on every pass (any n).
// Adaptive digits: the keys share every bit above the highest bit where
// their minimum and maximum differ, so 11 bits below it give a monotone
// histogram; the bin of the k-th key is refined by the next 11 bits while it
// holds many entries, and a small boundary group is ranked exactly.  Large
// groups of equal keys fall back to 8-bit passes over keys, then over
// inverted indices.  Returns the k-th kept key (the new threshold).
__device__ __noinline__ uint32_t sel_reduce_smem(const Sel &S, int n, int k) {
    unsigned *um = reinterpret_cast<unsigned *>(S.misc);
    if (S.st == 0) {
        um[12] = 0u;
        um[13] = 0xffffffffu;
    }
    sel_sync();
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int j = S.st; j < n; j += kSelT) {
        const uint32_t u = S.rk[j];
        lo = min(lo, u);
        hi = max(hi, u);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if ((S.st & 31) == 0) {
        atomicMax(&um[12], hi);
        atomicMin(&um[13], lo);
    }
    sel_sync();
    hi = um[12];
    lo = um[13];
    sel_sync();
    bool general = hi == lo;
    uint32_t pmask = 0u, pval = 0u;
    int kk = k, mb = 0;
    if (!general) {
        int top = 31 - __clz((int)(hi ^ lo));
        pmask = top == 31 ? 0u : ~((2u << top) - 1u);
        pval = hi & pmask;
        for (;;) {
            const int width = top + 1 < 11 ? top + 1 : 11;
            const int shift = top + 1 - width;
            const uint32_t dmask = (1u << width) - 1u;
            for (int d = S.st; d < kBins; d += kSelT) S.hist[d] = 0u;
            sel_sync();
            for (int j = S.st; j < n; j += kSelT) {
                const uint32_t u = S.rk[j];
                if ((u & pmask) == pval) atomicAdd(&S.hist[(u >> shift) & dmask], 1u);
            }
            sel_sync();
            constexpr int BPT = kBins / kSelT;  // bins per thread, descending
            const int bb = kBins - BPT * (S.st + 1);
            int cnt[BPT];
            int sum = 0;
#pragma unroll
            for (int q = 0; q < BPT; ++q) {
                cnt[q] = (int)S.hist[bb + BPT - 1 - q];
                sum += cnt[q];
            }
            int tot;
            int ex = sel_scan(sum, S.misc + 16, S.st, tot);
#pragma unroll
            for (int q = 0; q < BPT; ++q) {
                if (ex < kk && ex + cnt[q] >= kk) {
                    S.misc[4] = bb + BPT - 1 - q;
                    S.misc[5] = ex;
                    S.misc[6] = cnt[q];
                }
                ex += cnt[q];
            }
            sel_sync();
            pmask |= dmask << shift;
            pval |= (uint32_t)S.misc[4] << shift;
            kk -= S.misc[5];
            mb = S.misc[6];
            sel_sync();
            if (kk == mb || mb <= kBoundary || shift == 0) break;
            top = shift - 1;
        }
        general = kk != mb && mb > kBoundary;
    }
    if (general) {
        uint32_t tau, tau2 = 0u;
        int need, eq;
        sel_radix(
            S, n, k, [&](int) { return true; }, [&](int j) { return S.rk[j]; }, tau, need, eq);
        const bool all = need == eq;
        if (!all) {
            int need2, eq2;
            sel_radix(
                S, n, need, [&](int j) { return S.rk[j] == tau; }, [&](int j) { return ~(uint32_t)S.ri[j]; },
                tau2, need2, eq2);
        }
        return sel_compact(S, n, k, [&](uint32_t u, int32_t ix) {
            return u > tau || (u == tau && (all || ~(uint32_t)ix >= tau2));
        });
    }
    // boundary group: kk of its mb entries are kept, ranked exactly
    uint32_t kstar = 0u;
    int32_t istar = 0x7fffffff;
    const bool whole = kk == mb;
    if (!whole) {
        uint32_t *bk = S.hist;
        int32_t *bi = reinterpret_cast<int32_t *>(S.hist + kBoundary);
        if (S.st == 0) S.misc[7] = 0;
        sel_sync();
        for (int j = S.st; j < n; j += kSelT) {
            const uint32_t u = S.rk[j];
            if ((u & pmask) == pval) {
                const int p = atomicAdd(&S.misc[7], 1);
                bk[p] = u;
                bi[p] = S.ri[j];
            }
        }
        sel_sync();
        for (int i = S.st; i < mb; i += kSelT) {
            const uint32_t ki = bk[i];
            const int32_t ii = bi[i];
            int r = 0;
            for (int j = 0; j < mb; ++j) r += before(bk[j], bi[j], ki, ii);
            if (r == kk - 1) {
                um[14] = ki;
                S.misc[15] = ii;
            }
        }
        sel_sync();
        kstar = um[14];
        istar = S.misc[15];
        sel_sync();
    }
    return sel_compact(S, n, k, [&](uint32_t u, int32_t ix) {
        const uint32_t m = u & pmask;
        return m > pval || (m == pval && (whole || !before(kstar, istar, u, ix)));
    });
}

// The same reduction with the keys held in registers (n <= kRegKeys *
// kSelT): one shared-memory read of the candidates, one histogram pass per
// level, and the survivors written back in place after all reads are done.
constexpr int kRegKeys = 8;
__device__ uint32_t sel_reduce(const Sel &S, int n, int k) {
    if (n > kRegKeys * kSelT) return sel_reduce_smem(S, n, k);
    const int st = S.st, lane = st & 31, w = st >> 5;
    unsigned *um = reinterpret_cast<unsigned *>(S.misc);
    uint32_t u[kRegKeys];
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int q = 0; q < kRegKeys; ++q) {
        const int j = st + q * kSelT;
        u[q] = j < n ? S.rk[j] : 0u;
        if (j < n) {
            lo = min(lo, u[q]);
            hi = max(hi, u[q]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
        um[48 + w] = lo;
        um[56 + w] = hi;
    }
    if (st == 0) S.misc[7] = 0;  // boundary-group counter
    sel_sync();
#pragma unroll
    for (int i = 0; i < kSelWarps; ++i) {
        lo = min(lo, um[48 + i]);
        hi = max(hi, um[56 + i]);
    }
    if (hi == lo) return sel_reduce_smem(S, n, k);  // every key equal: order by index alone
    int top = 31 - __clz((int)(hi ^ lo));
    uint32_t pmask = top == 31 ? 0u : ~((2u << top) - 1u), pval = hi & pmask;
    int kk = k, mb = 0;
    for (;;) {
        const int width = top + 1 < 11 ? top + 1 : 11;
        const int shift = top + 1 - width;
        const uint32_t dmask = (1u << width) - 1u;
        constexpr int BPT = kBins / kSelT;
        uint4 *h4 = reinterpret_cast<uint4 *>(S.hist);
#pragma unroll
        for (int q = 0; q < BPT / 4; ++q) h4[st * (BPT / 4) + q] = make_uint4(0u, 0u, 0u, 0u);
        sel_sync();
#pragma unroll
        for (int q = 0; q < kRegKeys; ++q)
            if (st + q * kSelT < n && (u[q] & pmask) == pval) atomicAdd(&S.hist[(u[q] >> shift) & dmask], 1u);
        sel_sync();
        // descending scan: thread st owns bins [kBins - BPT (st+1), kBins - BPT st)
        const int bb = kBins - BPT * (st + 1);
        int cnt[BPT];
        int sum = 0;
#pragma unroll
        for (int q = 0; q < BPT; ++q) {
            cnt[q] = (int)S.hist[bb + BPT - 1 - q];
            sum += cnt[q];
        }
        int tot;
        int ex = sel_scan(sum, S.misc + 16, st, tot);
#pragma unroll
        for (int q = 0; q < BPT; ++q) {
            if (ex < kk && ex + cnt[q] >= kk) {
                S.misc[4] = bb + BPT - 1 - q;
                S.misc[5] = ex;
                S.misc[6] = cnt[q];
            }
            ex += cnt[q];
        }
        sel_sync();
        pmask |= dmask << shift;
        pval |= (uint32_t)S.misc[4] << shift;
        kk -= S.misc[5];
        mb = S.misc[6];
        if (kk == mb || mb <= kBoundary || shift == 0) break;
        top = shift - 1;
    }
    const bool whole = kk == mb;
    if (!whole && mb > kBoundary) return sel_reduce_smem(S, n, k);  // a large group of equal keys
    uint32_t kstar = 0u;
    int32_t istar = 0x7fffffff;
    if (!whole) {
        // boundary group: gather it (keys from registers) and rank it exactly
        uint32_t *bk = S.hist;
        int32_t *bi = reinterpret_cast<int32_t *>(S.hist + kBoundary);
#pragma unroll
        for (int q = 0; q < kRegKeys; ++q) {
            const int j = st + q * kSelT;
            if (j < n && (u[q] & pmask) == pval) {
                const int p = atomicAdd(&S.misc[7], 1);
                bk[p] = u[q];
                bi[p] = S.ri[j];
            }
        }
        sel_sync();
        if (st < mb) {
            const uint32_t ki = bk[st];
            const int32_t ii = bi[st];
            int r = 0;
            for (int j = 0; j < mb; ++j) r += before(bk[j], bi[j], ki, ii);
            if (r == kk - 1) {
                um[14] = ki;
                S.misc[15] = ii;
            }
        }
        sel_sync();
        kstar = um[14];
        istar = S.misc[15];
    }
    // compaction: read the kept indices, scan the counts, write in place
    int32_t ix[kRegKeys];
    unsigned keep = 0u;
    int c = 0;
    uint32_t kmin = 0xffffffffu;
#pragma unroll
    for (int q = 0; q < kRegKeys; ++q) {
        const int j = st + q * kSelT;
        ix[q] = 0;
        if (j < n) {
            const uint32_t m = u[q] & pmask;
            bool kp = m > pval;
            if (m == pval) {
                ix[q] = S.ri[j];
                kp = whole || !before(kstar, istar, u[q], ix[q]);
            } else if (kp) {
                ix[q] = S.ri[j];
            }
            if (kp) {
                keep |= 1u << q;
                ++c;
                kmin = min(kmin, u[q]);
            }
        }
    }
    int tot;
    int pos = sel_scan(c, S.misc + 16, st, tot);  // its barriers also end every read above
#pragma unroll
    for (int q = 0; q < kRegKeys; ++q) {
        if (keep & (1u << q)) {
            S.rk[pos] = u[q];
            S.ri[pos] = ix[q];
            ++pos;
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
    if (lane == 0) um[48 + w] = kmin;
    sel_sync();
#pragma unroll
    for (int i = 0; i < kSelWarps; ++i) kmin = min(kmin, um[48 + i]);
    sel_sync();
    return kmin;
}

// Mid-segment cut (n <= kRegKeys * kSelT): one histogram of the keys over
// [lo, hi] (the range the appends tracked) in 2048 equal bins, then keep the
// bins at and above the one holding the k-th key.  At least k kept keys are
// strictly above the returned threshold-1 edge, so a later token (higher
// index) whose key is at or below the threshold can never enter the top k;
// the kept set exceeds k by at most the population of one fine bin.  Returns
// the threshold (keys > it survive) and sets `kept`.
__device__ uint32_t sel_trim(const Sel &S, int n, int k, uint32_t lo, uint32_t hi, int &kept) {
    const int st = S.st, lane = st & 31;
    uint32_t u[kRegKeys];
#pragma unroll
    for (int q = 0; q < kRegKeys; ++q) {
        const int j = st + q * kSelT;
        u[q] = j < n ? S.rk[j] : 0u;
    }
    const uint32_t span = hi - lo;
    const int bits = span == 0u ? 0 : 32 - __clz((int)span);
    const int sh = bits > 11 ? bits - 11 : 0;
    constexpr int BPT = kBins / kSelT;
    uint4 *h4 = reinterpret_cast<uint4 *>(S.hist);
#pragma unroll
    for (int q = 0; q < BPT / 4; ++q) h4[st * (BPT / 4) + q] = make_uint4(0u, 0u, 0u, 0u);
    sel_sync();
#pragma unroll
    for (int q = 0; q < kRegKeys; ++q)
        if (st + q * kSelT < n && u[q] >= lo) atomicAdd(&S.hist[min((u[q] - lo) >> sh, (uint32_t)(kBins - 1))], 1u);
    sel_sync();
    const int bb = kBins - BPT * (st + 1);
    int cnt[BPT];
    int sum = 0;
#pragma unroll
    for (int q = 0; q < BPT; ++q) {
        cnt[q] = (int)S.hist[bb + BPT - 1 - q];
        sum += cnt[q];
    }
    int tot;
    int ex = sel_scan(sum, S.misc + 16, st, tot);
#pragma unroll
    for (int q = 0; q < BPT; ++q) {
        if (ex < k && ex + cnt[q] >= k) S.misc[4] = bb + BPT - 1 - q;
        ex += cnt[q];
    }
    sel_sync();
    const uint32_t edge = lo + ((uint32_t)S.misc[4] << sh);  // lowest key of the k-th key's bin
    if (tot < k || edge == 0u) {  // fewer than k keys in range, or nothing below key 0 to cut
        kept = n;
        sel_sync();
        return 0u;
    }
    const uint32_t thr = edge - 1u;
    int32_t ix[kRegKeys];
    unsigned keep = 0u;
    int c = 0;
#pragma unroll
    for (int q = 0; q < kRegKeys; ++q) {
        const int j = st + q * kSelT;
        ix[q] = 0;
        if (j < n && u[q] > thr) {
            ix[q] = S.ri[j];
            keep |= 1u << q;
            ++c;
        }
    }
    int pos = sel_scan(c, S.misc + 16, st, tot);  // its barriers also end every read above
#pragma unroll
    for (int q = 0; q < kRegKeys; ++q) {
        if (keep & (1u << q)) {
            S.rk[pos] = u[q];
            S.ri[pos] = ix[q];
            ++pos;
        }
    }
    (void)lane;
    kept = tot;
    sel_sync();
    return thr;
}

// Sort a[0..n) ascending (bitonic over npow2(n), padded with INT_MAX).
__device__ void sel_sort(int32_t *a, int n, int st) {
    const int P = npow2(n < 1 ? 1 : n);
    for (int j = n + st; j < P; j += kSelT) a[j] = 0x7fffffff;
    sel_sync();
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = st; i < P / 2; i += kSelT) {
                const int lo = 2 * stride * (i / stride) + (i % stride);
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const int32_t x = a[lo], y = a[hi];
                if ((x > y) == up) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
            sel_sync();
        }
    }
}

// Tile cursor over a CTA's range: (b,h) row and tile index within the row of
// the current tile, advanced without divisions.  An epoch ends after E tiles
// of one segment, at a segment end, or at the end of the range; consumers and
// selector walk the range identically.
struct Cursor {
    int bh, t, tpb;
    __device__ void next() {
        if (++t == tpb) {
            t = 0;
            ++bh;
        }
    }
    __device__ bool seg_last(int i, int ntiles) const { return i == ntiles - 1 || t + 1 == tpb; }
};

// Ring position: stage of the current tile and the parity of its phase.
struct RingPos {
    int s = 0, n;
    uint32_t ph = 0u;
    __device__ explicit RingPos(int stages) : n(stages) {}
    __device__ void next() {
        if (++s == n) {
            s = 0;
            ph ^= 1u;
        }
    }
};

// End of a segment (selector).  The segment takes its arrival ticket first:
// the last segment of the (b,h) to arrive merges the other segments'
// published candidates into its own candidate set (nothing published);
// every other segment cuts to k, publishes k slots (index -1 marks an empty
// slot), and counts itself published.  The last one waits (bounded) for the
// publish counts of segments that took their tickets before it, which are
// running and publish without waiting on anything; while some are still
// cutting, it cuts its own set to k, which also gives a threshold that
// filters the merged entries.  The merge loads the slots of up to kMergeSegs
// segments at once (one memory latency per group), as many groups as the
// candidate capacity holds between exact cuts.  Returns the selection's size
// when this CTA merged it, else -1.  counters[bh] = tickets, counters[BH +
// bh] = published segments; the merger resets both.
constexpr int kMergeSegs = 8;
__device__ int sel_finish(const ScanArgs &a, const Sel &S, int n, int bh, long long cta, int ept, int cap) {
    const int BH = a.B * a.Hkv;
    const int tpb = a.tiles_per_bh;
    const long long first = (long long)bh * tpb;
    const long long c_first = ((first + 1) * a.grid - 1) / a.total_tiles;
    const long long c_last = ((first + tpb) * a.grid - 1) / a.total_tiles;
    const int slot = (int)(cta - c_first), nseg = (int)(c_last - c_first + 1);
    if (S.st == 0) S.misc[9] = nseg == 1 || atomicAdd(&a.counters[bh], 1u) == (unsigned)(nseg - 1);
    sel_sync();
    const bool last = S.misc[9] != 0;
    sel_sync();
    if (!last) {
        if (n > a.k) {
            sel_reduce(S, n, a.k);
            n = a.k;
        }
        const size_t cb = ((size_t)bh * a.max_seg + slot) * a.k;
        for (int j = S.st; j < a.k; j += kSelT) {
            a.cand_key[cb + j] = j < n ? S.rk[j] : 0u;
            a.cand_idx[cb + j] = j < n ? S.ri[j] : -1;
        }
        __threadfence();
        sel_sync();
        if (S.st == 0) atomicAdd(&a.counters[BH + bh], 1u);
        return -1;
    }
    int m = n;
    bool valid = false;
    uint32_t thr = 0u;
    if (nseg > 1) {
        if (S.st == 0) S.misc[47] = (int)__ldcg(a.counters + BH + bh);
        sel_sync();
        if (S.misc[47] < nseg - 1 && m > a.k) {  // others still cutting: cut this set meanwhile
            thr = sel_reduce(S, m, a.k);
            valid = true;
            m = a.k;
        }
        if (S.st == 0 && !flag_wait_bounded(a.counters + BH + bh, (unsigned)(nseg - 1)) && a.status)
            atomicOr(a.status, (uint32_t)JSSA_DEV_TIMEOUT);
        __threadfence();
    }
    // merge the other segments' slots; equal keys stay candidates (order is arbitrary)
    if (nseg > 1) {
        sel_sync();
        if (S.st == 0) S.misc[3] = m;
        sel_sync();
    }
    const int lane = S.st & 31;
    const size_t rowbase = (size_t)bh * a.max_seg * a.k;
    // a wave holds at most what the register-resident cut takes (the cut of
    // a larger set reads shared memory on every level: several times slower)
    const int wcap = max(min(cap, kRegKeys * kSelT), 2 * a.k);
    for (int s0 = 0; nseg > 1 && s0 < nseg;) {
        int nb = (wcap - m) / a.k;  // segments that fit before the next exact cut
        if (nb < 1) {
            thr = sel_reduce(S, m, a.k);
            valid = true;
            m = a.k;
            if (S.st == 0) S.misc[3] = m;
            sel_sync();
            nb = (wcap - m) / a.k;
        }
        const int s_end = min(nseg, s0 + nb);
        for (int g0 = s0; g0 < s_end; g0 += kMergeSegs) {
            const int s1 = min(s_end, g0 + kMergeSegs);
            for (int j0 = 0; j0 < a.k; j0 += kSelT) {
                const int j = j0 + S.st;
                uint32_t u[kMergeSegs];
                int32_t ix[kMergeSegs];
#pragma unroll
                for (int q = 0; q < kMergeSegs; ++q) {  // every load of the group in flight at once
                    const int sg = g0 + q;
                    u[q] = 0u;
                    ix[q] = -1;
                    if (sg < s1 && sg != slot && j < a.k) {
                        const size_t o = rowbase + (size_t)sg * a.k + j;
                        u[q] = __ldcg(a.cand_key + o);
                        ix[q] = __ldcg(a.cand_idx + o);
                    }
                }
#pragma unroll
                for (int q = 0; q < kMergeSegs; ++q) {
                    const bool take = ix[q] >= 0 && (!valid || u[q] >= thr);
                    const unsigned msk = __ballot_sync(0xffffffffu, take);
                    int b0 = 0;
                    if (msk) {
                        const int ld = __ffs(msk) - 1;
                        if (lane == ld) b0 = atomicAdd(&S.misc[3], __popc(msk));
                        b0 = __shfl_sync(0xffffffffu, b0, ld);
                    }
                    if (take) {
                        const int p = b0 + __popc(msk & lane_lt());
                        S.rk[p] = u[q];
                        S.ri[p] = ix[q];
                    }
                }
            }
        }
        s0 = s_end;
        sel_sync();
        m = S.misc[3];
        sel_sync();
    }
    if (m > a.k) {
        sel_reduce(S, m, a.k);
        m = a.k;
    }
    if (m <= kSelT) {
        // bitonic sort, one value per selector thread (pads sort above every
        // index): partners within a warp by shuffle, across warps through
        // shared memory (the histogram is free after the cut)
        int32_t v = S.st < m ? S.ri[S.st] : 0x7fffffff;
        int32_t *xch = reinterpret_cast<int32_t *>(S.hist);
#pragma unroll
        for (int kk = 2; kk <= kSelT; kk <<= 1) {
#pragma unroll
            for (int j = kk >> 1; j > 0; j >>= 1) {
                int32_t o;
                if (j >= 32) {
                    xch[S.st] = v;
                    sel_sync();
                    o = xch[S.st ^ j];
                    sel_sync();
                } else {
                    o = __shfl_xor_sync(0xffffffffu, v, j);
                }
                const bool asc = (S.st & kk) == 0, lower = (S.st & j) == 0;
                v = lower == asc ? min(v, o) : max(v, o);
            }
        }
        if (S.st < m) S.si[S.st] = v;
        sel_sync();
    } else if (m <= 2 * kSelT) {
        // ascending order by rank: the indices are distinct, so each entry's
        // place is the number of smaller ones (broadcast reads, one barrier)
        const int m4 = (m + 3) & ~3;
        if (S.st < m4 - m) S.ri[m + S.st] = 0x7fffffff;  // pads count as larger than every index
        sel_sync();
        const int4 *r4 = reinterpret_cast<const int4 *>(S.ri);
        for (int j = S.st; j < m; j += kSelT) {
            const int32_t v = S.ri[j];
            int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
#pragma unroll 4
            for (int i = 0; i < m4 / 4; ++i) {
                const int4 w = r4[i];
                c0 += w.x < v;
                c1 += w.y < v;
                c2 += w.z < v;
                c3 += w.w < v;
            }
            S.si[(c0 + c1) + (c2 + c3)] = v;
        }
        sel_sync();
    } else {
        for (int j = S.st; j < m; j += kSelT) S.si[j] = S.ri[j];
        sel_sync();
        sel_sort(S.si, m, S.st);
    }
    for (int j = S.st; j < a.k; j += kSelT) a.idx_out[(size_t)bh * a.k + j] = j < m ? S.si[j] : -1;
    if (S.st == 0) {
        if (a.count_out) a.count_out[bh] = m;
        a.counters[bh] = 0u;
        a.counters[BH + bh] = 0u;
    }
    sel_sync();
    return m;
}

// ------------------------------------------------------ fused decode step ---
struct StreamArgs {
    ScanArgs s;
    StepExtra x;
};

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Barrier of the consumer warps alone.
__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync 2, %0;" ::"n"(kCons) : "memory"); }

// part[j][c] = sum over the c-th chunk of kChunkD inputs of xs[i] * P[i][j]
// (an fma chain from 0), the fixed order of the projection and append
// kernels, so every path yields bit-identical rows.
template <int R>
__device__ void sel_dots(const float *xs, const float *P, int d, float *part, int st) {
    const int nch = d / kChunkD;
    for (int p = st; p < R * nch; p += kSelT) {
        const int c = p / R, j = p - c * R;
        const float *xr = xs + c * kChunkD;
        const float *pc = P + (size_t)(c * kChunkD) * R + j;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < kChunkD; ++i) acc = fmaf(xr[i], __ldg(pc + (size_t)i * R), acc);
        part[(size_t)j * nch + c] = acc;
    }
    sel_sync();
}

__device__ __forceinline__ float sum_parts(const float *part, int j, int nch) {
    float s = part[(size_t)j * nch];
    for (int c = 1; c < nch; ++c) s += part[(size_t)j * nch + c];
    return s;
}

// Folded query of row bh: qb = P_h^T (sum of the group's queries, in head order).
// A work pair (chunk c of kChunkD inputs; outputs j and j + R/2) issues the
// loads of its two P column slices before the fold's query loads, so both
// are in flight together; the fold goes through shared memory (one dim per
// thread).  The arithmetic order matches the projection kernel's (head sum
// from 0 in head order, fma chain per chunk, chunk partials left to right),
// so both give the same bits.
template <int R>
__device__ void sel_project(const StepExtra &x, int Hkv, int bh, float *qb, float *xs, float *part, int st) {
    const int b = bh / Hkv, h = bh - b * Hkv, G = x.G, d = x.d;
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(x.q) + ((size_t)b * x.Hq + (size_t)h * G) * d;
    const float *P = x.P + (size_t)h * d * R;
    const int nch = d / kChunkD;
    constexpr int RH = R / 2;
    const int npair = RH * nch;
    float pv0[kChunkD], pv1[kChunkD];
    auto load_pair = [&](int pp) {
        const int c = pp / RH, j = pp - c * RH;
#pragma unroll
        for (int i = 0; i < kChunkD; ++i) {
            pv0[i] = __ldg(P + (size_t)(c * kChunkD + i) * R + j);
            pv1[i] = __ldg(P + (size_t)(c * kChunkD + i) * R + j + RH);
        }
    };
    if (st < npair) load_pair(st);
    for (int i = st; i < d; i += kSelT) {
        float sum = 0.f;
#pragma unroll 4
        for (int g = 0; g < G; ++g) sum += __bfloat162float(q[(size_t)g * d + i]);
        xs[i] = sum;
    }
    sel_sync();
    for (int pp = st; pp < npair; pp += kSelT) {
        if (pp != st) load_pair(pp);
        const int c = pp / RH, j = pp - c * RH;
        const float *xr = xs + c * kChunkD;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int i = 0; i < kChunkD; ++i) {
            a0 = fmaf(xr[i], pv0[i], a0);
            a1 = fmaf(xr[i], pv1[i], a1);
        }
        part[(size_t)j * nch + c] = a0;
        part[(size_t)(j + RH) * nch + c] = a1;
    }
    sel_sync();
    for (int j = st; j < R; j += kSelT) qb[j] = sum_parts(part, j, nch);
    sel_sync();
}

// New row of the low-rank cache: Kt[b,h,pos,:] = bf16(K[b,pos,h,:] . P_h),
// stored to global memory and fenced for the bulk copies that read it.
template <int R>
__device__ void sel_append(const ScanArgs &a, const StepExtra &x, int bh, int pos, float *xs, float *part, int st) {
    const int b = bh / a.Hkv, h = bh - b * a.Hkv, d = x.d;
    const __nv_bfloat16 *K = static_cast<const __nv_bfloat16 *>(x.K);
    for (int i = st; i < d; i += kSelT) xs[i] = __bfloat162float(K[(((size_t)b * a.T_cap + pos) * a.Hkv + h) * d + i]);
    sel_sync();
    sel_dots<R>(xs, x.P + (size_t)h * d * R, d, part, st);
    __nv_bfloat16 *Kt = static_cast<__nv_bfloat16 *>(const_cast<void *>(a.src));
    for (int j = st; j < R; j += kSelT) {
        const __nv_bfloat16 v = __float2bfloat16_rn(sum_parts(part, j, d / kChunkD));
        Kt[((size_t)bh * a.T_cap + pos) * R + j] = v;
        if (a.norms) {
            const float f = __bfloat162float(v);
            xs[j] = f * f;  // the input row is no longer read (sel_dots ended on a barrier)
        }
    }
    if (a.norms) {
        // screening bound of the row's block raised to cover the new row
        sel_sync();
        if (st == 0) {
            float ss = 0.f;
            for (int j = 0; j < R; ++j) ss += xs[j];
            atomicMax(reinterpret_cast<int *>(a.norms + (size_t)bh * a.norm_blocks + pos / JSSA_NORM_BLOCK),
                      __float_as_int(sqrtf(ss)));
        }
    }
    fence_proxy_async_global();
    sel_sync();
}

// ---- attention epilogue on the tensor cores (mma.sync m16n8k16, bf16) ----
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Attention of the G query heads of row bh over its kb selected tokens, by
// the 16 consumer warps (ct = consumer thread index), as two small matrix
// products on the tensor cores with the heads padded to 16 rows:
//   S[16 x n] = Q[16 x D] . K_sel^T      (fp32 accumulation of bf16 products)
//   O[16 x D] = P[16 x n] . V_sel        (P = softmax weights rounded to bf16)
// The selected K and V rows of a chunk of tokens are staged by 16-byte
// asynchronous copies straight from the cache into `buf` (16-byte chunks
// XOR-swizzled by token so that ldmatrix reads are conflict-free).  Each
// warp keeps the logits of its 8-token tiles in registers; the softmax runs
// in fp32 in the log2 domain, online across chunks, with the running max
// and each thread's share of the normaliser (sums of the bf16 weights the
// second product uses) in registers: three barriers per chunk.
template <int D>
__device__ void fused_attend(const ScanArgs &a, const StepExtra &x, int bh, int kb, unsigned char *buf,
                             size_t buf_bytes, int ct) {
    constexpr int ROWB = D * 2;         // bytes of a K (or V) row
    constexpr int CPR = ROWB / 16;      // 16-byte chunks per row
    constexpr int ROW2 = 2 * ROWB;      // staged K row then V row
    constexpr int QSTR = ROWB + 16;     // padded row stride of Q (bytes)
    constexpr int NTD = D / 8;          // 8-wide output tiles
    constexpr int TPW = NTD / kConsWarps;  // output tiles per warp (1 or 2)
    constexpr int TT = 2;                  // 8-token logit tiles per warp and chunk
    constexpr int CHMAX = kConsWarps * 8 * TT;
    static_assert(NTD % kConsWarps == 0, "head width");
    const int w = ct >> 5, lane = ct & 31, gid = lane >> 2, tig = lane & 3;
    const int G = x.G;
    const int b = bh / a.Hkv, h = bh - b * a.Hkv;
    // shared memory carve-up
    unsigned char *q_s = buf;                                  // [16][QSTR]
    float *red = reinterpret_cast<float *>(buf + 16 * QSTR);   // [kConsWarps][16] partial max, then sums
    int32_t *idx_s = reinterpret_cast<int32_t *>(red + kConsWarps * 16);  // the token list [kb], staged once
    unsigned char *p_s = reinterpret_cast<unsigned char *>(idx_s + ((kb + 3) & ~3));
    const size_t fixed = 16 * QSTR + (size_t)kConsWarps * 16 * 4 + (size_t)((kb + 3) & ~3) * 4;
    // chunk of CH tokens (a multiple of 16): P [16][CH] bf16 (+16 B per row),
    // then CH staged K/V row pairs
    int CH = (int)((buf_bytes - fixed - 16 * 16 - 128) / (ROW2 + 32)) & ~15;
    const int need = (kb + 15) & ~15;
    if (CH > need) CH = need;
    if (CH > CHMAX) CH = CHMAX;
    if (CH < 16) CH = 16;
    const int PSTR = CH * 2 + 16;  // padded row stride of P (bytes)
    unsigned char *stage = p_s + (((size_t)16 * PSTR + 127) & ~(size_t)127);
    const uint32_t q_a = smem_u32(q_s), p_a = smem_u32(p_s), st_a = smem_u32(stage);

    // Q: the G heads' queries as bf16 rows, zero rows up to 16
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(x.q) + ((size_t)b * x.Hq + (size_t)h * G) * D;
    for (int i = ct; i < 16 * CPR; i += kCons) {
        const int g = i / CPR, c = i - g * CPR;
        cp_async16(q_s + g * QSTR + c * 16, g < G ? qg + (size_t)g * D + c * 8 : qg, g < G ? 16u : 0u);
    }
    float o[TPW][4];
#pragma unroll
    for (int u = 0; u < TPW; ++u) o[u][0] = o[u][1] = o[u][2] = o[u][3] = 0.f;
    float mrun[2] = {-INFINITY, -INFINITY};  // running max of rows gid, gid + 8 (log2 domain)
    float lpart[2] = {0.f, 0.f};             // this thread's share of their normalisers
    // the token list in shared memory: one coalesced read instead of a
    // dependent global load before every staging copy
    const int32_t *idx_g = a.idx_out + (size_t)bh * a.k;
    for (int j = ct; j < kb; j += kCons) idx_s[j] = idx_g[j];
    cons_sync();
    const int32_t *idx = idx_s;
    const __nv_bfloat16 *Kc = static_cast<const __nv_bfloat16 *>(x.K);
    const __nv_bfloat16 *Vc = static_cast<const __nv_bfloat16 *>(x.V);

    for (int c0 = 0; c0 < kb; c0 += CH) {
        const int n = min(CH, kb - c0), n16 = (n + 15) & ~15;
        // stage K and V rows (zero rows past n), chunk c of token t at c ^ (t & 7)
        for (int p = ct; p < n16 * 2 * CPR; p += kCons) {
            const int t = p / (2 * CPR), rem = p - t * 2 * CPR;
            const int isv = rem >= CPR, c = rem - isv * CPR;
            int tok = 0;
            bool ok = false;
            if (t < n) {
                tok = idx[c0 + t];
                ok = (unsigned)tok < (unsigned)a.T_cap;
            }
            const __nv_bfloat16 *src =
                (isv ? Vc : Kc) + (((size_t)b * a.T_cap + (ok ? tok : 0)) * a.Hkv + h) * D + c * 8;
            cp_async16(stage + (size_t)t * ROW2 + isv * ROWB + ((c ^ (t & 7)) * 16), src, ok ? 16u : 0u);
        }
        cp_async_commit();
        cp_async_wait<0>();
        cons_sync();

        // S = Q K^T: warp w takes 8-token tiles w and w + 16 (logits stay in registers)
        const int ntt = n16 / 8;
        float sv[TT][4];
        float wmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int u = 0; u < TT; ++u) {
            const int nt = w + u * kConsWarps;
            sv[u][0] = sv[u][1] = sv[u][2] = sv[u][3] = -INFINITY;
            if (nt < ntt) {
                float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t a0, a1, a2, a3, b0, b1;
                    // A: rows (lane % 16), k chunk 2*ks + lane / 16
                    ldsm_x4(q_a + (lane & 15) * QSTR + (2 * ks + (lane >> 4)) * 16, a0, a1, a2, a3);
                    // B: token rows nt*8 + lane % 8, k chunk 2*ks + (lane / 8) % 2
                    const int t = nt * 8 + (lane & 7), c = 2 * ks + ((lane >> 3) & 1);
                    ldsm_x2(st_a + t * ROW2 + ((c ^ (t & 7)) * 16), b0, b1);
                    mma_bf16_16816(sc, a0, a1, a2, a3, b0, b1);
                }
                // scaled logits: rows gid, gid + 8; columns 2 tig, 2 tig + 1 of the tile
                const int tc = nt * 8 + 2 * tig;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int row = e < 2 ? gid : gid + 8, col = tc + (e & 1);
                    sv[u][e] = (row < G && col < n) ? sc[e] * x.scale_log2 : -INFINITY;
                }
                wmax[0] = fmaxf(wmax[0], fmaxf(sv[u][0], sv[u][1]));
                wmax[1] = fmaxf(wmax[1], fmaxf(sv[u][2], sv[u][3]));
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            wmax[r] = fmaxf(wmax[r], __shfl_xor_sync(0xffffffffu, wmax[r], 1));
            wmax[r] = fmaxf(wmax[r], __shfl_xor_sync(0xffffffffu, wmax[r], 2));
        }
        if (tig == 0) {
            red[w * 16 + gid] = wmax[0];
            red[w * 16 + gid + 8] = wmax[1];
        }
        cons_sync();
        // the chunk's row maxima (every thread of a row computes the same
        // values) and the correction of what came before
        float corr[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            float mx = mrun[r];
#pragma unroll
            for (int i = 0; i < kConsWarps; ++i) mx = fmaxf(mx, red[i * 16 + gid + 8 * r]);
            corr[r] = mrun[r] == -INFINITY ? 0.f : exp2f(mrun[r] - mx);
            mrun[r] = mx;
        }
        // weights: P = bf16(exp2(s - m)) into shared memory; this thread's row
        // sums of the rounded weights
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int u = 0; u < TT; ++u) {
            const int nt = w + u * kConsWarps;
            if (nt < ntt) {
                const int tc = nt * 8 + 2 * tig;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float m = mrun[r];
                    const float w0 = (sv[u][2 * r] == -INFINITY || m == -INFINITY) ? 0.f : exp2f(sv[u][2 * r] - m);
                    const float w1 =
                        (sv[u][2 * r + 1] == -INFINITY || m == -INFINITY) ? 0.f : exp2f(sv[u][2 * r + 1] - m);
                    const __nv_bfloat162 pw = __floats2bfloat162_rn(w0, w1);
                    rs[r] += __low2float(pw) + __high2float(pw);
                    *reinterpret_cast<__nv_bfloat162 *>(p_s + (gid + 8 * r) * PSTR + tc * 2) = pw;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) lpart[r] = lpart[r] * corr[r] + rs[r];
        cons_sync();  // P complete (and every read of the maxima done)
        // O = O * corr + P V: warp w takes output tiles w, w + 16
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
            o[u][0] *= corr[0];
            o[u][1] *= corr[0];
            o[u][2] *= corr[1];
            o[u][3] *= corr[1];
            const int dt = w + u * kConsWarps;  // 8-dim tile = one 16-byte chunk of the V row
            for (int ks = 0; ks < n16 / 16; ++ks) {
                uint32_t a0, a1, a2, a3, b0, b1;
                ldsm_x4(p_a + (lane & 15) * PSTR + (2 * ks + (lane >> 4)) * 16, a0, a1, a2, a3);
                const int t = ks * 16 + (lane & 15);
                ldsm_x2_t(st_a + t * ROW2 + ROWB + ((dt ^ (t & 7)) * 16), b0, b1);
                mma_bf16_16816(o[u], a0, a1, a2, a3, b0, b1);
            }
        }
        if (c0 + CH < kb) cons_sync();  // before the next chunk overwrites the stage and P
    }
    // normalisers: the four threads of a row in a warp, then the warps in order
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        lpart[r] += __shfl_xor_sync(0xffffffffu, lpart[r], 1);
        lpart[r] += __shfl_xor_sync(0xffffffffu, lpart[r], 2);
    }
    if (tig == 0) {
        red[w * 16 + gid] = lpart[0];
        red[w * 16 + gid + 8] = lpart[1];
    }
    cons_sync();
    // out = O / l, lse = (m + log2 l) ln 2, rows g < G
    const size_t row0 = (size_t)b * x.Hq + (size_t)h * G;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int g = gid + 8 * hr;
        if (g >= G) continue;
        float l = 0.f;
#pragma unroll
        for (int i = 0; i < kConsWarps; ++i) l += red[i * 16 + g];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16 *op = static_cast<__nv_bfloat16 *>(x.out) + (row0 + g) * D;
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
            const int col = (w + u * kConsWarps) * 8 + 2 * tig;
            *reinterpret_cast<__nv_bfloat162 *>(op + col) =
                __floats2bfloat162_rn(o[u][2 * hr] * inv, o[u][2 * hr + 1] * inv);
        }
        if (w == 0 && tig == 0 && x.lse)
            x.lse[row0 + g] = l > 0.f ? (mrun[hr] + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
    cons_sync();
}

// D = 0: the selection alone.  D > 0: the fused decode step with head width D.
template <int SRC, int R, int D>
__global__ void __launch_bounds__(kThreads, 1) stream_select_kernel(StreamArgs A) {
    const ScanArgs &a = A.s;
    constexpr bool FUSED = D > 0;
    using KT = typename std::conditional<SRC == SRC_KT_FP32, float, __nv_bfloat16>::type;
    constexpr int ES = SRC == SRC_KT_FP32 ? 4 : 2;
    constexpr int ROWB = R * ES;                  // bytes per token
    constexpr int TPB = ROWB > 64 ? 64 : ROWB;    // bytes of a token per thread
    constexpr int LPT = ROWB / TPB;               // lanes per token
    constexpr int CPT = TPB / 16;                 // 16-byte chunks per thread
    constexpr int EPL = 16 / ES;                  // elements per chunk
    constexpr int TILE = kTile / ROWB;            // tokens per tile
    constexpr int TPP = kCons / LPT;              // tokens per pass
    constexpr int PASSES = TILE / TPP;
    constexpr int QN = CPT * EPL;
    constexpr int E = TILE >= kEpochTokens ? 1 : kEpochTokens / TILE;  // tiles per epoch
    constexpr int EPT = E * TILE;                                      // tokens per epoch
    static_assert(LPT >= 1 && LPT <= 32 && (LPT & (LPT - 1)) == 0, "lanes per token");
    static_assert(CPT >= 1 && CPT <= 4, "chunks per thread");
    static_assert(PASSES >= 1 && TILE % TPP == 0, "tile / pass");

    extern __shared__ __align__(128) unsigned char smem[];
    const int S_ = a.nstages;
    const StreamSmem L = stream_smem(S_, EPT, a.cap, a.k, FUSED ? R : 0, a.nb_cap);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + S_;
    uint64_t *efull = empty + S_;  // [kEB]
    uint64_t *efree = efull + kEB; // [kEB]
    uint64_t *qready = efree + kEB;       // fused: folded query of row i in shared memory [kMaxRows]
    uint64_t *aready = qready + kMaxRows;  // fused: new low-rank rows stored
    uint64_t *nbready = aready + 1;        // screening: staged tile bounds written
    uint32_t *ek = reinterpret_cast<uint32_t *>(smem + L.ek);
    int32_t *ei = reinterpret_cast<int32_t *>(smem + L.ei);
    int *misc = reinterpret_cast<int *>(smem + L.misc);
    volatile int *abort_flag = misc;
    volatile unsigned long long *thr_word = reinterpret_cast<volatile unsigned long long *>(misc + 32);

    const int tid = threadIdx.x, lane = tid & 31;
    const long long cta = blockIdx.x;
    const long long x_begin = cta * a.total_tiles / a.grid;
    const long long x_end = (cta + 1) * a.total_tiles / a.grid;
    const int ntiles = (int)(x_end - x_begin);
    Cursor c0;
    c0.tpb = a.tiles_per_bh;
    c0.bh = (int)(x_begin / c0.tpb);
    c0.t = (int)(x_begin - (long long)c0.bh * c0.tpb);
    const int row0 = c0.bh;
    const int nrows = ntiles > 0 ? (int)((x_end - 1) / c0.tpb) - row0 + 1 : 0;
    float *qb = reinterpret_cast<float *>(smem + L.qb);

    if (tid == 0) {
        for (int s = 0; s < S_; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsWarps);
        }
        for (int p = 0; p < kEB; ++p) {
            mbar_init(&efull[p], kConsWarps);
            mbar_init(&efree[p], 1);
            misc[40 + p] = 0;
        }
        for (int i = 0; i < kMaxRows; ++i) mbar_init(&qready[i], 1);
        mbar_init(aready, 1);
        mbar_init(nbready, 1);
        misc[46] = 0;
        fence_barrier_init();
        misc[0] = 0;
        misc[3] = 0;
        misc[44] = (int)0xffffffffu;
        misc[45] = 0;
        *thr_word = 0ull;
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();

    if (tid >= kProdBase && tid < kConsBase) {
        // ------------------------------------------------------ producer
        // Screening bound of a tile: the largest block norm over the blocks
        // holding its n tokens (tiles and blocks align, or a tile lies in one block).
        auto tile_bound = [&](int bh_, int t0_, int n_) {
            const float *nr = a.norms + (size_t)bh_ * a.norm_blocks + t0_ / JSSA_NORM_BLOCK;
            float m = 0.f;
            for (int j = 0; j * JSSA_NORM_BLOCK < n_; ++j) m = fmaxf(m, __ldcg(nr + j));
            return m;
        };
        float *nbs = reinterpret_cast<float *>(smem + L.nb);
        const int nstaged = a.norms ? min(ntiles, a.nb_cap) : 0;
        if (tid != kProdBase) {
            // the warp's other lanes stage the bounds of the CTA's first
            // nstaged tiles, so that none of their loads sits on the path of
            // the copies (the ring is only a few stages deep)
            for (int i = lane - 1; i < nstaged; i += 31) {
                const int tt = c0.t + i, rr = tt / c0.tpb;  // tile i of the range: row c0.bh + rr
                const int bh_ = c0.bh + rr, t0_ = (tt - rr * c0.tpb) * TILE;
                const int Tb_ = clamp_seq(__ldg(a.seq_lens + bh_ / a.Hkv), a.T_cap, nullptr);
                const float *nr = a.norms + (size_t)bh_ * a.norm_blocks + t0_ / JSSA_NORM_BLOCK;
                const int n_ = min(TILE, Tb_ - t0_);
                float m = 0.f;
#pragma unroll
                for (int j = 0; j < (TILE + JSSA_NORM_BLOCK - 1) / JSSA_NORM_BLOCK; ++j)
                    if (j * JSSA_NORM_BLOCK < n_) m = fmaxf(m, __ldcg(nr + j));
                nbs[i] = m;
            }
            __syncwarp(0xfffffffeu);
            if (lane == 1) mbar_arrive(nbready);
        } else {
            const char *src = static_cast<const char *>(a.src);
            const uint64_t pol = policy_evict_first();
            int issued = 0;
            Cursor cur = c0;
            RingPos rp(S_);
            int Tb = 0, atile = -1;
            bool appended = false;
            bool staged = nstaged == 0;  // staged bounds visible to this thread
            float qn = -1.f;  // ||qbar|| of the current row (screening), -1 while unknown
            for (int i = 0; i < ntiles; ++i, cur.next(), rp.next()) {
                const int s = rp.s;
                const int bh = cur.bh, t0 = cur.t * TILE;
                if (i == 0 || cur.t == 0) {
                    qn = -1.f;
                    Tb = clamp_seq(__ldg(a.seq_lens + bh / a.Hkv), a.T_cap, nullptr);
                    if constexpr (FUSED) {
                        const int pos = __ldg(A.x.pos_begin + bh / a.Hkv);
                        atile = (pos >= 0 && pos < a.T_cap) ? pos / TILE : -1;
                    }
                }
                if (i >= S_ && !wait_or_abort(&empty[s], rp.ph ^ 1u, abort_flag)) {
                    *abort_flag = 1;
                    break;
                }
                bool newrow = false;  // this tile holds the row appended in the prologue
                if (FUSED && !appended && cur.t == atile) {
                    if (!wait_or_abort(aready, 0u, abort_flag)) {
                        *abort_flag = 1;
                        break;
                    }
                    appended = true;
                    newrow = true;
                }
                const int n = min(TILE, Tb - t0);
                // exact screening: skip the tile when ||qbar|| times its blocks'
                // norm bound (inflated for fp32 rounding) cannot beat the key
                // the row's segment already holds k candidates above.  The tile
                // of the new row is not screened: its staged bound may predate
                // the prologue's raise.
                bool skip = false;
                if (a.norms && n > 0 && !newrow) {
                    const bool tforce = t0 < a.n_sink || t0 + TILE > Tb - a.n_recent;
                    const unsigned long long tw = *thr_word;
                    if (!tforce && (uint32_t)(tw >> 32) == (uint32_t)bh + 1u) {
                        if (qn < 0.f) {
                            const float *qp = nullptr;
                            if constexpr (FUSED) {
                                // a test, not a wait: the producer must not stall on the prologue
                                if (mbar_test_wait(&qready[bh - row0], 0u)) qp = qb + (size_t)(bh - row0) * R;
                            } else {
                                qp = a.qproj + (size_t)bh * R;
                            }
                            if (qp) {
                                float ss = 0.f;
                                for (int j = 0; j < R; ++j) {
                                    const float v = FUSED ? qp[j] : __ldcg(qp + j);
                                    ss = fmaf(v, v, ss);
                                }
                                qn = sqrtf(ss);
                            }
                        }
                        float nb = -1.f;
                        if (i < nstaged) {
                            if (!staged) staged = mbar_test_wait(nbready, 0u);
                            if (staged) nb = nbs[i];
                        } else {
                            nb = tile_bound(bh, t0, n);
                        }
                        if (qn >= 0.f && nb >= 0.f) skip = score_key(qn * nb * 1.0001f) <= (uint32_t)tw;
                    }
                }
                misc[80 + s] = skip ? 1 : 0;
                if (n > 0 && !skip) {
                    mbar_arrive_expect_tx(&full[s], (uint32_t)n * ROWB);
                    bulk_g2s(smem + L.ring + (size_t)s * kTile, src + ((size_t)bh * a.T_cap + t0) * ROWB,
                             (uint32_t)n * ROWB, &full[s], pol);
                } else {
                    mbar_arrive(&full[s]);
                    if (skip && a.skip_count) atomicAdd(a.skip_count, 1u);
                }
                issued = i + 1;
            }
            misc[24] = issued;
        }
    } else if (tid >= kConsBase) {
        // ------------------------------------------------------ consumers
        const int ct = tid - kConsBase;  // consumer thread index
        const int sub = ct % LPT;
        const int rot = CPT == 4 ? (lane >> 1) & 3 : (CPT == 2 ? (lane >> 2) & 1 : 0);
        float qreg[QN];
#pragma unroll
        for (int e = 0; e < QN; ++e) qreg[e] = 0.f;
        int Tb = 0, e = 0, epos = 0, p = 0;
        uint32_t eph = 0u;  // use parity of epoch buffer p
        uint32_t tag = 0u;
        Cursor cur = c0;
        RingPos rp(S_);
        for (int i = 0; i < ntiles; ++i, cur.next(), rp.next()) {
            const int bh = cur.bh, t = cur.t, s = rp.s;
            if (i == 0 || t == 0) {
                Tb = clamp_seq(__ldg(a.seq_lens + bh / a.Hkv), a.T_cap, ct == 0 ? a.status : nullptr);
                tag = (uint32_t)bh + 1u;
                if constexpr (FUSED) {
                    // the folded query of this row comes from the selector's prologue
                    const bool qok = __all_sync(0xffffffffu, wait_or_abort(&qready[bh - row0], 0u, abort_flag));
                    if (!qok) {
                        *abort_flag = 1;
                        break;
                    }
                    const float *qp = qb + (size_t)(bh - row0) * R;
#pragma unroll
                    for (int c = 0; c < CPT; ++c) {
                        const int ch = sub * CPT + ((c + rot) % CPT);
#pragma unroll
                        for (int x = 0; x < EPL; ++x) qreg[c * EPL + x] = qp[ch * EPL + x];
                    }
                } else {
                    const float *qp = a.qproj + (size_t)bh * R;  // written by the preceding kernel: read through L2
#pragma unroll
                    for (int c = 0; c < CPT; ++c) {
                        const int ch = sub * CPT + ((c + rot) % CPT);
#pragma unroll
                        for (int x = 0; x < EPL; ++x) qreg[c * EPL + x] = __ldcg(qp + ch * EPL + x);
                    }
                }
            }
            if (epos == 0 && e >= kEB) {
                bool ok = wait_or_abort(&efree[p], eph ^ 1u, abort_flag);
                if (!__all_sync(0xffffffffu, ok)) {
                    *abort_flag = 1;
                    break;
                }
            }
            {
                bool ok = wait_or_abort(&full[s], rp.ph, abort_flag);
                if (!__all_sync(0xffffffffu, ok)) {
                    *abort_flag = 1;
                    break;
                }
            }
            const int t0 = t * TILE;
            const int n = misc[80 + s] ? 0 : max(0, min(TILE, Tb - t0));  // a screened-out tile holds nothing
            // does this tile hold always-selected tokens (warp-uniform)?
            const bool tforce = t0 < a.n_sink || t0 + TILE > Tb - a.n_recent;
            const unsigned long long tw = *thr_word;
            const bool use = (uint32_t)(tw >> 32) == tag;
            const uint32_t tk = (uint32_t)tw;
            const unsigned char *st = smem + L.ring + (size_t)s * kTile;
#pragma unroll
            for (int ps = 0; ps < PASSES; ++ps) {
                const int tt = ps * TPP + ct / LPT;
                const bool live = tt < n;
                const unsigned char *row = st + (size_t)tt * ROWB + sub * TPB;
                float pc[CPT];
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (live) v = *reinterpret_cast<const uint4 *>(row + ((c + rot) % CPT) * 16);
                    float kf[EPL];
                    Vec16<KT>::unpack(v, kf);
                    float acc = 0.f;
#pragma unroll
                    for (int x = 0; x < EPL; ++x) acc = fmaf(kf[x], qreg[c * EPL + x], acc);
                    pc[c] = acc;
                }
                float sc;
                if constexpr (CPT == 4) sc = (pc[0] + pc[2]) + (pc[1] + pc[3]);
                else if constexpr (CPT == 2) sc = pc[0] + pc[1];
                else sc = pc[0];
#pragma unroll
                for (int off = 1; off < LPT; off <<= 1) sc += __shfl_xor_sync(0xffffffffu, sc, off);
                uint32_t key = score_key(sc);
                if (tforce) key = forced_key(key, t0 + tt, Tb, a.n_sink, a.n_recent);
                const bool take = live && sub == 0 && (!use || key > tk);
                const unsigned msk = __ballot_sync(0xffffffffu, take);
                if (msk) {
                    const int ld = __ffs(msk) - 1;
                    int b0 = 0;
                    if (lane == ld) b0 = atomicAdd(&misc[40 + p], __popc(msk));
                    b0 = __shfl_sync(0xffffffffu, b0, ld);
                    if (take) {
                        const int q = b0 + __popc(msk & lane_lt());
                        ek[p * EPT + q] = key;
                        ei[p * EPT + q] = t0 + tt;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (epos == E - 1 || cur.seg_last(i, ntiles)) {
                if (lane == 0) mbar_arrive(&efull[p]);
                ++e;
                epos = 0;
                if (++p == kEB) {
                    p = 0;
                    eph ^= 1u;
                }
            } else {
                ++epos;
            }
        }
    } else {
        // ------------------------------------------------------ selector
        Sel S;
        S.rk = reinterpret_cast<uint32_t *>(smem + L.rk);
        S.ri = reinterpret_cast<int32_t *>(smem + L.ri);
        S.sk = reinterpret_cast<uint32_t *>(smem + L.sk);
        S.si = reinterpret_cast<int32_t *>(smem + L.si);
        S.hist = reinterpret_cast<uint32_t *>(smem + L.hist);
        S.misc = misc;
        S.st = tid - kSelBase;
        const int slane = S.st & 31;
        int epos = 0, m = 0, p = 0;
        uint32_t eph = 0u;
        bool valid = false;
        uint32_t thr = 0u;
        if constexpr (FUSED) {
            // prologue: folded queries of the range's rows, then the new rows of
            // the low-rank cache whose tiles this CTA streams
            float *xs = reinterpret_cast<float *>(smem + L.xs);
            float *part = reinterpret_cast<float *>(S.hist);
            for (int rl = 0; rl < nrows; ++rl) {
                sel_project<R>(A.x, a.Hkv, row0 + rl, qb + (size_t)rl * R, xs, part, S.st);
                if (S.st == 0) mbar_arrive(&qready[rl]);  // consumers of row rl may start
            }
            for (int rl = 0; rl < nrows; ++rl) {
                const int bh = row0 + rl;
                const int pos = __ldg(A.x.pos_begin + bh / a.Hkv);
                if (pos < 0 || pos >= a.T_cap) {
                    if (S.st == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_POS);
                    continue;
                }
                const long long xt = (long long)bh * a.tiles_per_bh + pos / TILE;
                if (xt >= x_begin && xt < x_end) sel_append<R>(a, A.x, bh, pos, xs, part, S.st);
            }
            if (S.st == 0) mbar_arrive(aready);
        }
        Cursor cur = c0;
        for (int i = 0; i < ntiles; ++i, cur.next()) {
            const bool send = cur.seg_last(i, ntiles);
            if (!(epos == E - 1 || send)) {
                ++epos;
                continue;
            }
            epos = 0;
            if (S.st == 0) {
                // one thread waits; the others are parked at the barrier
                const bool ok = wait_or_abort(&efull[p], eph, abort_flag);
                if (!ok) *abort_flag = 1;
                misc[8] = *abort_flag;
            }
            sel_sync();
            if (misc[8]) break;
            const int ne = misc[40 + p];
            for (int j0 = 0; j0 < ne; j0 += kSelT) {
                const int j = j0 + S.st;
                uint32_t u = 0u;
                int32_t ix = 0;
                if (j < ne) {
                    u = ek[p * EPT + j];
                    ix = ei[p * EPT + j];
                }
                const bool take = j < ne && (!valid || u > thr);
                const unsigned msk = __ballot_sync(0xffffffffu, take);
                int b0 = 0;
                if (msk) {
                    const int ld = __ffs(msk) - 1;
                    // forced keys stay out of the tracked range (they sit above every bin)
                    uint32_t mn = take ? u : 0xffffffffu, mx = (take && u != kForcedKey) ? u : 0u;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) {
                        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, off));
                        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                    }
                    if (slane == ld) {
                        b0 = atomicAdd(&misc[3], __popc(msk));
                        atomicMin(reinterpret_cast<unsigned *>(&misc[44]), mn);
                        atomicMax(reinterpret_cast<unsigned *>(&misc[45]), mx);
                    }
                    b0 = __shfl_sync(0xffffffffu, b0, ld);
                }
                if (take) {
                    const int q = b0 + __popc(msk & lane_lt());
                    S.rk[q] = u;
                    S.ri[q] = ix;
                }
            }
            sel_sync();
            m = misc[3];
            if (S.st == 0) {
                misc[40 + p] = 0;
                mbar_arrive(&efree[p]);  // the epoch buffer may be refilled
            }
            if (++p == kEB) {
                p = 0;
                eph ^= 1u;
            }
            const int bh = cur.bh;
            if (send) {
                const int fin = sel_finish(a, S, m, bh, cta, EPT, a.cap);
                if (FUSED && fin >= 0 && S.st == 0) {  // this CTA attends over the row at the end
                    const int na = misc[46];
                    misc[64 + na] = bh;
                    misc[72 + na] = fin;
                    misc[46] = na + 1;
                }
                m = 0;
                valid = false;
                if (S.st == 0) {
                    misc[3] = 0;
                    misc[44] = (int)0xffffffffu;
                    misc[45] = 0;
                }
                sel_sync();
            } else if ((!valid && m > a.k) || m > a.cap - EPT) {
                const uint32_t lo = valid ? thr + 1u : (uint32_t)misc[44], hi = (uint32_t)misc[45];
                uint32_t t = thr;
                int kept = m;
                bool done = false;
                if (m <= kRegKeys * kSelT) {
                    t = sel_trim(S, m, a.k, lo, hi, kept);
                    done = kept <= a.cap - EPT;
                }
                if (!done) {  // too many keys for registers, or one bin too full to make room
                    t = sel_reduce(S, kept, a.k);
                    kept = a.k;
                }
                m = kept;
                if (t > thr || !valid) {
                    thr = t;
                    valid = true;
                }
                if (S.st == 0) {
                    misc[3] = m;
                    misc[44] = (int)(thr + 1u);
                    *thr_word = ((unsigned long long)((uint32_t)bh + 1u) << 32) | thr;
                }
                sel_sync();
            }
        }
    }

    __syncthreads();
    if (*abort_flag) {
        if (tid == kProdBase) {
            if (a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_TIMEOUT);
            // let the copies already in flight land before the CTA exits
            const int issued = misc[24];
            for (int i = issued - S_ > 0 ? issued - S_ : 0; i < issued; ++i)
                (void)mbar_wait_bounded(&full[i % S_], (uint32_t)(i / S_) & 1u);
        }
        __syncthreads();
        return;
    }
    if constexpr (FUSED) {
        // epilogue: attention of the rows whose selection this CTA completed,
        // in the (now idle) ring and epoch buffers
        if (tid >= kConsBase) {
            const int na = misc[46];
            for (int i = 0; i < na; ++i)
                fused_attend<D>(a, A.x, misc[64 + i], misc[72 + i], smem + L.ring, L.bars - L.ring, tid - kConsBase);
        }
    }
}

template <int SRC>
void (*pick_r(int r))(StreamArgs) {
    switch (r) {
        case 8: return stream_select_kernel<SRC, 8, 0>;
        case 16: return stream_select_kernel<SRC, 16, 0>;
        case 32: return stream_select_kernel<SRC, 32, 0>;
        case 64: return stream_select_kernel<SRC, 64, 0>;
        case 128: return stream_select_kernel<SRC, 128, 0>;
        default: return nullptr;
    }
}

void (*pick_stream(int src, int r))(StreamArgs) {
    if (src == SRC_KT_BF16) return pick_r<SRC_KT_BF16>(r);
    if (src == SRC_KT_FP32) return pick_r<SRC_KT_FP32>(r);
    return nullptr;
}

void (*pick_fused(int r, int d))(StreamArgs) {
    if (r == 32 && d == 128) return stream_select_kernel<SRC_KT_BF16, 32, 128>;
    if (r == 32 && d == 256) return stream_select_kernel<SRC_KT_BF16, 32, 256>;
    if (r == 64 && d == 128) return stream_select_kernel<SRC_KT_BF16, 64, 128>;
    if (r == 64 && d == 256) return stream_select_kernel<SRC_KT_BF16, 64, 256>;
    return nullptr;
}

// Shared planning of both forms: tiles, epochs, ring depth, grid, segments.
cudaError_t plan_common(void (*kern)(StreamArgs), int src, int B, int Hkv, int T_cap, int r, int k, int fused_r,
                        ScanPlan *p) {
    const int rowb = r * (src == SRC_KT_FP32 ? 4 : 2);
    const int tile = kTile / rowb;
    const int ept = tile >= kEpochTokens ? tile : kEpochTokens;
    ScanPlan P;
    P.src = src;
    P.mode = MODE_SELECT;
    P.tile_tokens = tile;
    P.tiles_per_bh = (T_cap + tile - 1) / tile;
    P.total_tiles = (long long)B * Hkv * P.tiles_per_bh;
    // candidate capacity: the kept set after a cut (k plus up to 1024 more
    // before the next cut) and one epoch of new survivors
    P.cap = k + ept + 1024;
    if (P.cap < 2 * k) P.cap = 2 * k;  // the merge holds k kept entries and one segment's k slots
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    int ns = kMaxStages;
    while (ns >= 3 && stream_smem(ns, ept, P.cap, k, fused_r).total > (size_t)optin) --ns;
    if (ns < 3) return cudaErrorNotSupported;
    P.nstages = ns;
    // one CTA per SM, but no row split into segments of fewer than
    // kMinSegTiles tiles: a short row streams faster than the cross-CTA merge
    // of its segments would take (a 4K-token row is one 256 KiB segment)
    long long g = device_sm_count();
    const long long segs = (long long)B * Hkv * ((P.tiles_per_bh + kMinSegTiles - 1) / kMinSegTiles);
    if (g > segs) g = segs;
    if (g > P.total_tiles) g = P.total_tiles;
    if (g < 1) g = 1;
    P.grid = (int)g;
    // screening bounds staged per CTA: as many tiles of its range as the
    // space the ring leaves over holds (the rest load as they are needed)
    const size_t base = stream_smem(ns, ept, P.cap, k, fused_r).total;
    const long long per_cta = (P.total_tiles + g - 1) / g;
    long long nb = ((long long)optin - (long long)base - 128) / 4;
    if (nb > per_cta) nb = per_cta;
    P.nb_cap = nb > 0 ? (int)nb : 0;
    P.smem = stream_smem(ns, ept, P.cap, k, fused_r, P.nb_cap).total;
    e = ensure_smem(reinterpret_cast<const void *>(kern), P.smem);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, P.smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorNotSupported;
    int ms = 1;
    const long long BH = (long long)B * Hkv;
    for (long long bh = 0; bh < BH; ++bh) {
        const long long f = bh * P.tiles_per_bh, l = f + P.tiles_per_bh - 1;
        const long long cf = ((f + 1) * P.grid - 1) / P.total_tiles;
        const long long cl = ((l + 1) * P.grid - 1) / P.total_tiles;
        if (cl - cf + 1 > ms) ms = (int)(cl - cf + 1);
    }
    P.max_seg = ms;
    *p = P;
    return cudaSuccess;
}

}  // namespace

// Plan of the warp-specialised form: SUM aggregation over the low-rank key
// cache (the decode-step path).  cudaErrorNotSupported for other forms.
cudaError_t plan_stream(int src, int agg, int B, int Hkv, int T_cap, int r, int k, ScanPlan *p) {
    if (agg != JSSA_AGG_SUM) return cudaErrorNotSupported;
    auto kern = pick_stream(src, r);
    if (!kern) return cudaErrorNotSupported;
    return plan_common(kern, src, B, Hkv, T_cap, r, k, 0, p);
}

namespace {
void fill_plan(StreamArgs &A, const ScanPlan &p) {
    A.s.tile_tokens = p.tile_tokens;
    A.s.tiles_per_bh = p.tiles_per_bh;
    A.s.total_tiles = p.total_tiles;
    A.s.grid = p.grid;
    A.s.max_seg = p.max_seg;
    A.s.cap = p.cap;
    A.s.nstages = p.nstages;
    A.s.nb_cap = p.nb_cap;
}
}  // namespace

cudaError_t launch_stream(const ScanPlan &p, const ScanArgs &a0, cudaStream_t s, bool pdl) {
    auto kern = pick_stream(p.src, a0.r);
    if (!kern) return cudaErrorInvalidValue;
    if (p.total_tiles <= 0) return cudaSuccess;
    StreamArgs A;
    memset(&A, 0, sizeof A);
    A.s = a0;
    fill_plan(A, p);
    return launch_kernel(kern, dim3(p.grid), dim3(kThreads), p.smem, s, pdl, A);
}

cudaError_t plan_step_fused(int B, int Hkv, int Hq, int d, int T_cap, int r, int k, ScanPlan *p) {
    auto kern = pick_fused(r, d);
    if (!kern || Hkv < 1 || Hq % Hkv) return cudaErrorNotSupported;
    const int G = Hq / Hkv;
    if (G < 1 || G > kConsWarps || (G & (G - 1))) return cudaErrorNotSupported;
    cudaError_t e = plan_common(kern, SRC_KT_BF16, B, Hkv, T_cap, r, k, r, p);
    if (e != cudaSuccess) return e;
    // every CTA range spans at most kMaxRows (b,h) rows, and the ring holds
    // the attention's combine area plus one staged K/V row pair
    for (long long c = 0; c < p->grid; ++c) {
        const long long xb = c * p->total_tiles / p->grid, xe = (c + 1) * p->total_tiles / p->grid;
        if (xe > xb && (xe - 1) / p->tiles_per_bh - xb / p->tiles_per_bh + 1 > kMaxRows) return cudaErrorNotSupported;
    }
    // attention epilogue: Q, partials, and at least one 16-token chunk
    const size_t need = 16 * (size_t)(2 * d + 16) + kConsWarps * 16 * 4 + (size_t)((k + 3) & ~3) * 4 + 16 * 16 +
                        128 + 16 * (size_t)(4 * d + 32);
    const int tile = kTile / (r * 2), ept = tile >= kEpochTokens ? tile : kEpochTokens;
    const StreamSmem L = stream_smem(p->nstages, ept, p->cap, k, r);
    if (L.bars - L.ring < need) return cudaErrorNotSupported;
    return cudaSuccess;
}

cudaError_t launch_step_fused(const ScanPlan &p, const ScanArgs &a0, const StepExtra &x, cudaStream_t s, bool pdl) {
    auto kern = pick_fused(a0.r, x.d);
    if (!kern) return cudaErrorInvalidValue;
    if (p.total_tiles <= 0) return cudaSuccess;
    StreamArgs A;
    memset(&A, 0, sizeof A);
    A.s = a0;
    A.x = x;
    fill_plan(A, p);
    return launch_kernel(kern, dim3(p.grid), dim3(kThreads), p.smem, s, pdl, A);
}

}  // namespace jssa
