// Per-(batch, KV head) top-k selection by one thread-block cluster per (b, h).
//
// Method: news item "JSSA makes token-level sparse decoding gather-free",
// Synopsis (tokens scored in a shared low-dimensional query-key subspace; a
// distinct selected token set for each KV head); "Joint Subspace Sparse
// Attention for Efficient Long-Context Decoding", Abstract (distinct
// per-KV-head selections).
//
// The C CTAs of a cluster split the token range of one (b, h) into C
// contiguous slices.  Each CTA streams its slice of the low-rank key cache
// through a ring of 32 KiB bulk asynchronous copies (2 to 6 stages, the
// planner's choice; or reads its slice of a score array), computes the fp32
// scores exactly as the score pass does, and keeps their order-preserving
// uint32 keys in shared memory.  The cluster then finds the k-th key
// together: three radix levels of 11, 11 and 10 bits; at each level every
// CTA histograms its keys that match the prefix found so far and adds its
// non-empty bins into the CTA that owns them (bin d lives in rank
// d / (2048 / C), in one of three rotating copies), one cluster barrier
// later every CTA gathers the summed bins through distributed shared memory
// and scans them.  Keys
// equal to the k-th key are taken lowest token index first (CTAs hold
// ascending token ranges, so an exclusive scan of their tie counts orders
// them).  Each CTA finally writes its selected tokens, already ascending, at
// its offset in the index list (a warp's 32-token steps ordered by ballots):
// no merge and no sort.  The result is the same
// set, in the same order, as jssa_score + jssa_topk.
#include <cooperative_groups.h>

#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace cg = cooperative_groups;

namespace jssa {

namespace {

constexpr int NT = 256;
constexpr int kTileB = 32768;   // bytes per ring stage
constexpr int kMaxStagesC = 6;  // ring depth: chosen by the planner (2 .. 6)
constexpr int kBins = 2048;
constexpr int kMaxSlice = 16384;  // tokens per CTA kept in shared memory

struct CSmem {
    size_t stages, bars, qs, keys, hist, gsum, gall, misc, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) / 16 * 16; }

__host__ __device__ inline CSmem csel_smem(bool from_kt, int r, int nq, int slice, int nstages, int C) {
    CSmem L;
    size_t o = 0;
    L.stages = o;
    o += from_kt ? (size_t)nstages * kTileB : 0;
    L.bars = o;
    o = align16(o + 8 * kMaxStagesC);
    L.qs = o;
    o = align16(o + (from_kt ? (size_t)nq * r * 4 : 0));
    L.keys = o;
    o = align16(o + (size_t)slice * 4);
    L.hist = o;
    o = align16(o + (size_t)kBins * 4);
    L.gsum = o;
    o = align16(o + (size_t)3 * (kBins / C) * 4);  // three rotating copies of this CTA's slice of summed bins
    L.gall = o;
    o = align16(o + (size_t)kBins * 4);
    L.misc = o;
    o = align16(o + 64 * 4);
    L.total = (o + 127) / 128 * 128;
    return L;
}

template <int CPT>
__device__ __forceinline__ float chunk_sum(const float (&p)[CPT]) {
    if constexpr (CPT == 4) return (p[0] + p[2]) + (p[1] + p[3]);
    if constexpr (CPT == 2) return p[0] + p[1];
    return p[0];
}

template <int SRC, int R, int AGG>
__global__ void __launch_bounds__(NT, 2) select_cluster_kernel(CSelArgs a) {
    constexpr bool FROM_KT = SRC != SRC_SCORES;
    using KT = typename std::conditional<SRC == SRC_KT_FP32, float, __nv_bfloat16>::type;
    constexpr int ES = SRC == SRC_KT_FP32 ? 4 : 2;
    constexpr int ROWB = FROM_KT ? R * ES : 4;
    constexpr int TPB = ROWB > 64 ? 64 : ROWB;
    constexpr int LPT = ROWB / TPB;
    constexpr int CPT = FROM_KT ? TPB / 16 : 1;
    constexpr int EPL = 16 / ES;
    constexpr int TILE = FROM_KT ? kTileB / ROWB : 2048;
    constexpr int TPP = NT / LPT;
    constexpr int PASSES = FROM_KT ? TILE / TPP : TILE / NT;
    constexpr int QN = FROM_KT ? CPT * EPL : 1;
    static_assert(!FROM_KT || TILE % TPP == 0, "tile / pass");

    extern __shared__ __align__(128) unsigned char smem[];
    const int NS = a.nstages;
    const CSmem L = csel_smem(FROM_KT, FROM_KT ? R : 0, a.nq, a.slice, NS, a.csize);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
    float *qs = reinterpret_cast<float *>(smem + L.qs);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem + L.keys);
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem + L.hist);
    uint32_t *gsum = reinterpret_cast<uint32_t *>(smem + L.gsum);
    uint32_t *gall = reinterpret_cast<uint32_t *>(smem + L.gall);
    int *misc = reinterpret_cast<int *>(smem + L.misc);
    int *tmp = misc + 16;

    cg::cluster_group cluster = cg::this_cluster();
    const int C = a.csize;
    const int c = (int)cluster.block_rank();
    const int bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31;

    if (FROM_KT && tid == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
    }
    if (tid == 0) misc[6] = 0;
    {
        // copies 0 and 1 of the summed-bin slice start at zero; the cluster
        // barrier phase opened here closes before the first remote add
        const int bpc = kBins / a.csize;
        uint32_t *gs = reinterpret_cast<uint32_t *>(smem + L.gsum);
        for (int d = threadIdx.x; d < 2 * bpc; d += NT) gs[d] = 0u;
    }
    __syncthreads();
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    pdl_trigger();
    pdl_wait();

    const int Tb = clamp_seq(__ldg(a.seq_lens + bh / a.Hkv), a.T_cap, a.status);
    const int kb = min(a.k, Tb);
    const int lo = c * a.slice;
    const int n_loc = max(0, min(a.slice, Tb - lo));  // valid tokens of this CTA
    const int ntiles = (n_loc + TILE - 1) / TILE;

    // ---- scores of this slice into shared memory ---------------------------
    if constexpr (FROM_KT) {
        const int srow = a.src_div > 1 ? bh / a.src_div : bh;
        const char *src = static_cast<const char *>(a.src) + ((size_t)srow * a.T_cap + lo) * ROWB;
        uint64_t pol = 0;
        if (tid == 0) {
            pol = policy_evict_first();
            for (int i = 0; i < min(NS, ntiles); ++i) {
                const int n = min(TILE, n_loc - i * TILE);
                mbar_arrive_expect_tx(&bars[i], (uint32_t)n * ROWB);
                bulk_g2s(smem + L.stages + (size_t)i * kTileB, src + (size_t)i * TILE * ROWB, (uint32_t)n * ROWB, &bars[i],
                         pol);
            }
        }
        for (int p = tid; p < a.nq * R; p += NT) qs[p] = a.qproj[(size_t)bh * a.nq * R + p];
        __syncthreads();
        const int sub = tid % LPT;
        const int rot = CPT == 4 ? (lane >> 1) & 3 : (CPT == 2 ? (lane >> 2) & 1 : 0);
        float qreg[QN];
        if (AGG == JSSA_AGG_SUM) {
#pragma unroll
            for (int cc = 0; cc < CPT; ++cc) {
                const int ch = sub * CPT + ((cc + rot) % CPT);
#pragma unroll
                for (int e = 0; e < EPL; ++e) qreg[(cc * EPL + e) % QN] = qs[ch * EPL + e];
            }
        }
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % NS;
            const int t0 = i * TILE, n = min(TILE, n_loc - t0);
            if (!mbar_wait_bounded(&bars[s], (uint32_t)(i / NS) & 1u)) misc[6] = 1;
            const unsigned char *st = smem + L.stages + (size_t)s * kTileB;
#pragma unroll
            for (int ps = 0; ps < PASSES; ++ps) {
                const int tt = ps * TPP + tid / LPT;
                const bool live = tt < n;
                const unsigned char *row = st + (size_t)tt * ROWB + sub * TPB;
                float sc;
                if constexpr (AGG == JSSA_AGG_SUM) {
                    float pc[CPT];
#pragma unroll
                    for (int cc = 0; cc < CPT; ++cc) {
                        uint4 v = make_uint4(0u, 0u, 0u, 0u);
                        if (live) v = *reinterpret_cast<const uint4 *>(row + ((cc + rot) % CPT) * 16);
                        float kf[EPL];
                        Vec16<KT>::unpack(v, kf);
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < EPL; ++e) acc = fmaf(kf[e], qreg[cc * EPL + e], acc);
                        pc[cc] = acc;
                    }
                    float acc = chunk_sum<CPT>(pc);
#pragma unroll
                    for (int off = 1; off < LPT; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                    sc = acc;
                } else {
                    float kf[CPT][EPL];
#pragma unroll
                    for (int cc = 0; cc < CPT; ++cc) {
                        uint4 v = make_uint4(0u, 0u, 0u, 0u);
                        if (live) v = *reinterpret_cast<const uint4 *>(row + ((cc + rot) % CPT) * 16);
                        Vec16<KT>::unpack(v, kf[cc]);
                    }
                    float best = -INFINITY;
                    for (int g = 0; g < a.nq; ++g) {
                        float pc[CPT];
#pragma unroll
                        for (int cc = 0; cc < CPT; ++cc) {
                            const int ch = sub * CPT + ((cc + rot) % CPT);
                            const float *qg = qs + g * R + ch * EPL;
                            float acc = 0.f;
#pragma unroll
                            for (int e = 0; e < EPL; ++e) acc = fmaf(kf[cc][e], qg[e], acc);
                            pc[cc] = acc;
                        }
                        float acc = chunk_sum<CPT>(pc);
#pragma unroll
                        for (int off = 1; off < LPT; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                        best = fmaxf(best, acc);
                    }
                    sc = best;
                }
                if (live && sub == 0) keys[t0 + tt] = forced_key(score_key(sc), lo + t0 + tt, Tb, a.n_sink, a.n_recent);
            }
            __syncthreads();  // stage s consumed
            if (tid == 0 && i + NS < ntiles) {
                const int n2 = min(TILE, n_loc - (i + NS) * TILE);
                mbar_arrive_expect_tx(&bars[s], (uint32_t)n2 * ROWB);
                bulk_g2s(smem + L.stages + (size_t)s * kTileB, src + (size_t)(i + NS) * TILE * ROWB,
                         (uint32_t)n2 * ROWB, &bars[s], pol);
            }
        }
    } else {
        const float *srow = static_cast<const float *>(a.src) + (size_t)bh * a.T_cap + lo;
        for (int j0 = 0; j0 < n_loc; j0 += NT * 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u * NT + tid;
                v[u] = j < n_loc ? __ldcs(srow + j) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u * NT + tid;
                if (j < n_loc) keys[j] = forced_key(score_key(v[u]), lo + j, Tb, a.n_sink, a.n_recent);
            }
        }
    }
    __syncthreads();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    const bool local_timeout = misc[6] != 0;

    // ---- cluster radix select of the k-th key ------------------------------
    uint32_t prefix = 0u, mask = 0u;
    int kk = kb, grp = 0;
    bool whole = true;
    const int bins_per_cta = kBins / C;
    if (kb > 0 && kb < Tb) {
        const int shifts[3] = {21, 10, 0}, widths[3] = {11, 11, 10};
        for (int lev = 0; lev < 3; ++lev) {
            const int shift = shifts[lev];
            const uint32_t dmask = (1u << widths[lev]) - 1u;
            for (int d = tid; d < kBins; d += NT) hist[d] = 0u;
            __syncthreads();
            for (int j = tid; j < n_loc; j += NT) {
                const uint32_t u = keys[j];
                if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
            }
            __syncthreads();
            // add the non-empty bins into their owners' copy lev % 3 (owner of
            // bin d: rank d / bins_per_cta), then one cluster barrier
            uint32_t *cur = gsum + (lev % 3) * bins_per_cta;
            for (int d = tid; d < kBins; d += NT) {
                const uint32_t v = hist[d];
                if (v) atomicAdd(cluster.map_shared_rank(cur + d % bins_per_cta, d / bins_per_cta), v);
            }
            cluster.sync();
            // every CTA has read copy (lev + 2) % 3 one level back: clear it for two levels on
            {
                uint32_t *nxt = gsum + ((lev + 2) % 3) * bins_per_cta;
                for (int q = tid; q < bins_per_cta; q += NT) nxt[q] = 0u;
            }
            {
                uint32_t v[kBins / NT];
#pragma unroll
                for (int u = 0; u < kBins / NT; ++u) {
                    const int d = tid + u * NT;
                    v[u] = *cluster.map_shared_rank(cur + (d % bins_per_cta), d / bins_per_cta);
                }
#pragma unroll
                for (int u = 0; u < kBins / NT; ++u) gall[tid + u * NT] = v[u];
            }
            __syncthreads();
            // descending scan over all bins: thread t owns 8 bins from the top
            constexpr int BPT = kBins / NT;
            const int base_bin = kBins - BPT * (tid + 1);
            int cnt[BPT];
            int s = 0;
#pragma unroll
            for (int q = 0; q < BPT; ++q) {
                cnt[q] = (int)gall[base_bin + BPT - 1 - q];
                s += cnt[q];
            }
            int tot;
            int ex = block_excl_scan<NT>(s, tmp, tot);
#pragma unroll
            for (int q = 0; q < BPT; ++q) {
                if (ex < kk && ex + cnt[q] >= kk) {
                    misc[0] = base_bin + BPT - 1 - q;
                    misc[1] = ex;
                    misc[2] = cnt[q];
                }
                ex += cnt[q];
            }
            __syncthreads();
            prefix |= (uint32_t)misc[0] << shift;
            mask |= dmask << shift;
            kk -= misc[1];
            grp = misc[2];
            __syncthreads();
            if (kk == grp) break;
        }
        whole = kk == grp;
    }

    // ---- ties: equal keys go to the lowest token indices, CTA by CTA --------
    int take_ties = 0;
    if (!whole) {
        int e = 0;
        for (int j = tid; j < n_loc; j += NT) e += (keys[j] & mask) == prefix;
        int tot;
        (void)block_excl_scan<NT>(e, tmp, tot);
        if (tid == 0) misc[3] = tot;
        cluster.sync();
        // ties held by the CTAs before this one: one remote load per lane, all in flight
        const int before = __reduce_add_sync(0xffffffffu, lane < c ? *cluster.map_shared_rank(misc + 3, lane) : 0);
        take_ties = max(0, min(tot, kk - before));
    }

    // ---- emit the selection in ascending token order -----------------------
    // Warp wp takes the contiguous tokens [jb, je) of the slice, 32 at a time
    // (lane l reads token j0 + l, conflict-free), and compacts its selected
    // tokens and ties, in order, into the front of its own span of the key
    // array (the keys are not read again; a step only writes entries it has
    // already read): token index, bit 31 for a tie.  The warp totals are
    // scanned across the block, and each warp then writes from its short list.
    const bool take_all = kb >= Tb;
    const bool ties_on = !take_all && kb > 0 && !whole;
    constexpr int NW = NT / 32;
    const int wp = tid >> 5;
    const int span = ((n_loc + NW - 1) / NW + 31) & ~31;
    const int jb = min(wp * span, n_loc), je = min(jb + span, n_loc);
    const unsigned lt = (1u << lane) - 1u;
    auto sure_of = [&](uint32_t u) {
        return take_all || (kb > 0 && ((u & mask) > prefix || ((u & mask) == prefix && whole)));
    };
    int cs = 0, ce = 0;  // the warp's sure selections and ties
    for (int j0 = jb; j0 < je; j0 += 32) {
        const int j = j0 + lane;
        const bool ok = j < je;
        const uint32_t u = ok ? keys[j] : 0u;
        const bool sure = ok && sure_of(u);
        const bool tie = ok && ties_on && (u & mask) == prefix;
        const unsigned mb = __ballot_sync(0xffffffffu, sure || tie);
        if (sure || tie) keys[jb + cs + ce + __popc(mb & lt)] = (uint32_t)j | (tie ? 0x80000000u : 0u);
        cs += __popc(__ballot_sync(0xffffffffu, sure));
        ce += __popc(__ballot_sync(0xffffffffu, tie));
    }
    if (lane == 0) misc[32 + wp] = ce;
    __syncthreads();
    int e0 = 0;  // tie rank of the warp's first tie
#pragma unroll
    for (int q = 0; q < NW; ++q) e0 += q < wp ? misc[32 + q] : 0;
    const int mine = cs + max(0, min(ce, take_ties - e0));
    if (lane == 0) misc[40 + wp] = mine;
    __syncthreads();
    int w_off = 0, tot_s = 0;
#pragma unroll
    for (int q = 0; q < NW; ++q) {
        const int v = misc[40 + q];
        w_off += q < wp ? v : 0;
        tot_s += v;
    }
    if (tid == 0) misc[4] = tot_s;
    cluster.sync();
    const int base = __reduce_add_sync(0xffffffffu, lane < c ? *cluster.map_shared_rank(misc + 4, lane) : 0);
    int32_t *out = a.idx_out + (size_t)bh * a.k;
    {
        int w = base + w_off, e = e0;
        const int cnt = cs + ce;
        for (int i0 = 0; i0 < cnt; i0 += 32) {
            const int i = i0 + lane;
            const bool ok = i < cnt;
            const uint32_t v = ok ? keys[jb + i] : 0u;
            const bool tie = ok && (v >> 31);
            const unsigned tb = __ballot_sync(0xffffffffu, tie);
            const bool sel = ok && (!tie || e + __popc(tb & lt) < take_ties);
            const unsigned sb = __ballot_sync(0xffffffffu, sel);
            if (sel) {
                const int p = w + __popc(sb & lt);
                if (p < a.k) out[p] = lo + (int)(v & 0x7fffffffu);
            }
            w += __popc(sb);
            e += __popc(tb);
        }
    }
    if (c == C - 1) {
        const int total = base + tot_s;  // = k_b
        for (int j = total + tid; j < a.k; j += NT) out[j] = -1;
        if (tid == 0 && a.count_out) a.count_out[bh] = total;
    }
    if (local_timeout && tid == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_TIMEOUT);
    cluster.sync();  // peers may still read this CTA's shared memory until here
}

template <int SRC, int R, int AGG>
void (*pick_c3())(CSelArgs) {
    return select_cluster_kernel<SRC, R, AGG>;
}

template <int SRC>
void (*pick_cr(int r, int agg))(CSelArgs) {
    switch (r) {
        case 8: return agg ? pick_c3<SRC, 8, 1>() : pick_c3<SRC, 8, 0>();
        case 16: return agg ? pick_c3<SRC, 16, 1>() : pick_c3<SRC, 16, 0>();
        case 32: return agg ? pick_c3<SRC, 32, 1>() : pick_c3<SRC, 32, 0>();
        case 64: return agg ? pick_c3<SRC, 64, 1>() : pick_c3<SRC, 64, 0>();
        case 128: return agg ? pick_c3<SRC, 128, 1>() : pick_c3<SRC, 128, 0>();
        default: return nullptr;
    }
}

void (*pick_csel(int src, int r, int agg))(CSelArgs) {
    if (src == SRC_SCORES) return select_cluster_kernel<SRC_SCORES, 8, 0>;
    return src == SRC_KT_BF16 ? pick_cr<SRC_KT_BF16>(r, agg) : pick_cr<SRC_KT_FP32>(r, agg);
}

int csel_tile(int src, int r) {
    if (src == SRC_SCORES) return 2048;
    return kTileB / (r * (src == SRC_KT_FP32 ? 4 : 2));
}

}  // namespace

// Which selection form a shape uses.  The cluster form is taken when every
// (b,h) gets its own cluster, all resident at once, with the keys of its slice
// in shared memory: it has no segment merge and no second wave.  Otherwise
// (many (b,h) rows or rows too long for shared memory) a persistent streaming
// pass is taken: the warp-specialised one for SUM over the low-rank cache,
// the block-synchronous one for the other sources and aggregations.  All
// return the same indices.  A forced form (jssa_select_opts.form) overrides
// the choice: JSSA_FORM_CLUSTER takes the cluster form wherever its slices fit
// in shared memory (several waves allowed), JSSA_FORM_STREAM the
// warp-specialised pass where it has a kernel, JSSA_FORM_SCAN the
// block-synchronous pass.
namespace {

// Resident clusters of size C for this kernel and shared-memory size (0 on error).
int resident_clusters(void (*kern)(CSelArgs), int C, size_t smem) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, 1);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int ncl = 0;
    if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return ncl;
}

// Plans are cached per device and shape: the occupancy queries cost far more
// host time than a decode step's launches.
struct CSelKey {
    int dev, form, src, agg, B, Hkv, T_cap, r, nq, k;
    bool operator==(const CSelKey &o) const { return !memcmp(this, &o, sizeof *this); }
};
struct CSelEntry {
    CSelKey key;
    cudaError_t err;
    CSelPlan plan;
};
constexpr int kPlanCache = 64;
CSelEntry g_cache[kPlanCache];
int g_cache_n = 0, g_cache_next = 0;
std::mutex g_cache_mu;

cudaError_t plan_csel_uncached(int form, int src, int agg, int B, int Hkv, int T_cap, int r, int nq, int k,
                               CSelPlan *p) {
    if (form == 2 || form == 3) return cudaErrorNotSupported;
    auto kern = pick_csel(src, r, agg);
    if (!kern) return cudaErrorNotSupported;
    const int tile = csel_tile(src, r);
    const int tiles = (T_cap + tile - 1) / tile;
    const int BH = B * Hkv;
    // The largest power-of-two cluster (the summed histogram is split evenly
    // over its CTAs) whose slices fit in shared memory and whose B*Hkv
    // clusters are all resident at once (one wave).  "cluster" relaxes the
    // one-wave condition.
    for (int C = 16; C >= 2; C >>= 1) {
        if (C > tiles && C > 2) continue;
        int slice = (T_cap + C - 1) / C;
        slice = (slice + tile - 1) / tile * tile;
        if (slice > kMaxSlice) break;  // smaller clusters only lengthen the slices
        // deepest ring (most bytes in flight per CTA) that keeps the wave resident
        for (int ns = kMaxStagesC; ns >= 2; --ns) {
            if (src == SRC_SCORES && ns != 2) continue;  // no ring for a score source
            const size_t smem = csel_smem(src != SRC_SCORES, src == SRC_SCORES ? 0 : r, nq, slice, ns, C).total;
            int optin = 0, dev = 0;
            cudaError_t e = cudaGetDevice(&dev);
            if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
            if (e != cudaSuccess) return e;
            if (smem > (size_t)optin) continue;
            e = ensure_smem(reinterpret_cast<const void *>(kern), smem);
            if (e != cudaSuccess) return e;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
            const int ncl = resident_clusters(kern, C, smem);
            if (ncl < 1) continue;
            if (form == 0 && ncl < BH) continue;
            p->csize = C;
            p->slice = slice;
            p->smem = smem;
            p->grid_y = BH;
            p->nstages = ns;
            return cudaSuccess;
        }
    }
    return cudaErrorNotSupported;
}

}  // namespace

cudaError_t plan_csel(int form, int src, int agg, int B, int Hkv, int T_cap, int r, int nq, int k, CSelPlan *p) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    CSelKey key;
    memset(&key, 0, sizeof key);
    key.dev = dev;
    key.form = form;
    key.src = src;
    key.agg = agg;
    key.B = B;
    key.Hkv = Hkv;
    key.T_cap = T_cap;
    key.r = r;
    key.nq = nq;
    key.k = k;
    {
        std::lock_guard<std::mutex> lk(g_cache_mu);
        for (int i = 0; i < g_cache_n; ++i)
            if (g_cache[i].key == key) {
                if (g_cache[i].err == cudaSuccess) {
                    // the attributes are per device and function: set them again
                    // in case this thread planned nothing on the device yet
                    auto kern = pick_csel(src, r, agg);
                    ensure_smem(reinterpret_cast<const void *>(kern), g_cache[i].plan.smem);
                    cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
                    *p = g_cache[i].plan;
                }
                return g_cache[i].err;
            }
    }
    CSelPlan P{};
    e = plan_csel_uncached(key.form, src, agg, B, Hkv, T_cap, r, nq, k, &P);
    if (e != cudaSuccess && e != cudaErrorNotSupported) return e;  // not cached: a real failure
    std::lock_guard<std::mutex> lk(g_cache_mu);
    CSelEntry &slot = g_cache[g_cache_n < kPlanCache ? g_cache_n++ : (g_cache_next++ % kPlanCache)];
    slot.key = key;
    slot.err = e;
    slot.plan = P;
    if (e == cudaSuccess) *p = P;
    return e;
}

cudaError_t launch_csel(const CSelPlan &p, const CSelArgs &a0, int src, int agg, cudaStream_t s, bool pdl) {
    auto kern = pick_csel(src, a0.r, agg);
    if (!kern) return cudaErrorInvalidValue;
    CSelArgs a = a0;
    a.csize = p.csize;
    a.slice = p.slice;
    a.nstages = p.nstages;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.csize, p.grid_y);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p.csize;
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
        cudaError_t es = ensure_smem(reinterpret_cast<const void *>(kern), cfg.dynamicSmemBytes);
        if (es != cudaSuccess) return es;
    }
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace jssa
