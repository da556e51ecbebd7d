// Decode attention over a token list per (batch, KV head): the gather-free
// indexed path, the dense (full or sliding-window) path, and the dense kernel
// over gathered rows used by the gather-then-dense comparison path.
//
// Method: "Joint Subspace Sparse Attention for Efficient Long-Context
// Decoding", Abstract (gather-free token-level indexed-attention kernel with
// distinct per-KV-head selections under the standard GQA cache layout); news
// item "JSSA makes token-level sparse decoding gather-free", Interpretation
// para 3 (selected tokens read in place through their indices instead of
// staged into a contiguous buffer; a gather step followed by a dense kernel is
// the common alternative).
//
// One CTA handles all G query heads of one KV head for one split of the token
// list, so every K/V row is read once for the whole group.  Rows are staged
// with cp.async (16 B per request; a row of d = 128 bf16 is 256 B) straight
// from their place in the [B, T, Hkv, d] cache, in tiles of NT rows (one
// buffer when a split fits one tile, two for longer lists); rows are padded in
// shared memory so that the logit phase reads them without bank conflicts.
// Logits use fp32 with the softmax scale folded (times log2 e) into q; the
// softmax is online across tiles.  Split partials (unnormalised o, running max
// m, running sum l) are combined by log-sum-exp:
//  * short lists (indexed / gathered): the splits of one (b,h) form one
//    thread-block cluster and combine through distributed shared memory, each
//    CTA finishing a slice of the output;
//  * long lists (dense): partials go to the workspace and the last CTA of the
//    (b,h) to arrive (ticket, no waiting) combines them.
#include <cooperative_groups.h>

#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace cg = cooperative_groups;

namespace jssa {

namespace {

constexpr int NTH = kAttnThreads;
constexpr float kLn2 = 0.693147180559945309417f;
constexpr int kMaxCluster = 16;

template <typename KV, int D>
struct AttnShape {
    static constexpr int ES = (int)sizeof(KV);
    static constexpr int ROWB = D * ES;
    static constexpr int NT_RAW = 16384 / ROWB;
    static constexpr int NT = NT_RAW > 64 ? 64 : (NT_RAW < 16 ? 16 : NT_RAW);  // rows per tile
    static constexpr int TPR = NTH / NT;                                       // threads per row (logits)
    static constexpr int CPR = ROWB / 16;                                      // 16-byte chunks per row
    static constexpr int CPT = CPR / TPR;                                      // chunks per thread
    static constexpr int STRIDE = ROWB + (TPR <= 4 ? 16 * TPR : 16);           // padded row bytes
    static constexpr int EPL = 16 / ES;
    static constexpr int DPT = D >= NTH ? D / NTH : 1;  // output dims per thread
    static constexpr int STAGE = 2 * NT * STRIDE;       // K and V tiles
    static_assert(CPR % TPR == 0, "row split");
};

template <typename KV, int D, int GM, int STAGES>
constexpr size_t attend_smem_bytes() {
    using S = AttnShape<KV, D>;
    size_t st = (size_t)STAGES * S::STAGE;
    const size_t part = (size_t)GM * D * 4;  // cluster partial o reuses the stage buffers
    if (st < part) st = part;
    size_t o = st;
    o += (size_t)GM * D * 4;          // scaled queries
    o += (size_t)S::NT * GM * 4;      // logits / probabilities
    o += (size_t)STAGES * S::NT * 4;  // token ids per stage
    o += 3 * (size_t)GM * 4 + 16 * 4; // m, l, alpha, misc
    return (o + 127) / 128 * 128;
}

template <typename KV, int D, int GM, int SRC, int STAGES, bool CLUSTER>
__global__ void __launch_bounds__(NTH) attend_kernel(AttnArgs a) {
    using S = AttnShape<KV, D>;
    constexpr int NT = S::NT, TPR = S::TPR, CPT = S::CPT, STRIDE = S::STRIDE, EPL = S::EPL, DPT = S::DPT;
    constexpr size_t STAGE_BYTES = ((size_t)STAGES * S::STAGE > (size_t)GM * D * 4) ? (size_t)STAGES * S::STAGE
                                                                                    : (size_t)GM * D * 4;
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *stage0 = smem;
    float *q_s = reinterpret_cast<float *>(smem + STAGE_BYTES);
    float *lg = q_s + GM * D;
    int *tok_s = reinterpret_cast<int *>(lg + NT * GM);
    float *m_run = reinterpret_cast<float *>(tok_s + STAGES * NT);
    float *l_run = m_run + GM;
    float *alpha_s = l_run + GM;
    int *misc = reinterpret_cast<int *>(alpha_s + GM);

    const int tid = threadIdx.x;
    const int split = blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / a.Hkv, h = bh - b * a.Hkv;
    const int G = a.G;

    pdl_trigger();
    pdl_wait();

    const int Tb = clamp_seq(a.seq_lens[b], a.T_cap, a.status);
    int npos = 0, lo = 0;
    if (SRC == ATT_INDEXED) {
        if (a.count) {
            npos = a.count[bh];
            if (npos < 0 || npos > a.k) {
                if (tid == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_INDEX);
                npos = npos < 0 ? 0 : a.k;
            }
        } else {
            const int32_t *lst = a.idx + (size_t)bh * a.k;
            for (int j0 = 0; j0 < a.k; j0 += NTH) {
                const int j = j0 + tid;
                npos += __syncthreads_count(j < a.k && lst[j] >= 0);
            }
        }
    } else if (SRC == ATT_RANGE) {
        lo = (a.window > 0 && Tb > a.window) ? Tb - a.window : 0;
        npos = Tb - lo;
    } else {
        npos = a.count[bh];
        npos = npos < 0 ? 0 : (npos > a.k ? a.k : npos);
    }
    const int p0 = split * a.pos_per_split;
    const int p1 = min(p0 + a.pos_per_split, npos);
    const int ntile = p1 > p0 ? (p1 - p0 + NT - 1) / NT : 0;

    const char *Kb = static_cast<const char *>(a.K);
    const char *Vb = static_cast<const char *>(a.V);
    // stage the token ids of tile j (one global read per row), then its rows
    auto issue = [&](int j, int st) {
        const int pos0 = p0 + j * NT;
        const int rows = min(NT, p1 - pos0);
        int *tk = tok_s + st * NT;
        if (tid < NT) {
            int t = -1;
            if (tid < rows) {
                const int p = pos0 + tid;
                if (SRC == ATT_INDEXED) {
                    t = __ldg(a.idx + (size_t)bh * a.k + p);
                    if (t < 0 || t >= Tb) {
                        if (a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_INDEX);
                        t = -1;
                    }
                } else if (SRC == ATT_RANGE) {
                    t = lo + p;
                } else {
                    t = p;
                }
            }
            tk[tid] = t;
        }
        __syncthreads();
        unsigned char *ks = stage0 + (size_t)st * S::STAGE;
        constexpr int CH = NT * S::CPR;
        for (int c = tid; c < 2 * CH; c += NTH) {
            const int kv = c >= CH;
            const int rem = c - kv * CH;
            const int row = rem / S::CPR, ch = rem - row * S::CPR;
            const int t = tk[row];
            unsigned char *dst = ks + (size_t)kv * NT * STRIDE + (size_t)row * STRIDE + ch * 16;
            if (t >= 0) {
                const long long hp = a.head_div > 1 ? h / a.head_div : h;  // the K/V head this row reads
                const long long off = kv ? ((long long)b * a.v_sb + (long long)t * a.v_st + hp * a.v_sh)
                                         : ((long long)b * a.k_sb + (long long)t * a.k_st + hp * a.k_sh);
                cp_async16(dst, (kv ? Vb : Kb) + off * S::ES + ch * 16, 16);
            } else {
                cp_async16(dst, Kb, 0);
            }
        }
        cp_async_commit();
    };

    // scaled queries of the group and the m / l state (visible after the first wait + sync)
    const KV *q = static_cast<const KV *>(a.q) + ((size_t)b * a.Hq + (size_t)h * G) * D;
    for (int p = tid; p < G * D; p += NTH) q_s[p] = to_f32(q[p]) * a.scale_log2;
    if (tid < GM) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.f;
    }

    if (ntile > 0) issue(0, 0);
    if (STAGES > 1 && ntile > 1) issue(1, 1 % STAGES);

    float acc[GM][DPT];
#pragma unroll
    for (int g = 0; g < GM; ++g)
#pragma unroll
        for (int u = 0; u < DPT; ++u) acc[g][u] = 0.f;
    const int d0 = tid * DPT;
    const bool own = d0 < D;

    const int row = tid / TPR, sub = tid - row * TPR;
    const int lane = tid & 31, warp = tid >> 5;

    for (int j = 0; j < ntile; ++j) {
        if (STAGES > 1 && j + 1 < ntile)
            cp_async_wait<1>();
        else
            cp_async_wait<0>();
        __syncthreads();
        const int st = j % STAGES;
        const unsigned char *Ks = stage0 + (size_t)st * S::STAGE;
        const unsigned char *Vs = Ks + (size_t)NT * STRIDE;
        const int rows = min(NT, p1 - (p0 + j * NT));

        // (a) logits: TPR threads per row, chunks interleaved by thread
        {
            float part[GM];
#pragma unroll
            for (int g = 0; g < GM; ++g) part[g] = 0.f;
#pragma unroll
            for (int cc = 0; cc < CPT; ++cc) {
                const int ch = cc * TPR + sub;
                const uint4 v = *reinterpret_cast<const uint4 *>(Ks + (size_t)row * STRIDE + ch * 16);
                float kf[EPL];
                Vec16<KV>::unpack(v, kf);
#pragma unroll
                for (int g = 0; g < GM; ++g) {
                    if (g < G) {
                        const float *qg = q_s + g * D + ch * EPL;
#pragma unroll
                        for (int e = 0; e < EPL; ++e) part[g] = fmaf(kf[e], qg[e], part[g]);
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < GM; ++g) {
#pragma unroll
                for (int off = 1; off < TPR; off <<= 1) part[g] += __shfl_xor_sync(0xffffffffu, part[g], off);
            }
            if (sub == 0) {
                const bool live = row < rows && tok_s[st * NT + row] >= 0;
#pragma unroll
                for (int g = 0; g < GM; ++g)
                    if (g < G) lg[row * GM + g] = live ? part[g] : -INFINITY;
            }
        }
        __syncthreads();

        // (b) online softmax bookkeeping, one warp per query head
        for (int g = warp; g < G; g += NTH / 32) {
            float mt = -INFINITY;
            for (int r = lane; r < NT; r += 32) mt = fmaxf(mt, lg[r * GM + g]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            const float m_old = m_run[g];
            const float m_new = fmaxf(m_old, mt);
            const float alpha = m_new == -INFINITY ? 1.f : exp2f(m_old - m_new);
            float ps = 0.f;
            for (int r = lane; r < NT; r += 32) {
                const float l = lg[r * GM + g];
                const float p = l == -INFINITY ? 0.f : exp2f(l - m_new);
                lg[r * GM + g] = p;
                ps += p;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
            if (lane == 0) {
                m_run[g] = m_new;
                l_run[g] = l_run[g] * alpha + ps;
                alpha_s[g] = alpha;
            }
        }
        __syncthreads();

        // (c) o += p V over the tile's rows
        if (own) {
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                if (g < G) {
                    const float al = alpha_s[g];
#pragma unroll
                    for (int u = 0; u < DPT; ++u) acc[g][u] *= al;
                }
            }
            for (int r = 0; r < rows; ++r) {
                float v[DPT];
                const KV *vr = reinterpret_cast<const KV *>(Vs + (size_t)r * STRIDE) + d0;
#pragma unroll
                for (int u = 0; u < DPT; ++u) v[u] = to_f32(vr[u]);
                const float *pr = lg + r * GM;
#pragma unroll
                for (int g = 0; g < GM; ++g) {
                    if (g < G) {
                        const float p = pr[g];
#pragma unroll
                        for (int u = 0; u < DPT; ++u) acc[g][u] = fmaf(p, v[u], acc[g][u]);
                    }
                }
            }
        }
        __syncthreads();
        if (STAGES > 1 && j + STAGES < ntile) issue(j + STAGES, st);
    }

    KV *out = static_cast<KV *>(a.out);
    if (a.splits == 1) {
        if (own) {
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                if (g < G) {
                    const float l = l_run[g];
                    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
                    for (int u = 0; u < DPT; ++u)
                        store_elem(out + ((size_t)b * a.Hq + (size_t)h * G + g) * D + d0 + u, acc[g][u] * inv);
                }
            }
        }
        if (a.lse && tid < G) {
            const float l = l_run[tid];
            a.lse[(size_t)b * a.Hq + (size_t)h * G + tid] = l > 0.f ? (m_run[tid] + log2f(l)) * kLn2 : -INFINITY;
        }
        return;
    }

    if constexpr (CLUSTER) {
        // partial o into this CTA's shared memory (the stage buffers are free now)
        float *po = reinterpret_cast<float *>(stage0);
        if (own) {
#pragma unroll
            for (int g = 0; g < GM; ++g)
                if (g < G)
#pragma unroll
                    for (int u = 0; u < DPT; ++u) po[g * D + d0 + u] = acc[g][u];
        }
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        // CTA `split` combines dims [split*slice, (split+1)*slice) of every head
        const int ns = a.splits;
        const int slice = (D + ns - 1) / ns;
        const int c0 = split * slice, c1 = min(D, c0 + slice);
        const int width = c1 - c0;
        for (int p = tid; p < G * (width > 0 ? width : 0); p += NTH) {
            const int g = p / width, c = c0 + (p - g * width);
            float M = -INFINITY;
            for (int s = 0; s < ns; ++s) M = fmaxf(M, *cluster.map_shared_rank(m_run + g, s));
            float L = 0.f, o = 0.f;
            for (int s = 0; s < ns; ++s) {
                const float ms = *cluster.map_shared_rank(m_run + g, s);
                if (ms == -INFINITY) continue;
                const float w = exp2f(ms - M);
                L = fmaf(*cluster.map_shared_rank(l_run + g, s), w, L);
                o = fmaf(*cluster.map_shared_rank(po + g * D + c, s), w, o);
            }
            store_elem(out + ((size_t)b * a.Hq + (size_t)h * G + g) * D + c, L > 0.f ? o / L : 0.f);
            if (a.lse && split == 0 && c == c0)
                a.lse[(size_t)b * a.Hq + (size_t)h * G + g] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
        }
        cluster.sync();  // peers keep their shared memory until every slice is read
        return;
    } else {
        // split partials in the workspace; the last CTA of this (b,h) combines them
        const size_t pbase = ((size_t)bh * a.splits + split) * G;
        if (own) {
#pragma unroll
            for (int g = 0; g < GM; ++g)
                if (g < G)
#pragma unroll
                    for (int u = 0; u < DPT; ++u) a.part_o[(pbase + g) * D + d0 + u] = acc[g][u];
        }
        if (tid < G) {
            a.part_ml[(pbase + tid) * 2 + 0] = m_run[tid];
            a.part_ml[(pbase + tid) * 2 + 1] = l_run[tid];
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) misc[0] = atomicAdd(&a.counters[bh], 1u) == (unsigned)(a.splits - 1);
        __syncthreads();
        if (!misc[0]) return;
        __threadfence();
        for (int g = 0; g < G; ++g) {
            float M = -INFINITY;
            for (int s = 0; s < a.splits; ++s)
                M = fmaxf(M, __ldcg(a.part_ml + (((size_t)bh * a.splits + s) * G + g) * 2));
            float L = 0.f;
            float o[DPT];
#pragma unroll
            for (int u = 0; u < DPT; ++u) o[u] = 0.f;
            for (int s = 0; s < a.splits; ++s) {
                const size_t pb = ((size_t)bh * a.splits + s) * G + g;
                const float ms = __ldcg(a.part_ml + pb * 2);
                if (ms == -INFINITY) continue;
                const float w = exp2f(ms - M);
                L = fmaf(__ldcg(a.part_ml + pb * 2 + 1), w, L);
                if (own) {
#pragma unroll
                    for (int u = 0; u < DPT; ++u) o[u] = fmaf(__ldcg(a.part_o + pb * D + d0 + u), w, o[u]);
                }
            }
            const float inv = L > 0.f ? 1.f / L : 0.f;
            if (own) {
#pragma unroll
                for (int u = 0; u < DPT; ++u)
                    store_elem(out + ((size_t)b * a.Hq + (size_t)h * G + g) * D + d0 + u, o[u] * inv);
            }
            if (a.lse && tid == 0)
                a.lse[(size_t)b * a.Hq + (size_t)h * G + g] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
        }
        if (tid == 0) a.counters[bh] = 0u;
    }
}

// Copy the selected K and V rows of each (b,h) into contiguous [B,Hkv,k,d]
// buffers (the gather step of the gather-then-dense comparison path).  Out-of-
// range indices are dropped (and flagged), keeping the order of the rest.
template <typename KV>
__global__ void __launch_bounds__(NTH) gather_kernel(GatherArgs a) {
    extern __shared__ __align__(16) int g_sm[];
    int *comp = g_sm;       // [k] compacted token ids
    int *tmp = g_sm + a.k;  // [32]
    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int b = bh / a.Hkv, h = bh - b * a.Hkv;
    pdl_trigger();
    pdl_wait();
    const int Tb = clamp_seq(a.seq_lens[b], a.T_cap, a.status);
    const int32_t *lst = a.idx + (size_t)bh * a.k;
    int cnt;
    if (a.count) {
        cnt = a.count[bh];
        if (cnt < 0 || cnt > a.k) {
            if (tid == 0 && blockIdx.y == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_INDEX);
            cnt = cnt < 0 ? 0 : a.k;
        }
    } else {
        cnt = 0;
        for (int j0 = 0; j0 < a.k; j0 += NTH) cnt += __syncthreads_count(j0 + tid < a.k && lst[j0 + tid] >= 0);
    }
    const int per = (cnt + NTH - 1) / NTH;
    const int j0 = min(tid * per, cnt), j1 = min(j0 + per, cnt);
    int c = 0;
    for (int j = j0; j < j1; ++j) c += (lst[j] >= 0 && lst[j] < Tb);
    int total;
    int w = block_excl_scan<NTH>(c, tmp, total);
    for (int j = j0; j < j1; ++j) {
        const int t = lst[j];
        if (t >= 0 && t < Tb) comp[w++] = t;
    }
    if (total != cnt && tid == 0 && blockIdx.y == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_INDEX);
    if (blockIdx.y == 0 && tid == 0) a.gcount[bh] = total;
    __syncthreads();
    const int rpc = (a.k + gridDim.y - 1) / gridDim.y;
    const int r0 = blockIdx.y * rpc, r1 = min(r0 + rpc, total);
    const int cpr = a.d * (int)sizeof(KV) / 16;
    const uint4 *K = static_cast<const uint4 *>(a.K);
    const uint4 *V = static_cast<const uint4 *>(a.V);
    uint4 *gK = static_cast<uint4 *>(a.gK);
    uint4 *gV = static_cast<uint4 *>(a.gV);
    const int copies = a.V ? 2 : 1;  // a latent cache gathers its rows once (V is K)
    for (int p = tid; p < (r1 - r0) * cpr * copies; p += NTH) {
        const int kv = p >= (r1 - r0) * cpr;
        const int rem = p - kv * (r1 - r0) * cpr;
        const int rr = r0 + rem / cpr, ch = rem % cpr;
        const size_t src = (((size_t)b * a.T_cap + comp[rr]) * a.Hkv + h) * cpr + ch;
        const size_t dst = ((size_t)bh * a.k + rr) * cpr + ch;
        if (kv)
            gV[dst] = __ldg(V + src);
        else
            gK[dst] = __ldg(K + src);
    }
}

using AttnKernel = void (*)(AttnArgs);

struct AttnPick {
    AttnKernel kern = nullptr;
    size_t smem = 0;
    int nt = 0;
};

// Long lists (dense): two stages, workspace combine.  Short lists (indexed,
// gathered): one stage when a split fits one tile, cluster combine.
template <typename KV, int D, int GM>
AttnPick pick_attend_g(int src, int stages) {
    AttnPick p;
    p.nt = AttnShape<KV, D>::NT;
    if (src == ATT_RANGE) {
        p.kern = attend_kernel<KV, D, GM, ATT_RANGE, 2, false>;
        p.smem = attend_smem_bytes<KV, D, GM, 2>();
    } else if (src == ATT_INDEXED) {
        p.kern = stages == 1 ? attend_kernel<KV, D, GM, ATT_INDEXED, 1, true>
                             : attend_kernel<KV, D, GM, ATT_INDEXED, 2, true>;
        p.smem = stages == 1 ? attend_smem_bytes<KV, D, GM, 1>() : attend_smem_bytes<KV, D, GM, 2>();
    } else {
        p.kern = stages == 1 ? attend_kernel<KV, D, GM, ATT_RANGE_BH, 1, true>
                             : attend_kernel<KV, D, GM, ATT_RANGE_BH, 2, true>;
        p.smem = stages == 1 ? attend_smem_bytes<KV, D, GM, 1>() : attend_smem_bytes<KV, D, GM, 2>();
    }
    return p;
}

template <typename KV, int D>
AttnPick pick_attend_d(int src, int G, int stages) {
    if (G <= 4) return pick_attend_g<KV, D, 4>(src, stages);
    if (G <= 8) return pick_attend_g<KV, D, 8>(src, stages);
    return pick_attend_g<KV, D, 16>(src, stages);
}

template <typename KV>
AttnPick pick_attend_kv(int src, int d, int G, int stages) {
    switch (d) {
        case 64: return pick_attend_d<KV, 64>(src, G, stages);
        case 128: return pick_attend_d<KV, 128>(src, G, stages);
        case 256: return pick_attend_d<KV, 256>(src, G, stages);
        default: return AttnPick();
    }
}

AttnPick pick_attend(int src, int kv_dtype, int d, int G, int stages) {
    if (G < 1 || G > kMaxG) return AttnPick();
    return kv_dtype == JSSA_BF16 ? pick_attend_kv<__nv_bfloat16>(src, d, G, stages)
                                 : pick_attend_kv<float>(src, d, G, stages);
}

int rows_per_tile(int kv_dtype, int d) {
    const int rowb = d * (kv_dtype == JSSA_BF16 ? 2 : 4);
    int nt = 16384 / rowb;
    return nt > 64 ? 64 : (nt < 16 ? 16 : nt);
}

}  // namespace

cudaError_t plan_attend(int src, int kv_dtype, int d, int G, int B, int Hkv, int npos, AttnPlan *p) {
    const int nt = rows_per_tile(kv_dtype, d);
    const long long BH = (long long)B * Hkv;
    const int sms = device_sm_count();
    if (npos < 1) npos = 1;
    int splits, pps, stages;
    if (src == ATT_RANGE) {
        // long lists: ~16 tiles per CTA, many CTAs (the scheduler balances)
        splits = (npos + 16 * nt - 1) / (16 * nt);
        if (splits < 1) splits = 1;
        pps = (npos + splits - 1) / splits;
        pps = (pps + nt - 1) / nt * nt;
        splits = (npos + pps - 1) / pps;
        stages = 2;
        if (splits > 65535) return cudaErrorInvalidConfiguration;
    } else {
        // short lists: one cluster of splits per (b,h); enough CTAs for about two
        // per SM, at least 16 positions each, at most kMaxCluster splits
        long long want = (2LL * sms + BH - 1) / BH;
        const int by_tile = (npos + nt - 1) / nt;
        const int most = (npos + 15) / 16;
        splits = (int)(want > by_tile ? want : by_tile);
        if (splits > most) splits = most;
        if (splits > kMaxCluster) splits = kMaxCluster;
        if (splits < 1) splits = 1;
        pps = (npos + splits - 1) / splits;
        splits = (npos + pps - 1) / pps;
        stages = pps <= nt ? 1 : 2;
    }
    AttnPick pk;
    for (;;) {
        pk = pick_attend(src, kv_dtype, d, G, stages);
        if (!pk.kern) return cudaErrorInvalidValue;
        cudaError_t e = ensure_smem(reinterpret_cast<const void *>(pk.kern), pk.smem);
        if (e != cudaSuccess) return e;
        if (src == ATT_RANGE || splits == 1) break;
        if (splits > 8) {
            e = cudaFuncSetAttribute(pk.kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
        }
        // the cluster of `splits` CTAs must fit on the device; otherwise halve it
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(splits, 1);
        cfg.blockDim = dim3(NTH);
        cfg.dynamicSmemBytes = pk.smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = splits;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        e = cudaOccupancyMaxActiveClusters(&nclusters, pk.kern, &cfg);
        if (e != cudaSuccess) return e;
        if (nclusters > 0) break;
        splits = (splits + 1) / 2;
        pps = (npos + splits - 1) / splits;
        splits = (npos + pps - 1) / pps;
        stages = pps <= nt ? 1 : 2;
    }
    p->nt = nt;
    p->splits = splits;
    p->pos_per_split = pps;
    p->stages = stages;
    p->smem = pk.smem;
    return cudaSuccess;
}

cudaError_t launch_attend(const AttnPlan &p, int src, const AttnArgs &a0, int kv_dtype, int d, cudaStream_t s,
                          bool pdl) {
    AttnPick pk = pick_attend(src, kv_dtype, d, a0.G, p.stages);
    if (!pk.kern) return cudaErrorInvalidValue;
    AttnArgs a = a0;
    a.splits = p.splits;
    a.pos_per_split = p.pos_per_split;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.splits, a.B * a.Hkv);
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (src != ATT_RANGE && p.splits > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = p.splits;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    {
        cudaError_t es = ensure_smem(reinterpret_cast<const void *>(pk.kern), cfg.dynamicSmemBytes);
        if (es != cudaSuccess) return es;
    }
    return cudaLaunchKernelEx(&cfg, pk.kern, a);
}

cudaError_t launch_gather(const GatherArgs &a, int kv_dtype, cudaStream_t s, bool pdl) {
    const size_t smem = ((size_t)a.k + 32) * sizeof(int);
    const int ys = (a.k + 31) / 32;  // ~32 rows per CTA
    void (*k)(GatherArgs) = kv_dtype == JSSA_BF16 ? gather_kernel<__nv_bfloat16> : gather_kernel<float>;
    return launch_kernel(k, dim3(a.B * a.Hkv, ys), dim3(NTH), smem, s, pdl, a);
}

}  // namespace jssa
