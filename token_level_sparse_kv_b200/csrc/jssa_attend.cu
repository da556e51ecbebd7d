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
// from their place in the [B, T, Hkv, d] cache, double-buffered in tiles of
// NT rows; rows are padded in shared memory so that the logit phase reads
// them without bank conflicts.  Logits use fp32 with the softmax scale folded
// (times log2 e) into q; the softmax is online across tiles; the split partials
// (unnormalised o, running max m, running sum l) go to the workspace and the
// last CTA of each (b, h) to arrive (ticket, no waiting) combines them by
// log-sum-exp and writes out / lse.
#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace jssa {

namespace {

constexpr int NTH = kAttnThreads;
constexpr float kLn2 = 0.693147180559945309417f;

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

template <typename KV, int D, int GM>
size_t attend_smem_bytes() {
    using S = AttnShape<KV, D>;
    size_t o = 2 * (size_t)S::STAGE;           // two stages
    o += (size_t)GM * D * 4;                   // scaled queries
    o += (size_t)S::NT * GM * 4;               // logits / probabilities
    o += 2 * (size_t)S::NT * 4;                // token ids per stage
    o += 3 * (size_t)GM * 4 + 16 * 4;          // m, l, alpha, misc
    return (o + 127) / 128 * 128;
}

template <typename KV, int D, int GM, int SRC>
__global__ void __launch_bounds__(NTH) attend_kernel(AttnArgs a) {
    using S = AttnShape<KV, D>;
    constexpr int NT = S::NT, TPR = S::TPR, CPT = S::CPT, STRIDE = S::STRIDE, EPL = S::EPL, DPT = S::DPT;
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *stage0 = smem;
    float *q_s = reinterpret_cast<float *>(smem + 2 * S::STAGE);
    float *lg = q_s + GM * D;
    int *tok_s = reinterpret_cast<int *>(lg + NT * GM);
    float *m_run = reinterpret_cast<float *>(tok_s + 2 * NT);
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

    // token of list position p (-1 = skip)
    auto token_of = [&](int p) -> int {
        if (SRC == ATT_INDEXED) {
            const int t = __ldg(a.idx + (size_t)bh * a.k + p);
            if (t < 0 || t >= Tb) {
                if (a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_INDEX);
                return -1;
            }
            return t;
        } else if (SRC == ATT_RANGE) {
            return lo + p;
        }
        return p;
    };

    const char *Kb = static_cast<const char *>(a.K);
    const char *Vb = static_cast<const char *>(a.V);
    auto issue = [&](int j, int st) {
        const int pos0 = p0 + j * NT;
        const int rows = min(NT, p1 - pos0);
        unsigned char *ks = stage0 + (size_t)st * S::STAGE;
        constexpr int CH = NT * S::CPR;
        for (int c = tid; c < 2 * CH; c += NTH) {
            const int kv = c >= CH;
            const int rem = c - kv * CH;
            const int row = rem / S::CPR, ch = rem - row * S::CPR;
            int t = -1;
            if (row < rows) t = token_of(pos0 + row);
            unsigned char *dst = ks + (size_t)kv * NT * STRIDE + (size_t)row * STRIDE + ch * 16;
            if (t >= 0) {
                const long long off = kv ? ((long long)b * a.v_sb + (long long)t * a.v_st + (long long)h * a.v_sh)
                                         : ((long long)b * a.k_sb + (long long)t * a.k_st + (long long)h * a.k_sh);
                cp_async16(dst, (kv ? Vb : Kb) + off * S::ES + ch * 16, 16);
            } else {
                cp_async16(dst, Kb, 0);
            }
        }
        if (tid < NT) tok_s[st * NT + tid] = tid < rows ? token_of(pos0 + tid) : -1;
        cp_async_commit();
    };

    if (ntile > 0) issue(0, 0);
    if (ntile > 1) issue(1, 1);

    // scaled queries of the group, m / l state
    const KV *q = static_cast<const KV *>(a.q) + ((size_t)b * a.Hq + (size_t)h * G) * D;
    for (int p = tid; p < G * D; p += NTH) q_s[p] = to_f32(q[p]) * a.scale_log2;
    if (tid < GM) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.f;
    }

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
        if (j + 1 < ntile)
            cp_async_wait<1>();
        else
            cp_async_wait<0>();
        __syncthreads();
        const int st = j & 1;
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
        if (j + 2 < ntile) issue(j + 2, st);
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

    // split partials, then the last CTA of this (b,h) combines them
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

// Copy the selected K and V rows of each (b,h) into contiguous [B,Hkv,k,d]
// buffers (the gather step of the gather-then-dense comparison path).  Out-of-
// range indices are dropped (and flagged), keeping the order of the rest.
template <typename KV>
__global__ void __launch_bounds__(NTH) gather_kernel(GatherArgs a) {
    extern __shared__ __align__(16) int g_sm[];
    int *comp = g_sm;           // [k] compacted token ids
    int *tmp = g_sm + a.k;      // [32]
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
    for (int p = tid; p < (r1 - r0) * cpr * 2; p += NTH) {
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

template <typename KV, int D, int GM>
void (*pick_attend_src(int src))(AttnArgs) {
    switch (src) {
        case ATT_INDEXED: return attend_kernel<KV, D, GM, ATT_INDEXED>;
        case ATT_RANGE: return attend_kernel<KV, D, GM, ATT_RANGE>;
        default: return attend_kernel<KV, D, GM, ATT_RANGE_BH>;
    }
}

template <typename KV, int D>
void (*pick_attend_g(int src, int G, size_t *smem))(AttnArgs) {
    if (G <= 4) {
        *smem = attend_smem_bytes<KV, D, 4>();
        return pick_attend_src<KV, D, 4>(src);
    }
    if (G <= 8) {
        *smem = attend_smem_bytes<KV, D, 8>();
        return pick_attend_src<KV, D, 8>(src);
    }
    *smem = attend_smem_bytes<KV, D, 16>();
    return pick_attend_src<KV, D, 16>(src);
}

template <typename KV>
void (*pick_attend_d(int src, int d, int G, size_t *smem, int *nt))(AttnArgs) {
    switch (d) {
        case 64: *nt = AttnShape<KV, 64>::NT; return pick_attend_g<KV, 64>(src, G, smem);
        case 128: *nt = AttnShape<KV, 128>::NT; return pick_attend_g<KV, 128>(src, G, smem);
        case 256: *nt = AttnShape<KV, 256>::NT; return pick_attend_g<KV, 256>(src, G, smem);
        default: return nullptr;
    }
}

void (*pick_attend(int src, int kv_dtype, int d, int G, size_t *smem, int *nt))(AttnArgs) {
    if (G < 1 || G > kMaxG) return nullptr;
    return kv_dtype == JSSA_BF16 ? pick_attend_d<__nv_bfloat16>(src, d, G, smem, nt)
                                 : pick_attend_d<float>(src, d, G, smem, nt);
}

}  // namespace

cudaError_t plan_attend(int src, int kv_dtype, int d, int G, int B, int Hkv, int npos, AttnPlan *p) {
    size_t smem = 0;
    int nt = 0;
    auto kern = pick_attend(src, kv_dtype, d, G, &smem, &nt);
    if (!kern) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, NTH, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    const long long BH = (long long)B * Hkv;
    const int sms = device_sm_count();
    if (npos < 1) npos = 1;
    int splits;
    if (src == ATT_RANGE) {
        // long lists: ~16 tiles per CTA, many CTAs (the scheduler balances)
        splits = (npos + 16 * nt - 1) / (16 * nt);
    } else {
        // short lists: enough CTAs for two per SM, at least 16 positions each
        long long want = (2LL * sms + BH - 1) / BH;
        int by_tile = (npos + nt - 1) / nt;
        int most = (npos + 15) / 16;
        splits = (int)(want > by_tile ? want : by_tile);
        if (splits > most) splits = most;
    }
    if (splits < 1) splits = 1;
    int pps = (npos + splits - 1) / splits;
    if (src == ATT_RANGE) pps = (pps + nt - 1) / nt * nt;
    splits = (npos + pps - 1) / pps;
    if (splits > 65535) return cudaErrorInvalidConfiguration;
    p->nt = nt;
    p->splits = splits;
    p->pos_per_split = pps;
    p->stages = 2;
    p->smem = smem;
    return cudaSuccess;
}

cudaError_t launch_attend(const AttnPlan &p, int src, const AttnArgs &a0, int kv_dtype, int d, cudaStream_t s,
                          bool pdl) {
    size_t smem = 0;
    int nt = 0;
    auto kern = pick_attend(src, kv_dtype, d, a0.G, &smem, &nt);
    if (!kern) return cudaErrorInvalidValue;
    AttnArgs a = a0;
    a.splits = p.splits;
    a.pos_per_split = p.pos_per_split;
    return launch_kernel(kern, dim3(p.splits, a.B * a.Hkv), dim3(NTH), p.smem, s, pdl, a);
}

cudaError_t launch_gather(const GatherArgs &a, int kv_dtype, cudaStream_t s, bool pdl) {
    const size_t smem = ((size_t)a.k + 32) * sizeof(int);
    const int ys = (a.k + 31) / 32;  // ~32 rows per CTA
    void (*k)(GatherArgs) = kv_dtype == JSSA_BF16 ? gather_kernel<__nv_bfloat16> : gather_kernel<float>;
    return launch_kernel(k, dim3(a.B * a.Hkv, ys), dim3(NTH), smem, s, pdl, a);
}

}  // namespace jssa
