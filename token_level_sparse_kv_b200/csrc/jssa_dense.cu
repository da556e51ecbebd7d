// Dense decode attention over a contiguous token range per (batch, KV head),
// bf16, on the tensor cores: the full-KV and sliding-window comparison paths
// and the dense pass of gather-then-dense.
//
// Method: "Joint Subspace Sparse Attention for Efficient Long-Context
// Decoding", Abstract (speedups are reported against full-KV attention);
// news item "JSSA makes token-level sparse decoding gather-free",
// Interpretation para 3 (a gather step followed by a dense attention kernel
// is the common alternative to reading the selected rows in place) and
// Perspective para 1 (hybrid models pair a sparse global layer with a dense
// sliding-window local layer).
//
// The pass is bound by HBM bandwidth (4 flop per byte of K and V at four
// query heads per KV head), so its design is about keeping bytes in flight:
//  * a persistent grid of one CTA per SM walks a contiguous share of the
//    flattened (row, tile) list, rows being (b, h) pairs and tiles 64 tokens;
//  * one producer thread streams each tile's K and V rows with TMA tiled
//    loads (a 4-D map over the [B, T, Hkv, d] cache, or a 3-D map over a
//    gathered [B*Hkv, k, d] buffer), 128-byte swizzled, into a ring of
//    stages in shared memory (full / empty mbarriers, evict-first L2 hint);
//  * four consumer warps take 16 tokens of every tile each and run the two
//    products on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 out)
//    with the query heads of the KV head padded to 16 rows:
//      S = Q K^T   (ldmatrix of the swizzled K rows),
//      O += P V    (P = exp2(S - m) rounded to bf16, taken straight from the
//                   S accumulators as the A operand; ldmatrix.trans of V),
//    with an online softmax in fp32 (log2 domain) per warp;
//  * at the end of a row's segment each warp writes its unnormalised partial
//    (O, running max, running sum) to the workspace; a second kernel, chained
//    with programmatic dependent launch, merges each (row, head)'s partials
//    by log-sum-exp with one thread per output dim (a short row, such as a
//    1024-token window, is covered by up to ten CTAs: merging its 40
//    partials inside one CTA was latency-bound).
// Tiles past a row's end are skipped (no load); positions past it inside a
// tile are masked.  The CTA's rows are independent, so nothing waits on
// another CTA.
#include <cuda.h>

#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace jssa {

namespace {

constexpr int kNT = 64;                  // tokens per tile
constexpr int kNW = 4;                   // consumer warps, 16 tokens of each tile apiece
constexpr int kThr = (kNW + 1) * 32;     // + one producer warp
constexpr int kBoxBytes = kNT * 128;     // one TMA box: 64 rows x 64 bf16 columns (128 bytes)
constexpr size_t kStageBudget = 200 * 1024;

template <int D>
struct DenseShape {
    static constexpr int NB = D / 64;                  // boxes per K (or V) row
    static constexpr int STAGE = 2 * NB * kBoxBytes;   // K and V of one tile
    static constexpr int STAGES = (int)(kStageBudget / STAGE) > 8 ? 8 : (int)(kStageBudget / STAGE);
    static constexpr int QSTR = D * 2 + 16;            // padded row of the query tile (bytes)
};

template <int D>
constexpr size_t dense_smem_bytes() {
    using S = DenseShape<D>;
    size_t o = (size_t)S::STAGES * S::STAGE;  // ring (1024-byte aligned stages)
    o += 16 * (size_t)S::QSTR;                // query tile
    o += 16 * (size_t)D * 4;                  // merge buffer of the warps' O (fp32)
    o += kNW * 16 * 8;                        // the warps' (max, sum) per row
    o += 2 * (size_t)S::STAGES * 8;           // full / empty barriers
    o += 64;                                  // flags
    return o + 1024;                          // alignment slack of the dynamic base
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kNW * 32) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi, float &sum) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    sum += __low2float(p) + __high2float(p);
    return *reinterpret_cast<const uint32_t *>(&p);
}

// TMA tiled loads (no multicast), completing on `bar`.
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            uint64_t *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            uint64_t *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// Token range [lo, hi) of row bh: the cache (the last `window` tokens of
// T_b, or all of them) or the gathered rows (count[bh] of them).
__device__ __forceinline__ void row_range(const DenseArgs &a, int bh, int &lo, int &hi) {
    if (a.count) {
        int c = a.count[bh];
        hi = c < 0 ? 0 : (c > a.k ? a.k : c);
        lo = 0;
    } else {
        const int b = bh / a.Hkv;
        const int Tb = clamp_seq(a.seq_lens[b], a.T_cap, a.status);
        lo = (a.window > 0 && Tb > a.window) ? Tb - a.window : 0;
        hi = Tb;
    }
}

template <int D>
__global__ void __launch_bounds__(kThr, 1)
    dense_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, DenseArgs a) {
    using S = DenseShape<D>;
    constexpr int NB = S::NB, STAGES = S::STAGES, QSTR = S::QSTR;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *ring = smem;
    unsigned char *q_s = ring + (size_t)STAGES * S::STAGE;
    float *obuf = reinterpret_cast<float *>(q_s + 16 * QSTR);        // [16][D]
    float2 *mlw = reinterpret_cast<float2 *>(obuf + 16 * D);         // [kNW][16]
    uint64_t *full = reinterpret_cast<uint64_t *>(mlw + kNW * 16);
    uint64_t *empty = full + STAGES;
    volatile int *flags = reinterpret_cast<volatile int *>(empty + STAGES);  // [0] abort

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long total = a.total_tiles;
    const int rt = a.row_tiles;
    // the CTA's tiles: a contiguous share of the flattened (row, tile) list,
    // or (short problems) one of row_split equal parts of a single row
    long long i0, i1;
    if (a.row_split > 0) {
        const int bhs = blockIdx.x / a.row_split, part = blockIdx.x - bhs * a.row_split;
        i0 = (long long)bhs * rt + (long long)part * rt / a.row_split;
        i1 = (long long)bhs * rt + (long long)(part + 1) * rt / a.row_split;
    } else {
        i0 = (long long)blockIdx.x * total / a.grid;
        i1 = (long long)(blockIdx.x + 1) * total / a.grid;
    }

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kNW);
        }
        fence_barrier_init();
        flags[0] = 0;
    }
    if (tid == kNW * 32) {
        // the tensor maps are kernel parameters: fetch them into the TMA
        // unit's cache while the previous kernel may still be running
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)) : "memory");
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();
    if (i0 >= i1) return;

    if (warp == kNW) {
        // ------------------------------------------------------- producer ---
        if (lane != 0) return;
        const uint64_t pol = policy_evict_first();
        int bh = (int)(i0 / rt), j = (int)(i0 - (long long)bh * rt);
        int lo = 0, hi = 0;
        row_range(a, bh, lo, hi);
        long long n = 0;
        for (long long i = i0; i < i1; ++i, ++n) {
            const int s = (int)(n % STAGES);
            if (n >= STAGES && !wait_or_abort(&empty[s], (uint32_t)((n / STAGES) - 1) & 1u, flags)) {
                flags[0] = 1;
                break;
            }
            const int t0 = lo + j * kNT;
            if (t0 < hi) {
                unsigned char *st = ring + (size_t)s * S::STAGE;
                mbar_arrive_expect_tx(&full[s], (uint32_t)S::STAGE);
                const int b = bh / a.Hkv, h = bh - b * a.Hkv;
#pragma unroll
                for (int c = 0; c < NB; ++c) {
                    if (a.count) {
                        tma_load_3d(st + c * kBoxBytes, &tmK, c * 64, t0, bh, &full[s], pol);
                        tma_load_3d(st + (NB + c) * kBoxBytes, &tmV, c * 64, t0, bh, &full[s], pol);
                    } else {
                        tma_load_4d(st + c * kBoxBytes, &tmK, c * 64, h, t0, b, &full[s], pol);
                        tma_load_4d(st + (NB + c) * kBoxBytes, &tmV, c * 64, h, t0, b, &full[s], pol);
                    }
                }
            } else {
                mbar_arrive(&full[s]);  // past the row's end: nothing to load
            }
            if (++j == rt) {
                j = 0;
                ++bh;
                if (i + 1 < i1) row_range(a, bh, lo, hi);
            }
        }
        // drain: every load this thread issued completes before the CTA exits
        for (long long q = n > STAGES ? n - STAGES : 0; q < n; ++q)
            (void)mbar_wait_bounded(&full[q % STAGES], (uint32_t)(q / STAGES) & 1u);
        return;
    }

    // ----------------------------------------------------------- consumers ---
    const int gid = lane >> 2, tig = lane & 3;
    const int ctid = tid;  // 0 .. kNW*32-1
    const uint32_t ring_a = smem_u32(ring), q_a = smem_u32(q_s);
    const int G = a.G;
    const int parts_stride = a.part_stride;  // partial slots per row
    auto load_q = [&](int bh) {
        const int b = bh / a.Hkv, h = bh - b * a.Hkv;
        const uint4 *qg = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.q) +
                                                          ((size_t)b * a.Hq + (size_t)h * G) * D);
        constexpr int CPR = D / 8;
        for (int c = ctid; c < 16 * CPR; c += kNW * 32) {
            const int g = c / CPR, ch = c - g * CPR;
            *reinterpret_cast<uint4 *>(q_s + g * QSTR + ch * 16) = g < G ? qg[g * CPR + ch] : make_uint4(0, 0, 0, 0);
        }
    };

    int bh = (int)(i0 / rt), j = (int)(i0 - (long long)bh * rt);
    int lo = 0, hi = 0;
    row_range(a, bh, lo, hi);
    load_q(bh);
    consumer_sync();

    float o[D / 8][4];
    float mrun[2], lrun[2];
    auto reset = [&]() {
#pragma unroll
        for (int dt = 0; dt < D / 8; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
        mrun[0] = mrun[1] = -INFINITY;
        lrun[0] = lrun[1] = 0.f;
    };
    reset();

    long long n = 0;
    for (long long i = i0; i < i1; ++i, ++n) {
        const int s = (int)(n % STAGES);
        if (!wait_or_abort(&full[s], (uint32_t)(n / STAGES) & 1u, flags)) {
            flags[0] = 1;
            if (lane == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_TIMEOUT);
            break;
        }
        const int t0 = lo + j * kNT;
        const int tw = t0 + warp * 16;  // this warp's first token
        if (tw < hi) {
            const uint32_t Ks = ring_a + (uint32_t)(s * S::STAGE);
            const uint32_t Vs = Ks + (uint32_t)(NB * kBoxBytes);
            // S = Q K^T over the warp's 16 tokens (two 8-token tiles)
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            {
                const int r = warp * 16 + (lane & 7) + ((lane >> 4) << 3);  // token row in the tile
                const int half = (lane >> 3) & 1;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                    ldsm_x4(q_a + (lane & 15) * QSTR + (2 * ks + (lane >> 4)) * 16, a0, a1, a2, a3);
                    const int c = 2 * ks + half, box = c >> 3, cc = c & 7;
                    ldsm_x4(Ks + box * kBoxBytes + r * 128 + ((cc ^ (r & 7)) << 4), b0, b1, b2, b3);
                    mma16816(sc[0], a0, a1, a2, a3, b0, b1);
                    mma16816(sc[1], a0, a1, a2, a3, b2, b3);
                }
            }
            // online softmax of the warp's rows gid, gid + 8 (log2 domain)
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = tw + nt * 8 + 2 * tig + (e & 1);
                    const float v = t < hi ? sc[nt][e] * a.scale_log2 : -INFINITY;
                    sc[nt][e] = v;
                    mx[e >> 1] = fmaxf(mx[e >> 1], v);
                }
            float corr[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
                const float mn = fmaxf(mrun[r], mx[r]);
                corr[r] = mrun[r] == -INFINITY ? 0.f : exp2f(mrun[r] - mn);
                mrun[r] = mn;
            }
            float p[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float m = mrun[e >> 1];
                    p[nt][e] = sc[nt][e] == -INFINITY ? 0.f : exp2f(sc[nt][e] - m);
                }
            float rs0 = 0.f, rs1 = 0.f;
            const uint32_t pa0 = pack_bf16(p[0][0], p[0][1], rs0);
            const uint32_t pa1 = pack_bf16(p[0][2], p[0][3], rs1);
            const uint32_t pa2 = pack_bf16(p[1][0], p[1][1], rs0);
            const uint32_t pa3 = pack_bf16(p[1][2], p[1][3], rs1);
            lrun[0] = lrun[0] * corr[0] + rs0;
            lrun[1] = lrun[1] * corr[1] + rs1;
            // V rows past the row's end (the tail of its last tile) may hold
            // anything, NaN included, and 0 * NaN is NaN: zero them first
            if (tw + 16 > hi) {
                unsigned char *vg = ring + (size_t)s * S::STAGE + (size_t)NB * kBoxBytes;
                const int r0 = max(hi - t0, warp * 16), nrow = warp * 16 + 16 - r0;
                for (int c = lane; c < nrow * NB * 8; c += 32) {
                    const int row = r0 + c / (NB * 8), rem = c % (NB * 8);
                    *reinterpret_cast<uint4 *>(vg + (rem >> 3) * kBoxBytes + row * 128 + (rem & 7) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
                fence_async_smem();  // before the stage is refilled by TMA
                __syncwarp();
            }
            // O = O * corr + P V (two 8-dim output tiles per ldmatrix)
            const int r = warp * 16 + (lane & 15);
            const int second = lane >> 4;
#pragma unroll
            for (int dt = 0; dt < D / 8; dt += 2) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    o[dt + u][0] *= corr[0];
                    o[dt + u][1] *= corr[0];
                    o[dt + u][2] *= corr[1];
                    o[dt + u][3] *= corr[1];
                }
                const int c = dt + second, box = c >> 3, cc = c & 7;
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(Vs + box * kBoxBytes + r * 128 + ((cc ^ (r & 7)) << 4), b0, b1, b2, b3);
                mma16816(o[dt], pa0, pa1, pa2, pa3, b0, b1);
                mma16816(o[dt + 1], pa0, pa1, pa2, pa3, b2, b3);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        const bool seg_end = (j == rt - 1) || (i == i1 - 1);
        if (seg_end) {
            // the CTA's partial of the row: the four warps' (O, max, sum) merged
            // in shared memory, then one unnormalised partial per segment
            const long long first = (long long)bh * rt;
            const int slot = a.row_split > 0 ? (int)blockIdx.x % a.row_split
                                             : (int)blockIdx.x - (int)(((first + 1) * a.grid - 1) / total);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                lrun[r] += __shfl_xor_sync(0xffffffffu, lrun[r], 1);
                lrun[r] += __shfl_xor_sync(0xffffffffu, lrun[r], 2);
                if (tig == 0) mlw[warp * 16 + gid + 8 * r] = make_float2(mrun[r], lrun[r]);
            }
            consumer_sync();
            // the warps add their rescaled O into the buffer in turn (no atomics)
            float wgt[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int g = gid + 8 * r;
                float M = -INFINITY;
#pragma unroll
                for (int q = 0; q < kNW; ++q) M = fmaxf(M, mlw[q * 16 + g].x);
                wgt[r] = mrun[r] == -INFINITY ? 0.f : exp2f(mrun[r] - M);
            }
#pragma unroll 1
            for (int turn = 0; turn < kNW; ++turn) {
                if (warp == turn) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int g = gid + 8 * r;
                        if (g < G) {
                            float2 *ob = reinterpret_cast<float2 *>(obuf + g * D + 2 * tig);
#pragma unroll
                            for (int dt = 0; dt < D / 8; ++dt) {
                                float2 v = turn ? ob[dt * 4] : make_float2(0.f, 0.f);
                                v.x = fmaf(o[dt][2 * r], wgt[r], v.x);
                                v.y = fmaf(o[dt][2 * r + 1], wgt[r], v.y);
                                ob[dt * 4] = v;
                            }
                        }
                    }
                }
                consumer_sync();
            }
            const size_t pidx = (size_t)bh * parts_stride + slot;
            for (int e = ctid; e < G * D; e += kNW * 32) a.part_o[pidx * G * D + e] = obuf[e];
            if (ctid < G) {
                float M = -INFINITY, L = 0.f;
#pragma unroll
                for (int q = 0; q < kNW; ++q) M = fmaxf(M, mlw[q * 16 + ctid].x);
#pragma unroll
                for (int q = 0; q < kNW; ++q) {
                    const float2 v = mlw[q * 16 + ctid];
                    if (v.x != -INFINITY) L = fmaf(v.y, exp2f(v.x - M), L);
                }
                *reinterpret_cast<float2 *>(a.part_ml + (pidx * G + ctid) * 2) = make_float2(M, L);
            }
            if (i + 1 < i1) {
                ++bh;
                j = 0;
                row_range(a, bh, lo, hi);
                consumer_sync();  // every warp is done with the old query tile
                load_q(bh);
                consumer_sync();
                reset();
            }
        } else {
            ++j;
        }
    }
}

// Log-sum-exp merge of a row's partials (one per CTA segment that covered
// it; empty partials carry O = 0 and max -inf): one CTA per (row, head), one thread per output dim.  Chained
// after the dense kernel with programmatic dependent launch.
template <int D>
__global__ void __launch_bounds__(D) dense_combine_kernel(DenseArgs a) {
    __shared__ float stat[2];
    pdl_trigger();
    pdl_wait();
    const int bh = blockIdx.x, g = blockIdx.y, d = threadIdx.x;
    const int G = a.G, rt = a.row_tiles;
    const long long total = a.total_tiles, first = (long long)bh * rt;
    const int np = a.row_split > 0 ? a.row_split
                                   : (int)(((first + rt) * a.grid - 1) / total) - (int)(((first + 1) * a.grid - 1) / total) + 1;
    const size_t pb = (size_t)bh * a.part_stride;
    if (d < 32) {
        float M = -INFINITY;
        for (int q = d; q < np; q += 32) M = fmaxf(M, __ldcg(a.part_ml + ((pb + q) * G + g) * 2));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float L = 0.f;
        if (M != -INFINITY)
            for (int q = d; q < np; q += 32) {
                const float2 ml = __ldcg(reinterpret_cast<const float2 *>(a.part_ml + ((pb + q) * G + g) * 2));
                L += ml.x == -INFINITY ? 0.f : ml.y * exp2f(ml.x - M);
            }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
        if (d == 0) {
            stat[0] = M;
            stat[1] = L;
        }
    }
    __syncthreads();
    const float M = stat[0], L = stat[1];
    float acc = 0.f;
    if (M != -INFINITY) {
#pragma unroll 8
        for (int q = 0; q < np; ++q) {
            const float m = __ldcg(a.part_ml + ((pb + q) * G + g) * 2);
            const float o = __ldcg(a.part_o + ((pb + q) * G + g) * D + d);
            acc = fmaf(o, m == -INFINITY ? 0.f : exp2f(m - M), acc);
        }
    }
    const int b = bh / a.Hkv, h = bh - b * a.Hkv;
    const size_t row = (size_t)b * a.Hq + (size_t)h * G + g;
    static_cast<__nv_bfloat16 *>(a.out)[row * D + d] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
    if (d == 0 && a.lse) a.lse[row] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

using DenseKernel = void (*)(const CUtensorMap, const CUtensorMap, DenseArgs);

DenseKernel pick_dense(int d, size_t *smem) {
    switch (d) {
        case 64: *smem = dense_smem_bytes<64>(); return dense_tc_kernel<64>;
        case 128: *smem = dense_smem_bytes<128>(); return dense_tc_kernel<128>;
        case 256: *smem = dense_smem_bytes<256>(); return dense_tc_kernel<256>;
        default: return nullptr;
    }
}

// Map over bf16 rows of d elements: boxes of 64 columns x 64 rows; rank 4
// {d, Hkv, T, B} over the cache, rank 3 {d, k, B*Hkv} over a gathered buffer.
cudaError_t encode_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides) {
    cuuint32_t box[4] = {64, 1, 1, 1};
    box[rank == 4 ? 2 : 1] = kNT;
    return encode_tiled_bf16(m, base, rank, dims, strides, box);
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
        tried = true;
    }
    return fn;
}

bool tensor_maps_available() { return encode_fn() != nullptr; }

cudaError_t encode_tiled_bf16(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                              const cuuint64_t *strides, const cuuint32_t *box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int dense_part_stride(int B, int Hkv) {
    // partial slots per row: a row spans at most ceil(grid / rows) + 1 CTAs
    // of the persistent grid (grid <= SMs), whatever the row length
    const long long BH = (long long)B * Hkv;
    const long long sms = device_sm_count();
    return (int)((sms + BH - 1) / BH + 1);
}

cudaError_t plan_dense(int d, int B, int Hkv, int row_len, DensePlan *p) {
    size_t smem = 0;
    DenseKernel k = pick_dense(d, &smem);
    if (!k) return cudaErrorNotSupported;
    if (!tensor_maps_available()) return cudaErrorNotSupported;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(k), smem);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kThr, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorNotSupported;
    if (row_len < 1) row_len = 1;
    p->row_tiles = (row_len + kNT - 1) / kNT;
    p->total_tiles = (long long)B * Hkv * p->row_tiles;
    const long long sms = device_sm_count(), BH = (long long)B * Hkv;
    long long g = sms;
    if (g > p->total_tiles) g = p->total_tiles;
    if (g < 1) g = 1;
    p->grid = (int)g;
    p->row_split = 0;
    p->part_stride = dense_part_stride(B, Hkv);
    // short problems (under four tiles per SM): split each row evenly, so that
    // no CTA covers the end of one row and the start of the next
    if (p->total_tiles < 4 * sms && BH <= sms) {
        long long sp = sms / BH;
        if (sp > p->row_tiles) sp = p->row_tiles;
        if (sp < 1) sp = 1;
        p->row_split = (int)sp;
        p->grid = (int)(BH * sp);
    }
    p->smem = smem;
    return cudaSuccess;
}

cudaError_t launch_dense(const DensePlan &p, const DenseArgs &a0, const void *K, const void *V, int d,
                         cudaStream_t s, bool pdl) {
    size_t smem = 0;
    DenseKernel k = pick_dense(d, &smem);
    if (!k) return cudaErrorInvalidValue;
    DenseArgs a = a0;
    a.row_tiles = p.row_tiles;
    a.total_tiles = p.total_tiles;
    a.grid = p.grid;
    a.part_stride = p.part_stride;
    a.row_split = p.row_split;
    CUtensorMap mk, mv;
    cudaError_t e;
    if (a.count) {  // gathered [B*Hkv, k, d]
        const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)a.k, (cuuint64_t)a.B * a.Hkv};
        const cuuint64_t str[2] = {(cuuint64_t)d * 2, (cuuint64_t)a.k * d * 2};
        e = encode_map(&mk, K, 3, dims, str);
        if (e == cudaSuccess) e = encode_map(&mv, V, 3, dims, str);
    } else {  // the cache [B, T_cap, Hkv, d]
        const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)a.Hkv, (cuuint64_t)a.T_cap, (cuuint64_t)a.B};
        const cuuint64_t str[3] = {(cuuint64_t)d * 2, (cuuint64_t)a.Hkv * d * 2, (cuuint64_t)a.T_cap * a.Hkv * d * 2};
        e = encode_map(&mk, K, 4, dims, str);
        if (e == cudaSuccess) e = encode_map(&mv, V, 4, dims, str);
    }
    if (e != cudaSuccess) return e;
    e = launch_kernel(k, dim3(p.grid), dim3(kThr), smem, s, pdl, mk, mv, a);
    if (e != cudaSuccess) return e;
    void (*c)(DenseArgs) = d == 64 ? dense_combine_kernel<64> : (d == 128 ? dense_combine_kernel<128>
                                                                          : dense_combine_kernel<256>);
    return launch_kernel(c, dim3(a.B * a.Hkv, a.G), dim3(d), 0, s, true, a);
}

}  // namespace jssa
