// Attention of the 128 query heads of a latent-cache (multi-head latent
// attention) layer over a contiguous token range per batch row, on the
// 5th-generation tensor cores: the dense full-KV comparison path of the
// latent cache and the dense pass of its gather-then-dense path.
//
// Method: news item "JSSA makes token-level sparse decoding gather-free",
// Perspective para 1 (MLA models: the selection runs over the shared latent
// cache) and Interpretation para 3 (a gather step followed by a dense kernel
// is the alternative to reading the selected rows in place); "Joint Subspace
// Sparse Attention for Efficient Long-Context Decoding", Abstract (speedups
// against full-KV attention).
//
// A latent row of 576 bf16 is the key (all 576 dims) and the value (its first
// 512 dims) of its token.  The range is long (a whole 64K-token row), so the
// products must accumulate across tiles of 128 tokens, and tensor memory (512
// columns of 128 lanes) cannot hold a 128-head x 512 output next to the
// logits.  The products are therefore taken with the tokens on the M side and
// 64 heads per CTA (two CTAs per batch row share its tiles through the L2):
//   S^T[128 tokens x 64 heads] = K_tile[128 x 576] . Q_half^T        (TMEM cols 0..63)
//   O^T[512 dv x 64 heads]    += V_tile^T[512 x 128] . P^T[128 x 64] (four 128-row blocks, cols 128..383)
// K tiles arrive by TMA as nine 128-byte-swizzled 64-column blocks (K-major
// A operand of the first product, MN-major A operand of the second); the
// query half stays resident (nine 8 KiB blocks, K-major B operand).  The
// softmax runs per head over the tile's tokens in fp32 (log2 domain): column
// maxima and sums are reduced across the 128 token lanes with a halving
// butterfly inside each warp and shared memory across warps.  P^T (bf16,
// MN-major B operand) overwrites the tile's rope block, which only the first
// product reads.  The running maximum of a head is raised only when a tile
// exceeds it by more than 2^8 (the weights stay <= 256 otherwise), so the
// accumulated O^T is rescaled in tensor memory rarely; O / l is exact either
// way.  Splits of the token range write (O, max, sum) partials that the
// latent-cache combine kernel merges by log-sum-exp.
#include <cuda.h>

#include "jssa_common.cuh"
#include "jssa_internal.h"
#include "jssa_tc.cuh"

namespace jssa {

namespace {

constexpr int kD = 576, kDv = 512, kH = 128, kHC = 64, kTok = 128, kThr = 128;
constexpr int kKB = 9;                  // 64-column blocks of a latent row
constexpr int kKBlk = kTok * 128;       // 16 KiB: 128 token rows x 64 columns
constexpr int kQBlk = kHC * 128;        // 8 KiB: 64 head rows x 64 columns
constexpr uint32_t kColO = 128;         // TMEM column of O^T block 0 (S^T at 0)
constexpr float kLazy = 8.f;            // log2 headroom before the running max is raised

struct MlaSmem {
    static constexpr size_t K = 0;
    static constexpr size_t Q = K + (size_t)kKB * kKBlk;
    static constexpr size_t BAR = Q + (size_t)kKB * kQBlk;     // kfull[9], qfull, sdone, odone
    static constexpr size_t RED = BAR + 16 * 8;                // [4 warps][64] column partials
    static constexpr size_t MREF = RED + 4 * 64 * 4;           // [64] running max (log2 domain)
    static constexpr size_t LSUM = MREF + 64 * 4;              // [64] running sum
    static constexpr size_t CORR = LSUM + 64 * 4;              // [64] this tile's correction
    static constexpr size_t MISC = CORR + 64 * 4;              // tmem address, flags
    static constexpr size_t END = MISC + 64;
    static constexpr size_t TOTAL = END + 1024;                // alignment slack of the base
};
static_assert(MlaSmem::TOTAL <= 232448, "shared memory");

// Warp-wide reduction of 64 columns held one row per lane: afterwards lane L
// holds the reduction of columns 2L and 2L + 1 (v is overwritten).
template <bool MAX>
__device__ __forceinline__ void col_reduce64(float (&v)[64], int lane, float &c0, float &c1) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step, n = 64 >> step;
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int c = 0; c < n / 2; ++c) {
            const float send = up ? v[c] : v[c + n / 2];
            const float keep = up ? v[c + n / 2] : v[c];
            const float r = __shfl_xor_sync(0xffffffffu, send, o);
            v[c] = MAX ? fmaxf(keep, r) : keep + r;
        }
    }
    c0 = v[0];
    c1 = v[1];
}

__global__ void __launch_bounds__(kThr, 1)
    mla_range_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                     MlaRangeArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *sK = smem + MlaSmem::K;
    unsigned char *sQ = smem + MlaSmem::Q;
    uint64_t *kfull = reinterpret_cast<uint64_t *>(smem + MlaSmem::BAR);
    uint64_t *qfull = kfull + kKB, *sdone = kfull + kKB + 1, *odone = kfull + kKB + 2;
    float *red = reinterpret_cast<float *>(smem + MlaSmem::RED);
    float *mref = reinterpret_cast<float *>(smem + MlaSmem::MREF);
    float *lsum = reinterpret_cast<float *>(smem + MlaSmem::LSUM);
    float *corr = reinterpret_cast<float *>(smem + MlaSmem::CORR);
    uint32_t *tptr = reinterpret_cast<uint32_t *>(smem + MlaSmem::MISC);
    volatile int *flag = reinterpret_cast<volatile int *>(smem + MlaSmem::MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;

    pdl_trigger();
    pdl_wait();

    int npos, Tc;
    if (a.count) {
        const int c = a.count[b];
        npos = c < 0 ? 0 : (c > a.k ? a.k : c);
        Tc = a.k;
    } else {
        npos = clamp_seq(a.seq_lens[b], a.T_cap, a.status);
        Tc = a.T_cap;
    }
    const int j0 = (int)((long long)split * a.row_tiles / a.splits);
    const int j1 = (int)((long long)(split + 1) * a.row_tiles / a.splits);
    const int jend = min(j1, (npos + kTok - 1) / kTok);
    const int ntile = max(0, jend - j0);

    if (tid == 0) {
        for (int i = 0; i < kKB + 3; ++i) mbar_init(&kfull[i], 1);
        fence_barrier_init();
        *flag = 0;
    }
    if (tid < kHC) {
        mref[tid] = -INFINITY;
        lsum[tid] = 0.f;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tptr)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tptr;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint64_t pol = policy_evict_first();

    auto load_tile = [&](int j) {
        const int row = b * Tc + j * kTok;
#pragma unroll 1
        for (int kb = 0; kb < kKB; ++kb) {
            mbar_arrive_expect_tx(&kfull[kb], (uint32_t)kKBlk);
            tma_load_2d(sK + (size_t)kb * kKBlk, &tmK, kb * 64, row, &kfull[kb], pol);
        }
    };
    if (tid == 0 && ntile > 0) {
        mbar_arrive_expect_tx(qfull, (uint32_t)(kKB * kQBlk));
#pragma unroll 1
        for (int kb = 0; kb < kKB; ++kb) tma_load_2d(sQ + (size_t)kb * kQBlk, &tmQ, kb * 64, b * kH + hh * kHC, qfull);
        load_tile(j0);
    }

    constexpr uint32_t idS = mma_idesc(128, kHC, 0, 0);  // A = K tile (K-major), B = Q half (K-major)
    constexpr uint32_t idO = mma_idesc(128, kHC, 1, 1);  // A = V^T (MN-major), B = P^T (MN-major)
    const uint32_t ka = smem_u32(sK), qa = smem_u32(sQ);
    const uint32_t pa = ka + 8u * kKBlk;                  // P^T in the rope block
    unsigned char *sP = sK + (size_t)8 * kKBlk;
    const int tr = warp * 32 + lane;                      // this thread's token row (S^T lane)
    bool ok = true;

    for (int it = 0; it < ntile && ok; ++it) {
        const int t0 = (j0 + it) * kTok;
        const uint32_t par = (uint32_t)it & 1u;
        // ---- S^T = K_tile Q_half^T, block by block as the blocks land ----------------
        if (tid == 0) {
            bool good = it > 0 || mbar_wait_bounded(qfull, 0u);
            for (int kb = 0; kb < kKB && good; ++kb) {
                good = mbar_wait_bounded(&kfull[kb], par);
                if (!good) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem, sw128_desc(ka + kb * kKBlk + kk * 32, 16, 1024),
                             sw128_desc(qa + kb * kQBlk + kk * 32, 16, 1024), idS, (kb > 0 || kk > 0) ? 1u : 0u);
            }
            if (good)
                mma_commit(sdone);
            else
                *flag = 1;
        }
        if (*flag == 0 && !mbar_wait_bounded(sdone, par)) *flag = 1;
        tc_fence_after();
        __syncthreads();
        if (*flag) {
            ok = false;
            break;
        }
        // ---- softmax over the tile's tokens, per head -------------------------------
        const bool valid = t0 + tr < npos;
        float s[64], t[64];
        {
            float v0[32], v1[32];
            tmem_ld32(lane_base + 0, v0);
            tmem_ld32(lane_base + 32, v1);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                s[j] = valid ? v0[j] * a.scale_log2 : -INFINITY;
                s[32 + j] = valid ? v1[j] * a.scale_log2 : -INFINITY;
            }
        }
#pragma unroll
        for (int j = 0; j < 64; ++j) t[j] = s[j];
        float c0, c1;
        col_reduce64<true>(t, lane, c0, c1);
        red[warp * 64 + 2 * lane] = c0;
        red[warp * 64 + 2 * lane + 1] = c1;
        __syncthreads();
        int need = 0;
        if (tid < kHC) {
            const float M = fmaxf(fmaxf(red[tid], red[64 + tid]), fmaxf(red[128 + tid], red[192 + tid]));
            const float mo = mref[tid];
            float cr = 1.f;
            if (mo == -INFINITY) {
                mref[tid] = M;  // first tile with a live token: nothing accumulated yet
            } else if (M > mo + kLazy) {
                mref[tid] = M;
                cr = exp2f(mo - M);
                need = 1;
            }
            corr[tid] = cr;
        }
        const int any_rescale = __syncthreads_or(need);
        // weights P = exp2(s - mref) (bf16) into the rope block, token row tr
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h0 = c * 8 + 2 * e;
                const float p0 = s[h0] == -INFINITY ? 0.f : exp2f(s[h0] - mref[h0]);
                const float p1 = s[h0 + 1] == -INFINITY ? 0.f : exp2f(s[h0 + 1] - mref[h0 + 1]);
                const __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
                t[h0] = __low2float(pk);
                t[h0 + 1] = __high2float(pk);
                w[e] = *reinterpret_cast<const uint32_t *>(&pk);
            }
            *reinterpret_cast<uint4 *>(sP + tr * 128 + ((c ^ (tr & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        // value rows of tokens past the range may hold anything, NaN included
        // (0 * NaN is NaN in the second product): zero them
        if (!valid) {
#pragma unroll 1
            for (int c = 0; c < 8 * 8; ++c)
                *reinterpret_cast<uint4 *>(sK + (size_t)(c >> 3) * kKBlk + tr * 128 + (c & 7) * 16) =
                    make_uint4(0, 0, 0, 0);
        }
        col_reduce64<false>(t, lane, c0, c1);
        red[warp * 64 + 2 * lane] = c0;
        red[warp * 64 + 2 * lane + 1] = c1;
        // rescale the accumulated O^T where a head's running max was raised
        if (any_rescale) {
#pragma unroll 1
            for (int blk = 0; blk < 4; ++blk)
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    const uint32_t addr = lane_base + kColO + blk * kHC + half * 32;
                    tmem_ld32(addr, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] *= corr[half * 32 + j];
                    tmem_st32(addr, v);
                }
        }
        __syncthreads();
        if (tid < kHC)
            lsum[tid] = lsum[tid] * corr[tid] + ((red[tid] + red[64 + tid]) + (red[128 + tid] + red[192 + tid]));
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- O^T += V^T P^T, then the next tile's blocks once it is done -------------
        if (tid == 0) {
#pragma unroll
            for (int blk = 0; blk < 4; ++blk)
#pragma unroll
                for (int kk = 0; kk < kTok / 16; ++kk)
                    mma_bf16(tmem + kColO + blk * kHC,
                             sw128_desc(ka + 2 * blk * kKBlk + kk * 2048, kKBlk, 1024),
                             sw128_desc(pa + kk * 2048, kKBlk, 1024), idO, (it > 0 || kk > 0) ? 1u : 0u);
            mma_commit(odone);
            if (it + 1 < ntile) {
                if (mbar_wait_bounded(odone, par)) {
                    tc_fence_after();
                    load_tile(j0 + it + 1);
                } else {
                    *flag = 1;
                }
            }
        }
    }
    // ---- epilogue: the last product done, O^T out (normalised or as a partial) ------
    if (ok && ntile > 0 && !mbar_wait_bounded(odone, (uint32_t)(ntile - 1) & 1u)) ok = false;
    tc_fence_after();
    __syncthreads();
    if (*flag) ok = false;
    if (!ok && tid == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_TIMEOUT);
    if (ok) {
        const int hbase = hh * kHC;
        const bool part = a.splits > 1;
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
            const int dv = blk * 128 + warp * 32 + lane;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float v[32];
                if (ntile > 0) {
                    tmem_ld32(lane_base + kColO + blk * kHC + half * 32, v);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = 0.f;
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int h = hbase + half * 32 + j;
                    if (part) {
                        a.part_o[(((size_t)b * a.splits + split) * kH + h) * kDv + dv] = __float2bfloat16_rn(v[j]);
                    } else {
                        const float l = lsum[half * 32 + j];
                        static_cast<__nv_bfloat16 *>(a.out)[((size_t)b * kH + h) * kDv + dv] =
                            __float2bfloat16_rn(l > 0.f ? v[j] / l : 0.f);
                    }
                }
            }
        }
        if (tid < kHC) {
            const int h = hbase + tid;
            const float m = mref[tid], l = lsum[tid];
            if (part) {
                float *pml = a.part_ml + (((size_t)b * a.splits + split) * kH + h) * 2;
                pml[0] = l > 0.f ? m : -INFINITY;
                pml[1] = l;
            } else if (a.lse) {
                a.lse[(size_t)b * kH + h] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
}

// rows x 576 bf16, boxes of 64 columns x box_rows rows
cudaError_t encode_rows(CUtensorMap *m, const void *base, long long rows, int box_rows) {
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    return encode_tiled_bf16(m, base, 2, dims, strides, box);
}

}  // namespace

cudaError_t plan_mla_range(int B, int row_len, MlaRangePlan *p) {
    if (!tensor_maps_available()) return cudaErrorNotSupported;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(mla_range_kernel), MlaSmem::TOTAL);
    if (e != cudaSuccess) return e;
    if (row_len < 1) row_len = 1;
    p->row_tiles = (row_len + kTok - 1) / kTok;
    int s = device_sm_count() / (2 * (B > 0 ? B : 1));
    if (s < 1) s = 1;
    if (s > p->row_tiles) s = p->row_tiles;
    p->splits = s;
    p->smem = MlaSmem::TOTAL;
    return cudaSuccess;
}

cudaError_t launch_mla_range(const MlaRangePlan &p, const MlaRangeArgs &a0, const void *K, cudaStream_t s, bool pdl) {
    MlaRangeArgs a = a0;
    a.row_tiles = p.row_tiles;
    a.splits = p.splits;
    const long long rows = (long long)a.B * (a.count ? a.k : a.T_cap);
    if (rows + kTok > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA row coordinates are int32
    CUtensorMap mk, mq;
    cudaError_t e = encode_rows(&mk, K, rows, kTok);
    if (e == cudaSuccess) e = encode_rows(&mq, a.q, (long long)a.B * kH, kHC);
    if (e != cudaSuccess) return e;
    e = launch_kernel(mla_range_kernel, dim3(p.splits, 2, a.B), dim3(kThr), p.smem, s, pdl, mk, mq, a);
    if (e != cudaSuccess || p.splits == 1) return e;
    MlaArgs c;
    memset(&c, 0, sizeof c);
    c.B = a.B;
    c.splits = p.splits;
    c.part_o = a.part_o;
    c.part_ml = a.part_ml;
    c.out = a.out;
    c.lse = a.lse;
    return launch_mla_combine(c, s, pdl);
}

}  // namespace jssa
