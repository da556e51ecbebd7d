// Indexed decode attention over a shared latent cache (multi-head latent
// attention), on the 5th-generation tensor cores.
//
// Method: news item "JSSA makes token-level sparse decoding gather-free",
// Perspective para 1 (for MLA models the selection runs over the shared latent
// cache); "Joint Subspace Sparse Attention for Efficient Long-Context
// Decoding", Abstract (token-level indexed attention).  One latent row of 576
// bf16 per token is both the key (all 576 dims) and the value (its first 512
// dims); all 128 query heads attend over the selected rows of their batch row.
//
// With 128 heads the per-token work is a dense contraction (~228 flop per
// byte of selected rows), so it runs as two tcgen05 matrix products per CTA:
//   S[128 heads x 128 tokens] = Q[128 x 576] . K_sel^T      (fp32 in TMEM)
//   O[128 x 512]             = softmax(S) (bf16) . V_sel     (fp32 in TMEM)
// A CTA takes one batch row and one split of up to 128 selected tokens.  The
// selected rows are gathered in place from the [B, T, 1, 576] cache with
// cp.async into nine 128-byte-swizzled K-major blocks (the same bytes serve as
// the MN-major V operand of the second product); Q streams through four
// swizzled 16 KiB buffers; P is written to shared memory in the A-operand
// layout.  TMEM holds S in columns 0..127, then O in columns 0..511.  Splits
// write (unnormalised O, row max, row sum), merged by log-sum-exp inside the
// kernel when all its CTAs fit on the GPU at once, else by a second kernel
// (mla_combine_kernel).  Sixteen warps: warp w reads TMEM lanes 32 (w mod 4) .. +31
// (its heads) and a quarter of the columns, w / 4, so that the softmax (32
// logits per thread) and the readout of O (128 columns per thread) are four
// short chains instead of one long one.
#include "jssa_common.cuh"
#include "jssa_internal.h"
#include "jssa_tc.cuh"

namespace jssa {

namespace {

constexpr int kD = 576, kDv = 512, kH = 128, kTok = 128, kThr = 512;
constexpr int kWG = kThr / 128;  // warpgroups: column quarters of S and O
constexpr int kKB = 9;          // 64-column blocks of a latent row
constexpr int kQBuf = 4;        // Q block buffers
constexpr int kBlk = 16384;     // one block: 128 rows x 128 bytes
constexpr size_t kSmemK = (size_t)kKB * kBlk;
constexpr size_t kSmemQ = (size_t)kQBuf * kBlk;
constexpr size_t kSmemMisc = 2048 + 2 * kWG * kH * 4;  // barriers, tokens; row max / sum per quarter
constexpr size_t kSmemBytes = kSmemK + kSmemQ + kSmemMisc;

template <int N>
__device__ __forceinline__ void cp_wait_dyn(int n) {
    if (n >= N) {
        cp_async_wait<N>();
    } else if constexpr (N > 0) {
        cp_wait_dyn<N - 1>(n);
    }
}

// The log-sum-exp merge of heads [h0, h1) of batch row b over the splits'
// partials: one 8-column chunk of one head per thread and pass; the splits
// are read sixteen at a time, every (max, sum) pair and partial of a group in
// flight at once, and merged online (the running sums rescaled when a group
// raises the maximum).
__device__ void merge_heads(const MlaArgs &a, int b, int h0, int h1, int tid, int nthr) {
    constexpr int GS = 16;
    const int ns = a.splits;
    const int items = (h1 - h0) * (kDv / 8);
    for (int it = tid; it < items; it += nthr) {
        const int h = h0 + it / (kDv / 8), c0 = (it % (kDv / 8)) * 8;
        const float2 *pml = reinterpret_cast<const float2 *>(a.part_ml) + (size_t)b * ns * kH + h;
        const __nv_bfloat16 *pbase = a.part_o + ((size_t)b * ns * kH + h) * kDv + c0;
        float M = -INFINITY, L = 0.f, o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = 0.f;
        for (int s0 = 0; s0 < ns; s0 += GS) {
            float2 ml[GS];
            uint4 v[GS];
#pragma unroll
            for (int u = 0; u < GS; ++u) {
                const bool in = s0 + u < ns;
                ml[u] = in ? __ldcg(pml + (size_t)(s0 + u) * kH) : make_float2(-INFINITY, 0.f);
                v[u] = in ? __ldcg(reinterpret_cast<const uint4 *>(pbase + (size_t)(s0 + u) * kH * kDv))
                          : make_uint4(0u, 0u, 0u, 0u);
            }
            float mg = M;
#pragma unroll
            for (int u = 0; u < GS; ++u) mg = fmaxf(mg, ml[u].x);
            if (mg == -INFINITY) continue;  // nothing live so far
            const float r = exp2f(M - mg);  // 0 while M is -inf
            L *= r;
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] *= r;
            M = mg;
#pragma unroll
            for (int u = 0; u < GS; ++u) {
                if (ml[u].x == -INFINITY) continue;  // an empty split (or past the last)
                const float w = exp2f(ml[u].x - M);
                L = fmaf(ml[u].y, w, L);
                float f[8];
                Vec16<__nv_bfloat16>::unpack(v[u], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = fmaf(f[e], w, o[e]);
            }
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 pk = __floats2bfloat162_rn(o[2 * e] * inv, o[2 * e + 1] * inv);
            w4[e] = *reinterpret_cast<const uint32_t *>(&pk);
        }
        *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + ((size_t)b * kH + h) * kDv + c0) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
        if (a.lse && c0 == 0) a.lse[(size_t)b * kH + h] = L > 0.f ? (M + log2f(L)) * 0.693147180559945309417f : -INFINITY;
    }
}

template <bool INDEXED>
__global__ void __launch_bounds__(kThr, 1) mla_kernel(MlaArgs a) {
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *sK = smem;
    unsigned char *sQ = smem + kSmemK;
    unsigned char *sP = sQ;  // P reuses Q buffers 0-1 once S is complete
    uint64_t *qfree = reinterpret_cast<uint64_t *>(smem + kSmemK + kSmemQ);  // [kQBuf]
    uint64_t *sdone = qfree + kQBuf;
    uint64_t *odone = qfree + kQBuf + 1;
    uint32_t *tptr = reinterpret_cast<uint32_t *>(qfree + kQBuf + 2);
    int *flag = reinterpret_cast<int *>(tptr + 1);
    int *tok = reinterpret_cast<int *>(qfree + 8);  // [kTok]
    float *red_m = reinterpret_cast<float *>(smem + kSmemK + kSmemQ + 2048);  // [kWG][kH]
    float *red_l = red_m + kWG * kH;                                          // [kWG][kH]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, b = blockIdx.y;

    pdl_trigger();
    pdl_wait();

    const int Tb = clamp_seq(a.seq_lens[b], a.T_cap, a.status);
    int npos;
    if (INDEXED) {
        if (a.count) {
            npos = a.count[b];
            if (npos < 0 || npos > a.k) {
                if (tid == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_INDEX);
                npos = npos < 0 ? 0 : a.k;
            }
        } else {
            npos = 0;
            const int32_t *lst = a.idx + (size_t)b * a.k;
            for (int j0 = 0; j0 < a.k; j0 += kThr) npos += __syncthreads_count(j0 + tid < a.k && lst[j0 + tid] >= 0);
        }
    } else {
        npos = Tb;
    }
    const int p0 = split * kTok;
    const int rows = max(0, min(kTok, npos - p0));

    if (tid == 0) {
        for (int i = 0; i < kQBuf + 2; ++i) mbar_init(&qfree[i], 1);
        fence_barrier_init();
        *flag = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tptr)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    if (tid < kTok) {
        int t = -1;
        if (tid < rows) {
            t = INDEXED ? __ldg(a.idx + (size_t)b * a.k + p0 + tid) : p0 + tid;
            if (t < 0 || t >= Tb) {
                if (a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_INDEX);
                t = -1;
            }
        }
        tok[tid] = t;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tptr;

    // ---- loads: selected latent rows (9 blocks) and Q blocks 0..3 --------------
    const char *Kg = static_cast<const char *>(a.K);
    const char *Qg = static_cast<const char *>(a.q) + (size_t)b * kH * kD * 2;
    auto load_k_block = [&](int kb) {
        for (int c = tid; c < kTok * 8; c += kThr) {
            const int j = c >> 3, ch = c & 7;
            const int t = tok[j];
            unsigned char *dst = sK + (size_t)kb * kBlk + j * 128 + ((ch ^ (j & 7)) << 4);
            if (t >= 0)
                cp_async16(dst, Kg + ((size_t)b * a.T_cap + t) * (kD * 2) + kb * 128 + ch * 16, 16);
            else
                cp_async16(dst, Kg, 0);
        }
    };
    auto load_q_block = [&](int kb, int buf) {
        for (int c = tid; c < kH * 8; c += kThr) {
            const int hh = c >> 3, ch = c & 7;
            cp_async16(sQ + (size_t)buf * kBlk + hh * 128 + ((ch ^ (hh & 7)) << 4), Qg + (size_t)hh * (kD * 2) + kb * 128 + ch * 16,
                       16);
        }
    };
    for (int g = 0; g < kQBuf; ++g) {
        load_k_block(g);
        load_q_block(g, g);
        cp_async_commit();
    }
    for (int kb = kQBuf; kb < kKB; ++kb) load_k_block(kb);
    cp_async_commit();

    // ---- S = Q K^T over the nine 64-column blocks -------------------------------
    constexpr uint32_t idS = mma_idesc(128, kTok, 0, 0);
    bool ok = true;
    // Commit groups: G0..G3 = K block g + Q block g, G4 = K blocks 4..8, then
    // R_j = Q block j + 4 (j = 0..4), committed in iteration j + 1 once the
    // products of iteration j, which read its buffer, are done: by then they
    // have had a whole iteration to finish, so the wait rarely stalls.
    for (int kb = 0; kb < kKB; ++kb) {
        // groups committed after the one holding block kb when this iteration starts
        const int after = kb < kQBuf ? (kQBuf - kb) + max(0, kb - 1) : min(kQBuf, kb - 2) - kb + kQBuf;
        cp_wait_dyn<kQBuf>(after);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0 && ok) {
            const uint32_t qa = smem_u32(sQ + (size_t)(kb % kQBuf) * kBlk), ka = smem_u32(sK + (size_t)kb * kBlk);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem, sw128_desc(qa + kk * 32, 16, 1024), sw128_desc(ka + kk * 32, 16, 1024), idS,
                         (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&qfree[kb % kQBuf]);
        }
        const int jr = kb - 1;  // refill the buffer of the previous iteration's block
        if (jr >= 0 && jr + kQBuf < kKB) {
            if (ok && !mbar_wait_bounded(&qfree[jr % kQBuf], (uint32_t)(jr / kQBuf) & 1u)) atomicOr(flag, 1);
            fence_async_smem();
            if (*flag == 0) load_q_block(jr + kQBuf, jr % kQBuf);
            cp_async_commit();
        }
        __syncthreads();
        ok = *flag == 0;
    }
    if (tid == 0 && ok) mma_commit(sdone);
    if (ok && !mbar_wait_bounded(sdone, 0u)) atomicOr(flag, 1);
    tc_fence_after();
    __syncthreads();
    ok = *flag == 0;

    // ---- softmax over the tile's tokens: head = TMEM lane, 32 columns per warp --
    const int q4 = warp & 3, cg = warp >> 2;  // lane quarter (heads), column quarter
    const int h = q4 * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
    float m = -INFINITY, l = 0.f;
    if (ok) {
        // this quarter's live columns as a bit mask (the same in every warp),
        // and the head's 32 logits of the quarter read from TMEM once
        const int col = cg * 32 + lane;
        const unsigned live = __ballot_sync(0xffffffffu, col < rows && tok[col] >= 0);
        float v[32];
        tmem_ld32(lane_base + cg * 32, v);
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if ((live >> j) & 1u) mx = fmaxf(mx, v[j]);
        red_m[cg * kH + h] = mx;
        __syncthreads();
#pragma unroll
        for (int g = 0; g < kWG; ++g) mx = fmaxf(mx, red_m[g * kH + h]);
        m = mx == -INFINITY ? -INFINITY : mx * a.scale_log2;
        float lp = 0.f;
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = g8 * 8 + e * 2;
                const float p0 = ((live >> j) & 1u) ? exp2f(v[j] * a.scale_log2 - m) : 0.f;
                const float p1 = ((live >> (j + 1)) & 1u) ? exp2f(v[j + 1] * a.scale_log2 - m) : 0.f;
                lp += p0;
                lp += p1;
                const __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
                w[e] = *reinterpret_cast<const uint32_t *>(&pk);
            }
            const int c8 = cg * 32 + g8 * 8, col8 = c8 & 63, blk = c8 >> 6;
            *reinterpret_cast<uint4 *>(sP + (size_t)blk * kBlk + h * 128 + (((col8 >> 3) ^ (h & 7)) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        red_l[cg * kH + h] = lp;
    } else {
        __syncthreads();  // the exchange barrier of the branch above
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (ok) {
        // the row sum in quarter order (every warp of the head adds the same way)
#pragma unroll
        for (int g = 0; g < kWG; ++g) l += red_l[g * kH + h];
    }

    // ---- O = P V: V is the first 512 columns of the same rows (MN-major) --------
    constexpr uint32_t idO = mma_idesc(128, 256, 0, 1);
    if (tid == 0 && ok) {
        const uint32_t pa = smem_u32(sP), ka = smem_u32(sK);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int kk = 0; kk < kTok / 16; ++kk)
                mma_bf16(tmem + half * 256, sw128_desc(pa + (kk >> 2) * kBlk + (kk & 3) * 32, 16, 1024),
                         sw128_desc(ka + half * 4 * kBlk + kk * 2048, kBlk, 1024), idO, kk > 0 ? 1u : 0u);
        }
        mma_commit(odone);
    }
    if (ok && !mbar_wait_bounded(odone, 0u)) atomicOr(flag, 1);
    tc_fence_after();
    __syncthreads();
    ok = *flag == 0;
    if (!ok && tid == 0 && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_TIMEOUT);

    // ---- epilogue: this warp's heads, columns [128 cg, 128 cg + 128) of O ----------
    if (ok) {
        const int cb = cg * (kDv / kWG);
        if (a.splits == 1) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(a.out) + ((size_t)b * kH + h) * kDv;
#pragma unroll 1
            for (int c0 = cb; c0 < cb + kDv / kWG; c0 += 32) {
                float v[32];
                tmem_ld32(lane_base + c0, v);
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 pk = __floats2bfloat162_rn(v[j + 2 * e] * inv, v[j + 2 * e + 1] * inv);
                        w[e] = *reinterpret_cast<const uint32_t *>(&pk);
                    }
                    *reinterpret_cast<uint4 *>(orow + c0 + j) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            if (a.lse && cg == 0)
                a.lse[(size_t)b * kH + h] = l > 0.f ? (m + log2f(l)) * 0.693147180559945309417f : -INFINITY;
        } else {
            // unnormalised partial O in bf16: each thread converts its head's 128
            // columns into a shared-memory row (the K blocks are free once the
            // second product is done; a 1040-byte row stride keeps the 16-byte
            // stores of a warp on distinct banks) and copies its 256-byte segment
            // to the partial with one bulk copy
            constexpr int kRowS = kDv * 2 + 16;
            unsigned char *srow = sK + (size_t)h * kRowS + (size_t)cb * 2;
#pragma unroll 1
            for (int c0 = 0; c0 < kDv / kWG; c0 += 32) {
                float v[32];
                tmem_ld32(lane_base + cb + c0, v);
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 pk = __floats2bfloat162_rn(v[j + 2 * e], v[j + 2 * e + 1]);
                        w[e] = *reinterpret_cast<const uint32_t *>(&pk);
                    }
                    *reinterpret_cast<uint4 *>(srow + (size_t)(c0 + j) * 2) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_async_smem();
            __nv_bfloat16 *po = a.part_o + (((size_t)b * a.splits + split) * kH + h) * kDv + cb;
            bulk_s2g(po, srow, (uint32_t)(kDv / kWG) * 2);
            bulk_wait_all();  // the segment is in global memory before the split is published,
            asm volatile("fence.proxy.async.global;" ::: "memory");  // and ordered before the arrival
            if (cg == 0) {
                float *pml = a.part_ml + (((size_t)b * a.splits + split) * kH + h) * 2;
                pml[0] = m;
                pml[1] = l;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    if (a.splits > 1 && a.inline_combine) {
        // In-kernel merge (every CTA of the grid is resident at once, which
        // the launch checks): each split publishes its partial (stores, then a
        // fence and an arrival), waits for the other splits of its batch row,
        // and merges its share of the heads.  The last CTA to finish resets
        // the two counters for the next call.  A wait that runs out sets the
        // timeout status and skips the merge.
        if (tid == 0) {
            __threadfence();
            atomicAdd(a.ctr + b, 1u);
            const bool all = flag_wait_bounded(a.ctr + b, (unsigned)a.splits);
            __threadfence();
            *flag = all ? 0 : 1;
            if (!all && a.status) atomicOr(a.status, (uint32_t)JSSA_DEV_TIMEOUT);
        }
        __syncthreads();
        if (*flag == 0) {
            const int hps = (kH + a.splits - 1) / a.splits;
            const int h0 = min(kH, split * hps), h1 = min(kH, h0 + hps);
            merge_heads(a, b, h0, h1, tid, kThr);
        }
        __syncthreads();
        if (tid == 0 && atomicAdd(a.ctr + a.B + b, 1u) == (unsigned)(a.splits - 1)) {
            a.ctr[b] = 0u;
            a.ctr[a.B + b] = 0u;
        }
    }
}

// Log-sum-exp merge of the splits: CTA (b, 4 heads), 16 output dims per thread.
// The splits' maxima are read first; the partial rows and (max, sum) pairs
// are then read four splits at a time with all their loads in flight.
__global__ void __launch_bounds__(128) mla_combine_kernel(MlaArgs a) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x, h = blockIdx.y * 4 + (threadIdx.x >> 5), c0 = (threadIdx.x & 31) * 16;
    const int ns = a.splits;
    const float2 *pml = reinterpret_cast<const float2 *>(a.part_ml) + (size_t)b * ns * kH + h;
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, pml[(size_t)s * kH].x);
    float L = 0.f, o[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j] = 0.f;
    const __nv_bfloat16 *pbase = a.part_o + ((size_t)b * ns * kH + h) * kDv + c0;
    for (int s0 = 0; s0 < ns; s0 += 8) {
        float2 ml[8];
        uint4 v[8][2];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const bool in = s0 + u < ns;
            ml[u] = in ? pml[(size_t)(s0 + u) * kH] : make_float2(-INFINITY, 0.f);
#pragma unroll
            for (int qd = 0; qd < 2; ++qd)
                v[u][qd] = in ? reinterpret_cast<const uint4 *>(pbase + (size_t)(s0 + u) * kH * kDv)[qd]
                              : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (ml[u].x == -INFINITY) continue;  // an empty split (or past the last)
            const float w = exp2f(ml[u].x - M);
            L = fmaf(ml[u].y, w, L);
#pragma unroll
            for (int qd = 0; qd < 2; ++qd) {
                float f[8];
                Vec16<__nv_bfloat16>::unpack(v[u][qd], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[8 * qd + e] = fmaf(f[e], w, o[8 * qd + e]);
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(a.out) + ((size_t)b * kH + h) * kDv + c0;
    uint32_t w[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const __nv_bfloat162 pk = __floats2bfloat162_rn(o[2 * e] * inv, o[2 * e + 1] * inv);
        w[e] = *reinterpret_cast<const uint32_t *>(&pk);
    }
    reinterpret_cast<uint4 *>(orow)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4 *>(orow)[1] = make_uint4(w[4], w[5], w[6], w[7]);
    if (a.lse && (threadIdx.x & 31) == 0)
        a.lse[(size_t)b * kH + h] = L > 0.f ? (M + log2f(L)) * 0.693147180559945309417f : -INFINITY;
}

}  // namespace

int mla_splits(int npos) { return npos <= kTok ? 1 : (npos + kTok - 1) / kTok; }

bool mla_inline_combine(int splits, int B) { return splits > 1 && (long long)splits * B <= device_sm_count(); }

cudaError_t launch_mla(const MlaArgs &a0, bool indexed, cudaStream_t s, bool pdl) {
    MlaArgs a = a0;
    void (*k)(MlaArgs) = indexed ? mla_kernel<true> : mla_kernel<false>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(k), kSmemBytes);
    if (e != cudaSuccess) return e;
    // the splits merge inside the kernel when every CTA fits on the GPU at
    // once (one CTA per SM: its shared memory); else a second kernel merges
    a.inline_combine = a.ctr && mla_inline_combine(a.splits, a.B);
    e = launch_kernel(k, dim3(a.splits, a.B), dim3(kThr), kSmemBytes, s, pdl, a);
    if (e != cudaSuccess || a.splits == 1 || a.inline_combine) return e;
    return launch_mla_combine(a, s, pdl);
}

cudaError_t launch_mla_combine(const MlaArgs &a, cudaStream_t s, bool pdl) {
    return launch_kernel(mla_combine_kernel, dim3(a.B, kH / 4), dim3(128), 0, s, pdl, a);
}

}  // namespace jssa
