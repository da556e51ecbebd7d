// Shared device helpers of libjssa: element access, order-preserving score
// keys, block scans, and thin wrappers over the sm_90+/sm_100 PTX used by the
// kernels (mbarrier, bulk async copy, cp.async, programmatic dependent launch).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/jssa.h"

namespace jssa {

// ------------------------------------------------------------- elements ---
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 16 bytes -> 8 bf16 values (bf16) or 4 fp32 values (float).
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4 &v, float *f) {
        f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
        f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
        f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
        f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
    }
};
template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4 &v, float *f) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
};

__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void store_elem(float *p, float v) { *p = v; }

// Order-preserving map fp32 -> uint32 (larger score = larger key); -0.0 and
// +0.0 map to one key.  Finite inputs are a precondition.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Key of a token that is always selected (forced sink / recent tokens): above
// the key of every finite score, so a top-k by (key desc, index asc) takes
// forced tokens first, smallest indices first.
constexpr uint32_t kForcedKey = 0xffffffffu;
__device__ __forceinline__ uint32_t forced_key(uint32_t key, int t, int Tb, int n_sink, int n_recent) {
    return (t < n_sink || t >= Tb - n_recent) ? kForcedKey : key;
}

__device__ __forceinline__ int clamp_seq(int v, int cap, uint32_t *status) {
    if (v < 0 || v > cap) {
        if (status) atomicOr(status, (uint32_t)JSSA_DEV_SEQLEN);
        v = v < 0 ? 0 : cap;
    }
    return v;
}

// ---------------------------------------------------------------- scans ---
// Exclusive scan over a block of NT threads (NT a multiple of 32).  `tmp`
// holds >= NT/32 ints of shared memory.  Contains two __syncthreads().
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int *tmp, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    int pre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        int t = tmp[w];
        pre += (w < warp) ? t : 0;
        tot += t;
    }
    __syncthreads();
    total = tot;
    return pre + x - v;
}

// ------------------------------------------------------------------ PTX ---
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Programmatic dependent launch: wait for the preceding grid (and its memory)
// / allow the next grid in the stream to start launching.  Both are no-ops
// for a launch without the programmatic-serialisation attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}
// Non-blocking test of an mbarrier phase (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}
// try_wait that lets the hardware park the thread for up to `ns` nanoseconds
// while the phase is incomplete (a parked warp issues nothing).
__device__ __forceinline__ bool mbar_try_wait_for(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0u;
}
__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wall-time limit of every bounded on-chip wait in the library.  Normal
// waits last microseconds; a wait that reaches the limit gives up, the
// kernel records JSSA_DEV_TIMEOUT and returns.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Bounded wait on an mbarrier phase: gives up after limit_ns of wall time (or
// 2^28 polls), returning false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0; it < (1u << 28); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u && global_timer_ns() - t0 > limit_ns) return false;
    }
    return false;
}

// Bounded wait until a device word (written by other CTAs) reaches `target`:
// false after limit_ns of wall time.
__device__ __forceinline__ bool flag_wait_bounded(const volatile unsigned *word, unsigned target,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    const uint64_t t0 = global_timer_ns();
    while (*word < target) {
        if (global_timer_ns() - t0 > limit_ns) return false;
        __nanosleep(64);
    }
    return true;
}

// Suspend-time hint of the waits below (ns; 0 = the hardware's own limit).
constexpr uint32_t kParkNs = 20000;

// Bounded mbarrier wait that also gives up when another role of the CTA
// raised the abort flag.  Each poll is a try_wait, which may suspend the
// thread in hardware until the phase completes (or a time limit passes), so
// waiting warps take few issue slots from the working ones.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                              uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0; it < (1u << 28); ++it) {
        if (kParkNs ? mbar_try_wait_for(bar, parity, kParkNs) : mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 15u) == 15u && global_timer_ns() - t0 > limit_ns) return false;
    }
    return false;
}

// Bulk async copy global -> this CTA's shared memory, completing on `bar`
// (bytes and both addresses multiples of 16).  The L2 hint marks the
// streamed source as evict-first.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// cp.async 16 bytes (L2 only); src_bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace jssa
