// Failure-detection self-check: the library's bounded on-chip waits, run on
// a barrier and a flag that nothing completes, must give up after their
// limit, record JSSA_DEV_TIMEOUT in the status word and let the kernel return
// normally (no trap, no hang), leaving the context usable.  The method pages
// have no counterpart.
#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace jssa {

namespace {

// One CTA of 64 threads.  Warp 0 waits on an mbarrier phase that never
// completes (initialised for one arrival that nobody makes), with the plain
// bounded wait and with the abort-aware wait; warp 1 waits for a device word
// that nothing raises.  Each give-up sets JSSA_DEV_TIMEOUT; `seen` counts
// them (three when every wait expired).
__global__ void __launch_bounds__(64) wait_expiry_kernel(uint32_t *status, unsigned *word, unsigned *seen,
                                                         uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        abort_flag = 0;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0 && lane == 0) {
        if (!mbar_wait_bounded(&bar, 0u, limit_ns)) {
            atomicOr(status, (uint32_t)JSSA_DEV_TIMEOUT);
            atomicAdd(seen, 1u);
        }
        if (!wait_or_abort(&bar, 0u, &abort_flag, limit_ns)) {
            atomicOr(status, (uint32_t)JSSA_DEV_TIMEOUT);
            atomicAdd(seen, 1u);
        }
    } else if (warp == 1 && lane == 0) {
        if (!flag_wait_bounded(word, 1u, limit_ns)) {
            atomicOr(status, (uint32_t)JSSA_DEV_TIMEOUT);
            atomicAdd(seen, 1u);
        }
    }
    __syncthreads();
    // the barrier's phase is still pending: nothing is in flight on it, so
    // the CTA may exit
}

}  // namespace

cudaError_t launch_wait_expiry(void *ws, uint64_t limit_ns, cudaStream_t s) {
    uint32_t *status = static_cast<uint32_t *>(ws);
    unsigned *word = reinterpret_cast<unsigned *>(static_cast<char *>(ws) + 64);
    unsigned *seen = reinterpret_cast<unsigned *>(static_cast<char *>(ws) + 128);
    wait_expiry_kernel<<<1, 64, 0, s>>>(status, word, seen, limit_ns);
    return cudaGetLastError();
}

}  // namespace jssa
