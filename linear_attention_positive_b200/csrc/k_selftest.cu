// Self-test of the bounded-wait path every kernel of this library relies on.
//
// One CTA allocates tensor memory, initialises an mbarrier that nothing ever arrives on and waits
// on it through the library's own bounded wait (mbar_wait_for) with a short limit. The wait gives
// up, records FAVOR_ERR_TIMEOUT in the device status word and raises the CTA's abort flag; the
// other warps see the flag, the TMEM is freed and the kernel returns. No copy or MMA is in flight,
// so the exit is clean and the context stays usable: favor_sync_status then reports the timeout.

#include "common.cuh"

namespace favor {

__global__ void __launch_bounds__(128) k_wait_selftest(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    volatile int *abort = &abort_flag;
    if (warp == 1) {
        // the phase of parity 0 never completes: nobody arrives
        mbar_wait_for(&bar, 0, abort, limit_ns);
    } else {
        // the other warps poll the abort flag with the same bound, as a consumer warp would
        const unsigned long long t0 = globaltimer_ns();
        while (!*abort && globaltimer_ns() - t0 < 4 * limit_ns + 1000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem_slot, 32);
}

cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t st) {
    k_wait_selftest<<<1, 128, 0, st>>>(limit_ns);
    return cudaGetLastError();
}

}  // namespace favor
