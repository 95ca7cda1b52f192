// selftest.cu -- exercises the bounded waits that every kernel of the library
// relies on, on a wait that can never complete, so that the timeout path is
// tested on the GPU without hanging or faulting it: the kernel gives up after
// a short budget, records MIMI_DEV_ERR_TIMEOUT in the handle's error word and
// returns, and the host reads MIMI_RVQ_ETIMEOUT from mimi_rvq_get_error.
#include "handle.cuh"
#include "ptx.cuh"

namespace mimi {
namespace {

// ~50 ms at 2 GHz: long enough to be a real wait, short for a test.
constexpr long long kSelftestBudget = 100000000LL;

__global__ void k_wait_selftest(int which, unsigned* counter, int* err) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort;
    if (which == 0) {
        // an mbarrier phase that nothing completes (no arrival, no transaction)
        if (threadIdx.x == 0) {
            mbar_init(&bar, 1);
            abort = 0;
            fence_mbar_init();
        }
        __syncthreads();
        if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort, err, kSelftestBudget);
        __syncthreads();
    } else {
        // a group barrier of two members where only this CTA ever arrives
        group_arrive(counter);
        group_wait(counter, 2u, err, kSelftestBudget);
    }
}

}  // namespace

cudaError_t launch_wait_selftest(const Tables& t, int which, cudaStream_t s) {
    // the last group barrier, which no launch of the wide encoder uses (it has at
    // most kWideMaxFrames / 64 groups); mimi_rvq_get_error resets every barrier
    // after a timeout
    unsigned* counter = t.wide_bars + (kWideMaxGroups - 1) * kWideBarStride;
    k_wait_selftest<<<1, 32, 0, s>>>(which, counter, t.err);
    return cudaGetLastError();
}

}  // namespace mimi
