// Self-test of the bounded waits every kernel relies on (no counterpart in the source pages): a wait
// whose condition nothing ever satisfies must give up after its limit, record Q4_ERR_TIMEOUT in the
// caller's status word and return, leaving the context usable.  Nothing faults, traps or hangs.
#include "tc_ptx.cuh"

namespace {

// which = 0: an mbarrier phase that no thread completes; 1: a progress counter that no thread raises
// (the weak-load polling the MMA issuers use).
__global__ void selftest_wait_kernel(int which, uint64_t limit_ns, int32_t* status)
{
    __shared__ uint64_t bar;
    __shared__ uint32_t counter;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
        counter = 0;
        abort_flag = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (which == 0) tc::mbar_wait(&bar, 0, status, &abort_flag, limit_ns);
        else tc::poll_counters_slow(&counter, 1, 1u, status, &abort_flag, limit_ns);
    }
}

}  // namespace

extern "C" int q4_selftest_bounded_wait(int32_t which, int32_t limit_us, int32_t* dev_status, void* stream)
{
    if (!dev_status) return Q4_ERR_NULL;
    if ((which != 0 && which != 1) || limit_us < 1 || limit_us > 1000000) return Q4_ERR_SHAPE;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(which, (uint64_t)limit_us * 1000ull, dev_status);
    return q4_launch_status();
}
