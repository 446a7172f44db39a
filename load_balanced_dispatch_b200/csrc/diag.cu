// diag.cu -- a self-test of the bounded waits that every pipeline of the library uses.
//
// The FFN's second-GEMM tiles wait for counters that other CTAs raise (ptx::wait_count_geq),
// and its ring stages wait on mbarriers with the same clock bound. None of them can be made to
// run out by a caller's arguments, so this kernel waits with the same helper on a counter that
// the caller leaves at 0: after `limit` SM clock cycles it gives up, records the pipeline
// timeout in the device error word, and returns. Nothing faults or hangs; moe_sync_status then
// reports the timeout and the context stays usable.
#include "tc_ptx.cuh"

namespace moe {

__global__ void selftest_wait_kernel(const int32_t* __restrict__ flag, long long limit) {
    if (threadIdx.x == 0) (void)ptx::wait_count_geq(flag, 1, nullptr, limit);
}

cudaError_t launch_selftest_wait(const int32_t* flag, int64_t limit_cycles, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 32, 0, stream>>>(flag, (long long)limit_cycles);
    return cudaGetLastError();
}

}  // namespace moe
