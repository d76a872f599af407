// Failure-detection self-test of the bounded mbarrier wait that the pipelined kernels use
// (ptx::mbar_wait): one CTA with a producer thread and a consumer thread.  The producer
// arrives on `full` unless the host asks it to skip; the consumer waits on `full` and then
// arrives on `done`, which the producer waits for.  When the arrival is skipped the
// consumer's wait gives up after kPolls polls.  It records CSA2_ERR_TIMEOUT in the device
// error word and raises the CTA's abort flag, the producer's wait sees the flag, and both
// return.  Every wait is bounded and nothing traps, so the context stays usable.
#include "tc_ptx.cuh"

namespace csa2 {
namespace stest {

constexpr uint32_t kPolls = 1u << 10;   // far below the back-off threshold: the test ends quickly

__global__ void __launch_bounds__(64, 1) bounded_wait_kernel(int skip_arrival) {
    __shared__ __align__(8) uint64_t full, done;
    __shared__ volatile int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&full, 1);
        ptx::mbar_init(&done, 1);
        abort_flag = 0;
        ptx::fence_async_smem();
    }
    __syncthreads();
    if (threadIdx.x == 0) {                         // producer
        if (!skip_arrival) ptx::mbar_arrive(&full);
        ptx::mbar_wait<kPolls>(&done, 0, &abort_flag);
    } else if (threadIdx.x == 32) {                 // consumer
        if (ptx::mbar_wait<kPolls>(&full, 0, &abort_flag)) ptx::mbar_arrive(&done);
    }
}

}  // namespace stest

cudaError_t launch_selftest_bounded_wait(int skip_arrival, cudaStream_t st) {
    stest::bounded_wait_kernel<<<1, 64, 0, st>>>(skip_arrival);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace csa2
