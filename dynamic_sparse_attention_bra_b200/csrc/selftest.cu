// Self-test of the bounded-wait error path used by every kernel that waits
// on an mbarrier (the pages describe no such mechanism; it is this library's
// failure detection).  One CTA initialises an mbarrier that expects one
// arrival, never arrives on it, and polls it at most ``tries`` times with
// mbarrier.try_wait; when the limit runs out it records kDevTimeout in the
// status word exactly as the attention kernels do, and returns.  The GPU
// context stays usable and the host reads the code with bra_device_status.
#include "common.cuh"
#include "tc_ptx.cuh"

namespace bra {
namespace {

__global__ void bra_bounded_wait_selftest_kernel(int* status, uint32_t tries, int arrive) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    if (arrive) ptx::mbar_arrive(&bar);  // the control case: the wait succeeds at once
    for (uint32_t i = 0; i < tries; ++i)
        if (ptx::mbar_try_wait(&bar, 0)) return;
    raise_status(status, kDevTimeout);
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int* status, uint32_t tries, bool arrive, cudaStream_t stream) {
    bra_bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(status, tries, arrive ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace bra
