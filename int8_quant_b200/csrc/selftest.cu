// selftest.cu — ssd_selftest_bounded_wait: runs the bounded mbarrier wait and the
// CTA abort flag that the warp-specialised kernels rely on, on a wait that can never
// be satisfied, so that the timeout path is tested without faulting or hanging a GPU.
//
// One CTA of two warps.  Each warp waits on its own mbarrier, on which nothing ever
// arrives: warp 0 with the caller's limit, warp 1 with the kernels' full limit
// (tc::kWaitLimit, about two seconds).  Warp 0's wait expires, raises the abort flag
// and records SSD_ERR_TIMEOUT in the status word; warp 1 has to notice the flag and
// give up early instead of waiting out its own limit.  Each warp's lane 0 writes the
// cycles it spent waiting, so a caller can check both halves.
#include "../../include/ssd.h"
#include "kernels.h"
#include "tc.cuh"

namespace ssd {
namespace {

__global__ void bounded_wait_kernel(long long limit, int* status, unsigned long long* cycles) {
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bars[0], 1);
        tc::mbar_init(&bars[1], 1);
        abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    volatile int* flag = &abort_flag;
    const long long t0 = clock64();
    if (warp == 0) tc::wait_or_abort(&bars[0], 0, flag, status, kStatusTimeout, limit);
    else tc::wait_or_abort(&bars[1], 0, flag, status, kStatusTimeout);
    const long long t1 = clock64();
    if (lane == 0) cycles[warp] = (unsigned long long)(t1 - t0);
}

}  // namespace
}  // namespace ssd

extern "C" ssd_status ssd_selftest_bounded_wait(long long limit_cycles, int* status,
                                                unsigned long long* cycles, cudaStream_t stream) {
    if (!status || !cycles || limit_cycles <= 0 || limit_cycles > ssd::tc::kWaitLimit) return SSD_ERR_INVALID_ARG;
    if (cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return ssd::from_cuda(cudaGetLastError());
    ssd::bounded_wait_kernel<<<1, 64, 0, stream>>>(limit_cycles, status, cycles);
    return ssd::from_cuda(cudaGetLastError());
}
