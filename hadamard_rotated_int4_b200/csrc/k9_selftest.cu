// k9_selftest.cu -- a self-test of the failure path every pipelined kernel of
// the library uses: an mbarrier wait bounded by global time that, when nothing
// ever arrives, gives up, records HBL_ERR_TIMEOUT in the caller's status word
// and returns, leaving the context usable.  The probe waits on a barrier that
// either receives its one arrival first (arrive != 0: the wait succeeds) or
// never does (arrive == 0: the wait runs out after limit_ns).
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k9 {

__global__ void bounded_wait_probe(int arrive, uint64_t limit_ns, int32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init_count(b, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (arrive) mbar_arrive_one(b);
        if (!mbar_wait_bounded<true>(b, 0, limit_ns)) report_status(status, HBL_ERR_TIMEOUT);
    }
}

}  // namespace k9

hbl_status launch_bounded_wait_probe(int arrive, int timeout_us, int32_t* status,
                                     cudaStream_t stream) {
    k9::bounded_wait_probe<<<1, 32, 0, stream>>>(arrive, (uint64_t)timeout_us * 1000ull, status);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

}  // namespace hbl
