// probe.cu -- a kernel whose only job is to run the library's bounded
// mbarrier wait to its limit, so that the timeout path (the status bit, the
// early return) can be observed without any real wait going wrong.
//
// One CTA of one warp initialises an mbarrier that expects one arrival and
// never arrives on it; every lane then waits on its first phase through the
// same mbar_wait_for the kernels use, with a caller-chosen limit.  The wait
// gives up, ORs DUO_DEV_WAIT_TIMEOUT into the status word and returns; no
// copy, MMA or tensor memory is ever in flight, so the kernel ends cleanly.
#include "common.cuh"
#include "internal.h"

namespace duo {
namespace {

__global__ void wait_probe_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    mbar_wait_for(&bar, 0, threadIdx.x == 0 ? status : nullptr, limit_ns);
    __syncwarp();
}

}  // namespace

cudaError_t launch_wait_probe(int32_t* status, uint64_t limit_ns, cudaStream_t s) {
    wait_probe_kernel<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace duo
