// Test hook for the library's failure detection: one CTA waits, with the same bounded mbarrier wait every
// kernel uses, on a barrier that nothing arrives at (unless asked to arrive first), so the wait runs out
// and the kernel records it in a device error word exactly as a kernel whose copy never landed would.
// The barrier is fed by no bulk copy and no tensor-core operation, so nothing is in flight when the CTA
// leaves; the context stays usable.
#include "internal.h"
#include "tma.cuh"

namespace hils {

namespace {

__device__ unsigned int g_wait_expiry_errors = 0;

__global__ void wait_expiry_kernel(uint32_t max_polls, int arrive_first) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (arrive_first) mbar_arrive(&bar);
        if (!mbar_wait_polls(&bar, 0, max_polls)) atomicOr(&g_wait_expiry_errors, 1u);
    }
}

}  // namespace

unsigned int wait_expiry_error_flags(bool clear) {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_wait_expiry_errors, sizeof(v));
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_wait_expiry_errors, &zero, sizeof(zero));
    }
    return v;
}

cudaError_t launch_wait_expiry(uint32_t max_polls, int arrive_first, cudaStream_t stream) {
    wait_expiry_kernel<<<1, 32, 0, stream>>>(max_polls, arrive_first);
    return cudaGetLastError();
}

}  // namespace hils
