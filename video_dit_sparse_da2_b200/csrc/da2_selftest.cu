// da2_selftest.cu -- a kernel that exercises the bounded-wait failure path of
// the library's kernels without faulting or hanging the GPU.
//
// Warp 0 waits, through the same bounded wait the attention kernel uses, on
// an mbarrier that nothing ever arrives on; after `limit_ns` it gives up,
// raises the CTA's abort flag and sets the timeout bit of the status word.
// Warp 1 waits on the same barrier with a limit 1000 times longer and must
// return as soon as it sees the abort flag (the short-cut by which the other
// roles of a stuck kernel stop waiting).  Both then return normally.
#include "da2_common.cuh"
#include "da2_kernels.h"

namespace da2 {

namespace {

__global__ void __launch_bounds__(64) wait_selftest_kernel(unsigned* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_sh;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_sh = 0;
        fence_mbar_init();
    }
    __syncthreads();
    volatile int* abort_v = &abort_sh;
    const int warp = threadIdx.x >> 5;
    const unsigned long long limit = warp == 0 ? limit_ns : 1000ull * limit_ns;
    // every lane of a warp waits (as the roles of the attention kernel do)
    const bool done = mbar_wait(&bar, 0, abort_v, status, limit);
    (void)done;
    __syncthreads();
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned* status, unsigned long long limit_ns, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 64, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace da2
