// da2_plan_static.cu -- da2_plan_static: the routing step with its working
// memory in a fixed device array owned by the library, for callers that
// cannot allocate device memory themselves (see include/da2.h).
//
// The array lives in this shared library: every GPU on which the library is
// used holds DA2_PLAN_STATIC_BYTES of it until the process exits.  Its device
// address is looked up once per device (cudaGetSymbolAddress, with that
// device current) on the first call made on that device; later calls reuse
// it.  The routing kernels clear every part of their working memory that must
// start at zero at the start of each call, so leftovers of the previous call
// are harmless; two calls that run at the same time on one GPU share the
// array and corrupt each other.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/da2.h"
#include "da2_kernels.h"

// The working memory (file scope; host code must not pass its name to a
// kernel: on the host it is only a stand-in, the device address comes from
// cudaGetSymbolAddress below).
static __device__ __align__(256) unsigned char g_plan_static[DA2_PLAN_STATIC_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_addr[kMaxDevices] = {};

// Device address of the array on the handle's device, which must be the
// current device (looked up once per device).
int static_scratch(da2_handle h, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return da2::record_cuda_error(e);
    if (dev != da2::handle_device(h) || dev < 0 || dev >= kMaxDevices) return DA2_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_plan_static);
        if (e != cudaSuccess) {
            cudaGetLastError();  // take the error out of the runtime's last-error slot
            return da2::record_cuda_error(e);
        }
        if (!p) return DA2_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return DA2_OK;
}

}  // namespace

extern "C" int da2_plan_static(da2_handle h, const da2_prepared* prep, const da2_budget* budget, uint8_t* prec,
                               int32_t* cnt, int64_t* off, uint16_t* kidx, double* A, void* stream) {
    if (!h) return DA2_ERR_ARG;
    da2_sizes_t sz;
    int rc = da2_sizes(h, &sz);
    if (rc != DA2_OK) return rc;
    if (sz.plan_scratch > (size_t)DA2_PLAN_STATIC_BYTES) return DA2_ERR_ARG;  // problem too large for the array
    void* scratch = nullptr;
    if ((rc = static_scratch(h, &scratch)) != DA2_OK) return rc;
    da2_plan_bufs bufs;
    bufs.prec = prec;
    bufs.cnt = cnt;
    bufs.off = off;
    bufs.kidx = kidx;
    bufs.A = A;
    bufs.scratch = scratch;
    return da2_plan(h, prep, budget, &bufs, stream);
}
