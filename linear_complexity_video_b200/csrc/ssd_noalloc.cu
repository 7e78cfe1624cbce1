// Allocation-free entry point of the bi-SSD token mix.
//
// Some callers cannot allocate device memory on their call path: a plugin
// running inside a host application that owns the whole device memory pool,
// code that must not pay the implicit device synchronisation of
// cudaMalloc/cudaFree, or a process whose device memory budget is fixed up
// front. mate_bissd_fwd_noalloc serves them: it runs mate_bissd_fwd with its
// scratch taken from a fixed array that is part of this library's device
// image, so the caller passes only inputs and outputs.
//
// Contract (also in include/mate.h):
//   - The array holds MATE_NOALLOC_SCRATCH_BYTES bytes on every GPU that
//     loads the library, for the life of the process.
//   - A call whose scratch need (mate_bissd_workspace_bytes) exceeds that
//     returns MATE_ERR_WORKSPACE before enqueueing anything.
//   - The first call on a device looks up the array's device address with
//     cudaGetSymbolAddress (that device current); make that first call
//     before any stream capture. A call that finds the device's context
//     re-created since then looks it up again.
//   - All calls share the one array: calls whose work overlaps on the GPU
//     (different streams, no ordering between them) race on it. The array
//     keeps the last call's contents; the kernels write every scratch word
//     they read, so nothing needs clearing between calls.
//   - No cudaMalloc, cudaFree or allocating library routine is called.
#include <cuda_runtime.h>
#include <stddef.h>

#include <mutex>

#include "../../include/mate.h"
#include "devctx.h"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_bissd_scratch[MATE_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

// Device address of g_bissd_scratch in the current device's context (looked up
// once per device, and again after that device's context has been re-created,
// e.g. by cudaDeviceReset), or nullptr with *rc set.
void *scratch_on_current_device(int *rc)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        *rc = MATE_ERR_CUDA;
        return nullptr;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        *rc = MATE_ERR_UNSUPPORTED;
        return nullptr;
    }
    const unsigned long long ctx = mate::current_context_id();
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev] || ctx != g_scratch_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bissd_scratch) != cudaSuccess || !p) {
            *rc = MATE_ERR_CUDA;
            return nullptr;
        }
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" int mate_bissd_fwd_noalloc(const void *x, const float *dt, const float *A, const void *B, const void *C,
                                      const float *D, int T, int H, int W, int scan_mode, const int review_pool[3],
                                      void *out, const mate_ssd_dims *d, void *stream)
{
    const size_t need = mate_bissd_workspace_bytes(T, H, W, review_pool, d);
    if (need == 0)  // invalid or unsupported arguments: let the main entry point name the error
        return mate_bissd_fwd(x, dt, A, B, C, D, T, H, W, scan_mode, review_pool, out, d, nullptr, 0, stream);
    if (need > (size_t)MATE_NOALLOC_SCRATCH_BYTES) return MATE_ERR_WORKSPACE;
    int rc = MATE_OK;
    void *scratch = scratch_on_current_device(&rc);
    if (!scratch) return rc;
    return mate_bissd_fwd(x, dt, A, B, C, D, T, H, W, scan_mode, review_pool, out, d, scratch,
                          (size_t)MATE_NOALLOC_SCRATCH_BYTES, stream);
}
