// See devctx.h.
#include "devctx.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

namespace mate {

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct CtxFns {
    CtxGetCurrentFn get_current = nullptr;
    CtxGetIdFn get_id = nullptr;
};

const CtxFns &ctx_fns()
{
    static CtxFns fns;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    return fns;
}

}  // namespace

unsigned long long current_context_id()
{
    const CtxFns &f = ctx_fns();
    if (!f.get_current || !f.get_id) return 0;
    // make sure the runtime has made the device's primary context current
    if (cudaFree(nullptr) != cudaSuccess) return 0;
    CUcontext ctx = nullptr;
    if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

}  // namespace mate
