// ctx_id.cu -- the current CUDA context's process-unique id (ctx_memo.h),
// through the driver's cuCtxGetCurrent and cuCtxGetId, looked up once via
// the runtime's driver entry-point query.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "ctx_memo.h"

namespace qlora {
namespace {

typedef CUresult (*GetCurrentFn)(CUcontext*);
typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);

struct DriverFns {
    GetCurrentFn get_current = nullptr;
    GetIdFn get_id = nullptr;
};

const DriverFns& driver_fns() {
    static DriverFns fns;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_current = reinterpret_cast<GetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_id = reinterpret_cast<GetIdFn>(f);
    });
    return fns;
}

}  // namespace

bool current_context_id(uint64_t* id) {
    const DriverFns& d = driver_fns();
    if (!d.get_current || !d.get_id) return false;
    CUcontext ctx = nullptr;
    if (d.get_current(&ctx) != CUDA_SUCCESS) return false;
    if (!ctx) {
        // no context bound to this thread yet: let the runtime bind the
        // current device's primary context
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return false;
        if (d.get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    }
    unsigned long long v = 0;
    if (d.get_id(ctx, &v) != CUDA_SUCCESS) return false;
    *id = static_cast<uint64_t>(v);
    return true;
}

}  // namespace qlora
