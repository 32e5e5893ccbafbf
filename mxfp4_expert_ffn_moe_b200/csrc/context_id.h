// context_id.h -- identifier of the calling thread's current CUDA context (host side).
//
// Per-context state that the library caches (the allocation-free entry point's scratch
// address, the shared-memory attributes already set on its kernels) belongs to one
// context: after cudaDeviceReset the primary context is created again, modules are
// loaded again and earlier settings are gone.  Keying such caches on the context's
// identifier (cuCtxGetId, through the runtime's driver entry point) makes a new context
// look like a cache miss.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

namespace moe {

// 0 when there is no current context or the driver entry points are unavailable (then
// callers treat every call as a miss).
inline unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *a = nullptr, *b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        const bool ok_a = cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
                          qa == cudaDriverEntryPointSuccess;
        const bool ok_b = cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
                          qb == cudaDriverEntryPointSuccess;
        if (ok_a && ok_b) {
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(a);
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(b);
        } else {
            cudaGetLastError();
        }
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

}  // namespace moe
