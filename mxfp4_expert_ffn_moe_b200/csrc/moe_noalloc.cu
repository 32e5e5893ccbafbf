// moe_noalloc.cu -- the layer for callers that cannot allocate device memory.
//
// moe_mxfp4_forward_noalloc (declared in include/moe_mxfp4.h) runs exactly the
// path of moe_mxfp4_forward_ex, with its workspace placed in a file-scope device
// array instead of memory the caller or the stream-ordered pool provides.  Some
// callers cannot allocate: plugins that only receive input and output buffers
// from a host framework owning all device memory, serving loops that must not
// allocate (and so risk blocking, failing or synchronising) after start-up, and
// processes whose device memory is partitioned up front.
//
// The array's name is only a host-side stand-in in this file; the device address
// is looked up with cudaGetSymbolAddress while the device is current, and that
// address is what the kernels receive.  It is cached per device together with the
// identifier of the device's current context: when the primary context is
// destroyed and created again (cudaDeviceReset), the module is loaded again and the
// array may sit at another address, so a new context identifier means a new lookup.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe_mxfp4.h"

// Held by every GPU that loads this library, until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
struct ScratchAddr {
    unsigned long long ctx_id;   // context the address belongs to (0: unknown)
    void *addr;
};
std::mutex g_scratch_mutex;
ScratchAddr g_scratch[kMaxDevices] = {};

// Identifier of the calling thread's current context, or 0 when there is none or
// the driver entry points are unavailable (then every call looks the address up).
// Called with g_scratch_mutex held.
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {
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
        resolved = true;
    }
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array on the current device, looked up on the
// first call in each context of the device.
int scratch_address(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    const unsigned long long ctx = current_context_id();
    if (ctx != 0 && g_scratch[dev].addr && g_scratch[dev].ctx_id == ctx) {
        *addr = g_scratch[dev].addr;
        return MOE_OK;
    }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        g_scratch[dev] = ScratchAddr{0, nullptr};
        return MOE_ERR_CUDA;
    }
    // the lookup has made the device's context current if it was not yet
    g_scratch[dev] = ScratchAddr{current_context_id(), p};
    *addr = p;
    return MOE_OK;
}

}  // namespace

extern "C" int moe_mxfp4_forward_noalloc(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                                         int64_t E, int k, const int32_t *ids,
                                         const float *weights, const uint8_t *gate_up_blocks,
                                         const uint8_t *gate_up_scales, const float *gate_up_bias,
                                         const uint8_t *down_blocks, const uint8_t *down_scales,
                                         const float *down_bias, float alpha, float limit,
                                         uint16_t *out, uint32_t flags, void *stream) {
    const size_t need = moe_mxfp4_workspace_size(T, H, I, E, k);
    if (need == 0) return MOE_ERR_INVALID_ARG;
    if (need > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_NO_MEMORY;
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != MOE_OK) return rc;
    return moe_mxfp4_forward_ex(x, T, H, I, E, k, ids, weights, gate_up_blocks, gate_up_scales,
                                gate_up_bias, down_blocks, down_scales, down_bias, alpha, limit,
                                out, flags, scratch, MOE_NOALLOC_SCRATCH_BYTES, stream);
}
