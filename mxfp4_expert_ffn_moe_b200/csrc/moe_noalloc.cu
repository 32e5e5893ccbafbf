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
#include "context_id.h"

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

// Device address of the scratch array on the current device, looked up on the
// first call in each context of the device.
int scratch_address(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    const unsigned long long ctx = moe::current_context_id();
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
    g_scratch[dev] = ScratchAddr{moe::current_context_id(), p};
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
