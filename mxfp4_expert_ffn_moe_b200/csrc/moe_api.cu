// moe_api.cu -- C ABI and host launch layer of the MXFP4 expert-FFN MoE library.
//
// Declared and documented in include/moe_mxfp4.h.  Validates every argument on
// the host, carves the workspace, and enqueues the kernels on the caller's
// stream: permute -> gather -> gate_up grouped GEMM (+bias, clamped SwiGLU) ->
// down grouped GEMM (+bias, routing weight) -> combine.  No host synchronisation.
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/moe_mxfp4.h"
#include "combine.cuh"
#include "common.cuh"
#include "dequant.cuh"
#include "gemm_simt.cuh"
#include "permute.cuh"
#include "route.cuh"

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Workspace carve-up; offsets in bytes from the workspace base.
struct Workspace {
    size_t counts, offsets, tile_offsets, sorted_pairs, x_perm, act, yp, total;
};

Workspace workspace_layout(int64_t T, int64_t H, int64_t I, int64_t E, int k) {
    const int64_t P = T * k;
    Workspace w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align_up(bytes);
        return o;
    };
    w.counts = take(sizeof(int32_t) * E);
    w.offsets = take(sizeof(int32_t) * (E + 1));
    w.tile_offsets = take(sizeof(int32_t) * (E + 1));
    w.sorted_pairs = take(sizeof(int32_t) * P);
    w.x_perm = take(sizeof(uint16_t) * P * H);
    w.act = take(sizeof(uint16_t) * P * I);
    w.yp = take(sizeof(float) * P * H);
    w.total = off;
    return w;
}

bool forward_sizes_ok(int64_t T, int64_t H, int64_t I, int64_t E, int k) {
    if (T < 1 || E < 1 || E > 256 || k < 1 || k > 8 || k > E) return false;
    if (H < 64 || I < 64 || H % 64 != 0 || I % 64 != 0) return false;
    if (T * k >= (int64_t(1) << 31)) return false;
    if (2 * I >= (int64_t(1) << 31) || H >= (int64_t(1) << 31)) return false;
    return true;
}

int launch_check() { return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ---- per-stage launch counting and optional CUDA-event timing ---------------
struct TimedLaunch {
    int stage;
    cudaEvent_t start, stop;
};
struct Profiler {
    bool timing = false;
    int64_t launches[MOE_PROFILE_STAGES] = {};
    std::vector<TimedLaunch> pending;
};
Profiler g_prof;

// Brackets one kernel launch of `stage` on stream s.
class StageScope {
   public:
    StageScope(int stage, cudaStream_t s) : stage_(stage), s_(s) {
        ++g_prof.launches[stage];
        if (g_prof.timing && cudaEventCreate(&a_) == cudaSuccess && cudaEventCreate(&b_) == cudaSuccess)
            cudaEventRecord(a_, s_);
        else
            a_ = b_ = nullptr;
    }
    ~StageScope() {
        if (a_ && b_) {
            cudaEventRecord(b_, s_);
            g_prof.pending.push_back({stage_, a_, b_});
        }
    }

   private:
    int stage_;
    cudaStream_t s_;
    cudaEvent_t a_ = nullptr, b_ = nullptr;
};

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

}  // namespace

extern "C" {

const char *moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "success";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_NO_MEMORY: return "out of memory or workspace too small";
        case MOE_ERR_DEVICE: return "device-side error flag set";
        default: return "unknown status";
    }
}

int mxfp4_dequantize(const uint8_t *blocks, const uint8_t *scales, uint16_t *out, int64_t E,
                     int64_t N, int64_t K, void *stream) {
    if (!blocks || !scales || !out) return MOE_ERR_INVALID_ARG;
    if (E < 1 || N < 1 || K < 32 || K % 32 != 0) return MOE_ERR_INVALID_ARG;
    if (!aligned(blocks, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
    const int64_t n_words = E * N * (K / 8);
    const int threads = 256;
    int64_t blocks_needed = (n_words + threads - 1) / threads;
    const int64_t cap = (int64_t)sm_count() * 8;
    const int grid = (int)(blocks_needed < cap ? blocks_needed : cap);
    StageScope scope(MOE_STAGE_DEQUANT, (cudaStream_t)stream);
    moe::mxfp4_dequant_kernel<<<grid, threads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint32_t *>(blocks), scales, reinterpret_cast<uint4 *>(out), n_words);
    return launch_check();
}

int moe_route(const float *router_logits, int64_t T, int64_t E, int k, int32_t *ids,
              float *weights, void *stream) {
    if (!router_logits || !ids || !weights) return MOE_ERR_INVALID_ARG;
    if (T < 1 || E < 1 || k < 1 || k > 8 || k > E) return MOE_ERR_INVALID_ARG;
    if (E > 256) return MOE_ERR_UNSUPPORTED;
    const int warps_per_block = 8;
    const int64_t grid = (T + warps_per_block - 1) / warps_per_block;
    if (grid > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    const int vpl = (int)((E + 31) / 32);
    StageScope scope(MOE_STAGE_ROUTE, s);
    switch (vpl) {
#define MOE_ROUTE_CASE(V) \
    case V: moe::route_topk_kernel<V><<<(unsigned)grid, 256, 0, s>>>(router_logits, T, (int)E, k, ids, weights); break;
        MOE_ROUTE_CASE(1)
        MOE_ROUTE_CASE(2)
        MOE_ROUTE_CASE(3)
        MOE_ROUTE_CASE(4)
        MOE_ROUTE_CASE(5)
        MOE_ROUTE_CASE(6)
        MOE_ROUTE_CASE(7)
        MOE_ROUTE_CASE(8)
#undef MOE_ROUTE_CASE
        default: return MOE_ERR_UNSUPPORTED;
    }
    return launch_check();
}

size_t moe_mxfp4_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E, int k) {
    if (!forward_sizes_ok(T, H, I, E, k)) return 0;
    return workspace_layout(T, H, I, E, k).total;
}

int moe_mxfp4_forward_ex(const uint16_t *x, int64_t T, int64_t H, int64_t I, int64_t E, int k,
                         const int32_t *ids, const float *weights,
                         const uint8_t *gate_up_blocks, const uint8_t *gate_up_scales,
                         const float *gate_up_bias, const uint8_t *down_blocks,
                         const uint8_t *down_scales, const float *down_bias, float alpha,
                         float limit, uint16_t *out, uint32_t flags, void *workspace,
                         size_t workspace_bytes, void *stream) {
    if (!x || !ids || !weights || !gate_up_blocks || !gate_up_scales || !down_blocks ||
        !down_scales || !out)
        return MOE_ERR_INVALID_ARG;
    if (!forward_sizes_ok(T, H, I, E, k)) return MOE_ERR_INVALID_ARG;
    if (flags & ~MOE_FLAG_WEIGHT_ON_INPUT) return MOE_ERR_INVALID_ARG;
    const bool woi = (flags & MOE_FLAG_WEIGHT_ON_INPUT) != 0;
    if (woi && (gate_up_bias || down_bias)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(gate_up_blocks, 16) ||
        !aligned(down_blocks, 16) || !aligned(ids, 4) || !aligned(weights, 4) ||
        !aligned(gate_up_bias, 4) || !aligned(down_bias, 4))
        return MOE_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, kAlign)) return MOE_ERR_INVALID_ARG;

    cudaStream_t s = (cudaStream_t)stream;
    const Workspace L = workspace_layout(T, H, I, E, k);
    bool owned = false;
    if (!workspace) {
        if (cudaMallocAsync(&workspace, L.total, s) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_NO_MEMORY;
        }
        owned = true;
    } else if (workspace_bytes < L.total) {
        return MOE_ERR_NO_MEMORY;
    }
    char *ws = static_cast<char *>(workspace);
    int32_t *counts = reinterpret_cast<int32_t *>(ws + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(ws + L.offsets);
    int32_t *tile_offsets = reinterpret_cast<int32_t *>(ws + L.tile_offsets);
    int32_t *sorted_pairs = reinterpret_cast<int32_t *>(ws + L.sorted_pairs);
    uint16_t *x_perm = reinterpret_cast<uint16_t *>(ws + L.x_perm);
    uint16_t *act = reinterpret_cast<uint16_t *>(ws + L.act);
    float *yp = reinterpret_cast<float *>(ws + L.yp);

    const int64_t P = T * k;
    int rc = MOE_OK;
    do {
        {
            const size_t perm_smem = sizeof(int) * (32 * E + E + 1);
            StageScope sp(MOE_STAGE_PERMUTE, s);
            moe::permute_pairs_kernel<<<1, moe::kPermuteThreads, perm_smem, s>>>(
                ids, P, (int)E, moe::kSimtBM, counts, offsets, tile_offsets, sorted_pairs);
        }
        if ((rc = launch_check()) != MOE_OK) break;
        {
            const int64_t gather_grid = moe::ceil_div(P, 8) < sm_count() * 8 ? moe::ceil_div(P, 8) : sm_count() * 8;
            StageScope sg(MOE_STAGE_GATHER, s);
            moe::gather_rows_kernel<<<(unsigned)gather_grid, 256, 0, s>>>(
                x, weights, sorted_pairs, offsets, (int)E, k, H, woi ? 1 : 0, x_perm);
        }
        if ((rc = launch_check()) != MOE_OK) break;
        const int64_t mtiles = moe::ceil_div(P, moe::kSimtBM) + E;
        {
            dim3 g1((unsigned)mtiles, (unsigned)((2 * I) / moe::kSimtBN));
            StageScope su(MOE_STAGE_GATE_UP, s);
            moe::grouped_mxfp4_simt_kernel<true><<<g1, 256, 0, s>>>(
                x_perm, gate_up_blocks, gate_up_scales, gate_up_bias, counts, offsets, tile_offsets,
                (int)E, (int)(2 * I), (int)H, act, alpha, limit, nullptr, sorted_pairs, weights, 0);
        }
        if ((rc = launch_check()) != MOE_OK) break;
        {
            dim3 g2((unsigned)mtiles, (unsigned)(H / moe::kSimtBN));
            StageScope sd(MOE_STAGE_DOWN, s);
            moe::grouped_mxfp4_simt_kernel<false><<<g2, 256, 0, s>>>(
                act, down_blocks, down_scales, down_bias, counts, offsets, tile_offsets, (int)E,
                (int)H, (int)I, nullptr, alpha, limit, yp, sorted_pairs, weights, woi ? 1 : 0);
        }
        if ((rc = launch_check()) != MOE_OK) break;
        {
            const int64_t n4 = T * (H / 4);
            const int64_t cgrid = moe::ceil_div(n4, 256) < sm_count() * 16 ? moe::ceil_div(n4, 256) : sm_count() * 16;
            StageScope sc(MOE_STAGE_COMBINE, s);
            moe::combine_rows_kernel<<<(unsigned)cgrid, 256, 0, s>>>(yp, ids, T, k, (int)E, H, out);
        }
        rc = launch_check();
    } while (0);

    if (owned && cudaFreeAsync(workspace, s) != cudaSuccess && rc == MOE_OK) rc = MOE_ERR_CUDA;
    return rc;
}

int moe_mxfp4_forward(const uint16_t *x, int64_t T, int64_t H, int64_t I, int64_t E, int k,
                      const int32_t *ids, const float *weights, const uint8_t *gate_up_blocks,
                      const uint8_t *gate_up_scales, const float *gate_up_bias,
                      const uint8_t *down_blocks, const uint8_t *down_scales,
                      const float *down_bias, float alpha, float limit, uint16_t *out,
                      void *stream) {
    return moe_mxfp4_forward_ex(x, T, H, I, E, k, ids, weights, gate_up_blocks, gate_up_scales,
                                gate_up_bias, down_blocks, down_scales, down_bias, alpha, limit,
                                out, 0u, nullptr, 0, stream);
}

int moe_profile_enable(int on) {
    g_prof.timing = on != 0;
    return MOE_OK;
}

int moe_profile_read(double *ms, int64_t *launches) {
    double acc[MOE_PROFILE_STAGES] = {};
    int rc = MOE_OK;
    for (const TimedLaunch &t : g_prof.pending) {
        float e = 0.f;
        if (cudaEventSynchronize(t.stop) != cudaSuccess || cudaEventElapsedTime(&e, t.start, t.stop) != cudaSuccess)
            rc = MOE_ERR_CUDA;
        acc[t.stage] += e;
        cudaEventDestroy(t.start);
        cudaEventDestroy(t.stop);
    }
    g_prof.pending.clear();
    for (int i = 0; i < MOE_PROFILE_STAGES; ++i) {
        if (ms) ms[i] = acc[i];
        if (launches) launches[i] = g_prof.launches[i];
        g_prof.launches[i] = 0;
    }
    return rc;
}

int moe_get_device_error(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, moe::g_device_error, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(moe::g_device_error, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    return v;
}

}  // extern "C"
