// moe_api.cu -- C ABI and host launch layer of the MXFP4 expert-FFN MoE library.
//
// Declared and documented in include/moe_mxfp4.h.  Validates every argument on
// the host, carves the workspace, and enqueues the kernels on the caller's
// stream: permute -> gather -> gate_up grouped GEMM (+bias, clamped SwiGLU) ->
// down grouped GEMM (+bias, routing weight) -> combine.  No host synchronisation.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>
#include <stdlib.h>

#include "../../include/moe_mxfp4.h"
#include "context_id.h"
#include "combine.cuh"
#include "common.cuh"
#include "dequant.cuh"
#include "gemm_mxf.cuh"
#include "gemm_swap.cuh"
#include "permute.cuh"
#include "split.cuh"
#include "route.cuh"
#include "router.cuh"

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Workspace carve-up; offsets in bytes from the workspace base.
struct Workspace {
    // x_perm / act: bf16 rows, or (block-scaled path) the rows split into two E4M3
    // planes with per-step scale slots
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
    const auto rows_bytes = [&](int64_t K) {
        const int64_t bf16 = int64_t(sizeof(uint16_t)) * P * K, split = 2 * P * moe::split_row_bytes(K);
        return (size_t)(bf16 > split ? bf16 : split);
    };
    w.x_perm = take(rows_bytes(H));
    w.act = take(rows_bytes(I));
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

// An NVTX range around one entry point (named on a profiler's timeline; free when no
// tool is attached).
class NvtxRange {
   public:
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

// Average (token, slot) pairs per expert up to which the layer uses decode tiles:
// MOE_DECODE_MAX_TOKENS_PER_EXPERT from the environment (read once; a non-negative
// integer), 32 by default (FreeToken PR #838's mmvq_max_tokens plays the same role
// between its decode and prefill kernels).
int64_t decode_max_tokens_per_expert() {
    static const int64_t v = [] {
        const char *e = getenv("MOE_DECODE_MAX_TOKENS_PER_EXPERT");
        if (!e || !*e) return (int64_t)32;
        char *end = nullptr;
        const long long x = strtoll(e, &end, 10);
        return (end && *end == '\0' && x >= 0 && x <= (1ll << 30)) ? (int64_t)x : (int64_t)32;
    }();
    return v;
}

// Launch with programmatic stream serialisation: the kernel may be scheduled while
// its predecessor in the stream is still running; every kernel of the layer calls
// pdl_wait() before touching data its predecessor writes (see common.cuh).
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);   // errors surface in launch_check
}

// The same with thread-block clusters of `cluster` CTAs along x (grid.x a multiple).
template <typename... KArgs, typename... Args>
void launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, unsigned cluster,
                        cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);   // errors surface in launch_check
}

// ---- per-stage launch counting and optional CUDA-event timing ---------------
struct TimedLaunch {
    int stage;
    cudaEvent_t start, stop;
};
struct Profiler {
    uint32_t timed_stages = 0;   // bit i: bracket stage i's launches with events
    int64_t launches[MOE_PROFILE_STAGES] = {};
    std::vector<TimedLaunch> pending;
};
Profiler g_prof;

// Brackets one kernel launch of `stage` on stream s.
class StageScope {
   public:
    StageScope(int stage, cudaStream_t s) : stage_(stage), s_(s) {
        ++g_prof.launches[stage];
        if (((g_prof.timed_stages >> stage) & 1u) && cudaEventCreate(&a_) == cudaSuccess &&
            cudaEventCreate(&b_) == cudaSuccess)
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

// ---- TMA descriptors ---------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// bf16 activations [rows, K], K-major: box of 64 elements (128 B, swizzled) x 32 rows.
bool make_act_map(CUtensorMap *m, const void *ptr, int64_t rows, int64_t K) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K * 2)};
    cuuint32_t box[2] = {(cuuint32_t)moe::swp::BK, moe::swp::XBOX_ROWS};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// packed MXFP4 codes [E, N, K/2] bytes: box of 32 bytes (64 codes) x 128 rows x 1 expert.
bool make_weight_map(CUtensorMap *m, const void *ptr, int64_t E, int64_t N, int64_t K) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)(K / 2), (cuuint64_t)N, (cuuint64_t)E};
    cuuint64_t strides[2] = {(cuuint64_t)(K / 2), (cuuint64_t)(N * (K / 2))};
    cuuint32_t box[3] = {(cuuint32_t)(moe::swp::BK / 2), (cuuint32_t)moe::swp::BM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// split activations [2][rows][K] bytes (hi plane, lo plane): box of 128 bytes
// (swizzled) x 16 rows x 1 plane.
bool make_split_map(CUtensorMap *m, const void *ptr, int64_t rows, int64_t K) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const int64_t RS = moe::split_row_bytes(K);
    cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, 2};
    cuuint64_t strides[2] = {(cuuint64_t)RS, (cuuint64_t)(rows * RS)};
    cuuint32_t box[3] = {(cuuint32_t)moe::mxf::BK, (cuuint32_t)moe::mxf::XBOX_ROWS, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// the 16-byte per-step scale slots of the same rows: box of 16 bytes x 16 rows x 1 plane.
bool make_split_scale_map(CUtensorMap *m, const uint8_t *ptr, int64_t rows, int64_t K) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const int64_t RS = moe::split_row_bytes(K);
    cuuint64_t dims[3] = {(cuuint64_t)(RS - K), (cuuint64_t)rows, 2};
    cuuint64_t strides[2] = {(cuuint64_t)RS, (cuuint64_t)(rows * RS)};
    cuuint32_t box[3] = {16, (cuuint32_t)moe::mxf::XBOX_ROWS, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(ptr + K), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// packed MXFP4 codes [E, N, K/2] bytes: box of WP_ROW bytes (128: 128-byte swizzle;
// 256: unswizzled) x 128 rows x 1 expert.
bool make_packed_map(CUtensorMap *m, const void *ptr, int64_t E, int64_t N, int64_t K) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)(K / 2), (cuuint64_t)N, (cuuint64_t)E};
    cuuint64_t strides[2] = {(cuuint64_t)(K / 2), (cuuint64_t)(N * (K / 2))};
    cuuint32_t box[3] = {moe::mxf::WP_ROW, (cuuint32_t)moe::mxf::BM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE,
               moe::mxf::WP_SWIZZLED ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) is a driver call per function and
// context; the largest size already set is remembered per (kernel, device, context), so
// that repeated calls of an entry point skip it (a new context is a miss).
bool ensure_smem_attr(const void *kernel, int bytes) {
    static std::mutex mu;
    static std::map<std::tuple<const void *, int, unsigned long long>, int> done;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const unsigned long long ctx = moe::current_context_id();
    const auto key = std::make_tuple(kernel, dev, ctx);
    if (ctx != 0) {
        std::lock_guard<std::mutex> lock(mu);
        const auto it = done.find(key);
        if (it != done.end() && it->second >= bytes) return true;
    }
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (ctx != 0) {
        std::lock_guard<std::mutex> lock(mu);
        int &v = done[key];
        if (v < bytes) v = bytes;
    }
    return true;
}

int max_smem_optin() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
    return v;
}

// Grouped projection: rows of A (expert order, [rows, K] bf16) x packed weights
// [E, N, K/2] of each row's expert, with the gate_up or the down epilogue; kNv
// selects NVFP4 scales (E4M3 per 16 elements, weight_scale_2 in scale2).
template <class Cfg, bool kGateUp, bool kNv>
int launch_grouped_gemm(int stage, const uint16_t *A, int64_t rows, int64_t K, const uint8_t *wblocks,
                        const uint8_t *wscales, const float *scale2, const float *bias, int64_t E, int64_t N,
                        const int32_t *counts, const int32_t *offsets, const int32_t *tile_offsets,
                        uint16_t *act, float alpha, float limit, float *yp,
                        const int32_t *sorted_pairs, const float *weights, int woi, cudaStream_t s) {
    CUtensorMap mx, mw;
    if (!make_act_map(&mx, A, rows, K) || !make_weight_map(&mw, wblocks, E, N, K)) return MOE_ERR_CUDA;
    moe::swp::Params p{};
    p.counts = counts;
    p.offsets = offsets;
    p.tile_offsets = tile_offsets;
    p.wscales = wscales;
    p.scale2 = scale2;
    p.bias = bias;
    p.E = (int)E;
    p.N = (int)N;
    p.K = (int)K;
    p.act = act;
    p.alpha = alpha;
    p.limit = limit;
    p.yp = yp;
    p.sorted_pairs = sorted_pairs;
    p.weights = weights;
    p.weight_on_input = woi;
    p.rows_cap = (int)rows;
    const uint32_t smem = Cfg::smem_bytes((int)(K / 32));
    if ((int)smem > max_smem_optin()) return MOE_ERR_UNSUPPORTED;
    auto kernel = moe::swp::grouped_mxfp4_swap_kernel<Cfg, kGateUp, kNv>;
    if (!ensure_smem_attr(reinterpret_cast<const void *>(kernel), (int)smem))
        return MOE_ERR_CUDA;
    const int64_t w_tiles = moe::ceil_div(N, moe::swp::BM);
    const int64_t max_items = (moe::ceil_div(rows, Cfg::TOK) + E) * w_tiles;
    const int grid = (int)(max_items < sm_count() ? max_items : sm_count());
    StageScope scope(stage, s);
    launch_pdl(kernel, dim3(grid), dim3(moe::swp::kThreads), smem, s, mx, mw, p);
    return launch_check();
}

// Both projections with one tile configuration.
template <class Cfg, bool kNv>
int launch_projections(const uint16_t *x_perm, uint16_t *act, float *yp, int64_t P, int64_t H,
                       int64_t I, int64_t E, const uint8_t *gate_up_blocks,
                       const uint8_t *gate_up_scales, const float *gate_up_scale2,
                       const float *gate_up_bias, const uint8_t *down_blocks,
                       const uint8_t *down_scales, const float *down_scale2,
                       const float *down_bias, float alpha, float limit, const int32_t *counts,
                       const int32_t *offsets, const int32_t *tile_offsets,
                       const int32_t *sorted_pairs, const float *weights, bool woi, cudaStream_t s) {
    int rc = launch_grouped_gemm<Cfg, true, kNv>(MOE_STAGE_GATE_UP, x_perm, P, H, gate_up_blocks,
                                                 gate_up_scales, gate_up_scale2, gate_up_bias, E, 2 * I,
                                                 counts, offsets, tile_offsets, act, alpha, limit, nullptr,
                                                 sorted_pairs, weights, 0, s);
    if (rc != MOE_OK) return rc;
    return launch_grouped_gemm<Cfg, false, kNv>(MOE_STAGE_DOWN, act, P, I, down_blocks, down_scales,
                                                down_scale2, down_bias, E, H, counts, offsets, tile_offsets,
                                                nullptr, alpha, limit, yp, sorted_pairs, weights,
                                                woi ? 1 : 0, s);
}

// Block-scaled grouped projection: split rows B ([2][P][K] + scale words) x packed
// weights [E, N, K/2] of each row's expert, with the gate_up or the down epilogue.
template <class Cfg, bool kGateUp>
int launch_mxf_gemm(int stage, const uint8_t *bq, int64_t P, int64_t K, const uint8_t *wblocks,
                    const uint8_t *wscales, const float *bias, int64_t E, int64_t N,
                    const int32_t *counts, const int32_t *offsets, const int32_t *tile_offsets,
                    uint8_t *actq, float alpha, float limit, float *yp,
                    const int32_t *sorted_pairs, const float *weights, int woi, cudaStream_t s) {
    CUtensorMap mb, mbs, mw;
    if (!make_split_map(&mb, bq, P, K) || !make_split_scale_map(&mbs, bq, P, K) ||
        !make_packed_map(&mw, wblocks, E, N, K))
        return MOE_ERR_CUDA;
    moe::mxf::Params p{};
    p.counts = counts;
    p.offsets = offsets;
    p.tile_offsets = tile_offsets;
    p.wscales = wscales;
    p.bias = bias;
    p.E = (int)E;
    p.N = (int)N;
    p.K = (int)K;
    p.P = (int)P;
    p.actq = actq;
    p.alpha = alpha;
    p.limit = limit;
    p.yp = yp;
    p.sorted_pairs = sorted_pairs;
    p.weights = weights;
    p.weight_on_input = woi;
    const uint32_t smem = Cfg::smem_bytes((int)(K / 32));
    if ((int)smem > max_smem_optin()) return MOE_ERR_UNSUPPORTED;
    auto kernel = moe::mxf::grouped_mxfp4_mxf_kernel<Cfg, kGateUp>;
    if (!ensure_smem_attr(reinterpret_cast<const void *>(kernel), (int)smem))
        return MOE_ERR_CUDA;
    const int64_t w_tiles = moe::ceil_div(N, moe::mxf::BM);
    const int64_t max_items = (moe::ceil_div(P, Cfg::TOK) + E) * w_tiles;
    const int grid = (int)(max_items < sm_count() ? max_items : sm_count());
    StageScope scope(stage, s);
    launch_pdl(kernel, dim3(grid), dim3(Cfg::kThreads), smem, s, mb, mbs, mw, p);
    return launch_check();
}

// Split of the gathered rows, then both projections on the block-scaled path.
template <class Cfg>
int launch_mxf_layer(const uint16_t *x, const float *weights, const int32_t *sorted_pairs,
                     uint8_t *xq, uint8_t *actq, float *yp, int64_t P,
                     int64_t H, int64_t I, int64_t E, int k, const uint8_t *gate_up_blocks,
                     const uint8_t *gate_up_scales, const float *gate_up_bias,
                     const uint8_t *down_blocks, const uint8_t *down_scales,
                     const float *down_bias, float alpha, float limit, const int32_t *counts,
                     const int32_t *offsets, const int32_t *tile_offsets, bool woi, cudaStream_t s) {
    {
        const int64_t items = P * moe::ceil_div(H, 128);
        const int64_t grid = moe::ceil_div(items, 8) < sm_count() * 8 ? moe::ceil_div(items, 8) : sm_count() * 8;
        StageScope sg(MOE_STAGE_GATHER, s);
        launch_pdl(moe::split_rows_kernel, dim3((unsigned)grid), dim3(256), 0, s, x, weights, sorted_pairs,
                   offsets, (int)E, k, H, P, woi ? 1 : 0, xq);
    }
    int rc = launch_check();
    if (rc != MOE_OK) return rc;
    rc = launch_mxf_gemm<Cfg, true>(MOE_STAGE_GATE_UP, xq, P, H, gate_up_blocks, gate_up_scales,
                                    gate_up_bias, E, 2 * I, counts, offsets, tile_offsets, actq,
                                    alpha, limit, nullptr, sorted_pairs, weights, 0, s);
    if (rc != MOE_OK) return rc;
    return launch_mxf_gemm<Cfg, false>(MOE_STAGE_DOWN, actq, P, I, down_blocks, down_scales,
                                       down_bias, E, H, counts, offsets, tile_offsets, nullptr,
                                       alpha, limit, yp, sorted_pairs, weights, woi ? 1 : 0, s);
}

// Token tiles of 32 rows (deep weight pipeline) when experts see few rows on
// average (decode_max_tokens_per_expert), 256-row tiles otherwise.
bool use_decode_tiles(int64_t P, int64_t E) { return P <= decode_max_tokens_per_expert() * E; }

// Tile configurations of the grouped GEMMs: the block-scaled kernel (decode tiles) holds
// two tiles' scale rows (128 x K/32 bytes each) in shared memory; for K too large for
// that, the converter kernel's 32-token tiles take over.
enum TileConfig { kDecodeSmem, kPrefillSmem, kDecodeMxf, kPrefillMxf };

#ifndef MOE_MXF_DECODE
#define MOE_MXF_DECODE 1
#endif

#ifndef MOE_MXF_PREFILL
#define MOE_MXF_PREFILL 0
#endif

template <class Cfg>
bool config_fits(int64_t H, int64_t I) {
    const int optin = max_smem_optin();
    return (int)Cfg::smem_bytes((int)(H / 32)) <= optin && (int)Cfg::smem_bytes((int)(I / 32)) <= optin;
}

// NVFP4 banks always take the converter kernel: the block-scaled MMA of the decode
// tiles reads E8M0 scales per 32 elements only.
TileConfig pick_config(int64_t P, int64_t H, int64_t I, int64_t E, bool nv) {
    if (nv) return use_decode_tiles(P, E) ? kDecodeSmem : kPrefillSmem;
    if (use_decode_tiles(P, E))
        return (MOE_MXF_DECODE && config_fits<moe::mxf::DecodeCfg>(H, I)) ? kDecodeMxf : kDecodeSmem;
    return (MOE_MXF_PREFILL && config_fits<moe::mxf::PrefillCfg>(H, I)) ? kPrefillMxf : kPrefillSmem;
}

int config_tok(TileConfig c) {
    switch (c) {
        case kDecodeSmem: return moe::swp::DecodeCfg::TOK;
        case kPrefillSmem: return moe::swp::PrefillCfg::TOK;
        case kDecodeMxf: return moe::mxf::DecodeCfg::TOK;
        default: return moe::mxf::PrefillCfg::TOK;
    }
}

// Pair permutation: about one CTA per 2048 pairs (at most 64 unless the sub-chunk
// ids would not fit in shared memory), each placing its own range.
int launch_permute(const int32_t *ids, int expert_base, int64_t P, int64_t E, int tile_rows, int32_t *counts,
                   int32_t *offsets, int32_t *tile_offsets, int32_t *sorted_pairs, int32_t *pair_rows,
                   cudaStream_t s) {
    const size_t cap = std::min<size_t>(moe::kPermuteSmemCap, (size_t)max_smem_optin());
    const size_t fixed = moe::permute_smem_bytes((int)E, 0);
    if (fixed + 64 > cap) return MOE_ERR_UNSUPPORTED;
    const int64_t sc_max = (int64_t)((cap - fixed) / 64);
    int64_t C = std::min<int64_t>(std::max<int64_t>(1, moe::ceil_div(P, moe::kPermutePairsPerCta)), 64);
    if (moe::permute_subchunk(P, (int)C) > sc_max) C = moe::ceil_div(P, 32 * sc_max);
    if (C > 0x7FFFFFFF) return MOE_ERR_INVALID_ARG;
    const size_t smem = moe::permute_smem_bytes((int)E, moe::permute_subchunk(P, (int)C));
    if (!ensure_smem_attr(reinterpret_cast<const void *>(moe::permute_pairs_kernel), (int)smem))
        return MOE_ERR_CUDA;
    StageScope sp(MOE_STAGE_PERMUTE, s);
    launch_pdl(moe::permute_pairs_kernel, dim3((unsigned)C), dim3(moe::kPermuteThreads), smem, s, ids, expert_base,
               P, (int)E, tile_rows, counts, offsets, tile_offsets, sorted_pairs, pair_rows);
    return launch_check();
}

// The whole layer on the caller's stream: permute -> gather (or split) -> gate_up ->
// down -> combine.  nv: NVFP4 banks (E4M3 scales per 16 elements, weight_scale_2).
// expert_base: ids are taken relative to it (the banks hold experts expert_base ..
// expert_base + E - 1).  rows_out: when given, the weighted expert rows (fp32 [T*k, H],
// indexed by pair) are written there and the combine is skipped (out unused).
int forward_layer(bool nv, const uint16_t *x, int64_t T, int64_t H, int64_t I, int64_t E, int k,
                  const int32_t *ids, const float *weights, const uint8_t *gate_up_blocks,
                  const uint8_t *gate_up_scales, const float *gate_up_scale2, const float *gate_up_bias,
                  const uint8_t *down_blocks, const uint8_t *down_scales, const float *down_scale2,
                  const float *down_bias, float alpha, float limit, uint16_t *out, uint32_t flags,
                  void *workspace, size_t workspace_bytes, void *stream, int64_t expert_base = 0,
                  float *rows_out = nullptr) {
    if (!x || !ids || !weights || !gate_up_blocks || !gate_up_scales || !down_blocks ||
        !down_scales || (!out && !rows_out))
        return MOE_ERR_INVALID_ARG;
    if (expert_base < 0 || expert_base > (int64_t)0x7FFFFFFF) return MOE_ERR_INVALID_ARG;
    if (rows_out && !aligned(rows_out, 16)) return MOE_ERR_INVALID_ARG;
    if (!forward_sizes_ok(T, H, I, E, k)) return MOE_ERR_INVALID_ARG;
    if (flags & ~MOE_FLAG_WEIGHT_ON_INPUT) return MOE_ERR_INVALID_ARG;
    const bool woi = (flags & MOE_FLAG_WEIGHT_ON_INPUT) != 0;
    if (woi && (gate_up_bias || down_bias)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || (out && !aligned(out, 16)) || !aligned(gate_up_blocks, 16) ||
        !aligned(down_blocks, 16) || !aligned(gate_up_scales, 16) || !aligned(down_scales, 16) ||
        !aligned(ids, 4) || !aligned(weights, 4) ||
        !aligned(gate_up_bias, 4) || !aligned(down_bias, 4) ||
        !aligned(gate_up_scale2, 4) || !aligned(down_scale2, 4))
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
    float *yp = rows_out ? rows_out : reinterpret_cast<float *>(ws + L.yp);

    const int64_t P = T * k;
    const TileConfig cfg = pick_config(P, H, I, E, nv);
    int rc = MOE_OK;
    do {
        if ((rc = launch_permute(ids, (int)expert_base, P, E, config_tok(cfg), counts, offsets, tile_offsets,
                                 sorted_pairs, nullptr, s)) != MOE_OK)
            break;
        const bool mxf = cfg == kDecodeMxf || cfg == kPrefillMxf;
        if (mxf) {
            uint8_t *xq = reinterpret_cast<uint8_t *>(x_perm);
            uint8_t *actq = reinterpret_cast<uint8_t *>(act);
#define MOE_MXF_LAYER(C)                                                                          \
    launch_mxf_layer<C>(x, weights, sorted_pairs, xq, actq, yp, P, H, I, E, k, gate_up_blocks,           \
                        gate_up_scales, gate_up_bias, down_blocks, down_scales, down_bias, alpha,    \
                        limit, counts, offsets, tile_offsets, woi, s)
            rc = cfg == kDecodeMxf ? MOE_MXF_LAYER(moe::mxf::DecodeCfg) : MOE_MXF_LAYER(moe::mxf::PrefillCfg);
#undef MOE_MXF_LAYER
            if (rc != MOE_OK) break;
        } else {
            {
                const int64_t gather_grid =
                    moe::ceil_div(P, 8) < sm_count() * 8 ? moe::ceil_div(P, 8) : sm_count() * 8;
                StageScope sg(MOE_STAGE_GATHER, s);
                launch_pdl(moe::gather_rows_kernel, dim3((unsigned)gather_grid), dim3(256), 0, s, x, weights,
                           sorted_pairs, offsets, (int)E, k, H, woi ? 1 : 0, x_perm, nullptr, nullptr,
                           nullptr, P);
            }
            if ((rc = launch_check()) != MOE_OK) break;
#define MOE_PROJECTIONS(C, NV)                                                                    \
    launch_projections<C, NV>(x_perm, act, yp, P, H, I, E, gate_up_blocks, gate_up_scales,           \
                              gate_up_scale2, gate_up_bias, down_blocks, down_scales, down_scale2,   \
                              down_bias, alpha, limit, counts, offsets, tile_offsets, sorted_pairs,  \
                              weights, woi, s)
            if (nv)
                rc = cfg == kDecodeSmem ? MOE_PROJECTIONS(moe::swp::DecodeCfg, true)
                                        : MOE_PROJECTIONS(moe::swp::PrefillCfg, true);
            else
                rc = cfg == kDecodeSmem ? MOE_PROJECTIONS(moe::swp::DecodeCfg, false)
                                        : MOE_PROJECTIONS(moe::swp::PrefillCfg, false);
#undef MOE_PROJECTIONS
        }
        if (rc != MOE_OK || rows_out) break;
        {
            const int64_t n4 = T * (H / 4);
            const int64_t cgrid = moe::ceil_div(n4, 256) < sm_count() * 16 ? moe::ceil_div(n4, 256) : sm_count() * 16;
            StageScope sc(MOE_STAGE_COMBINE, s);
            launch_pdl(moe::combine_rows_kernel, dim3((unsigned)cgrid), dim3(256), 0, s, yp, ids, T, k, (int)E, H,
                       out);
        }
        rc = launch_check();
    } while (0);

    if (owned && cudaFreeAsync(workspace, s) != cudaSuccess && rc == MOE_OK) rc = MOE_ERR_CUDA;
    return rc;
}

// Standalone decode of a packed bank to bf16; kHostSrc: blocks and scales are the
// device mappings of page-locked host memory.
template <bool kHostSrc>
int launch_mxfp4_dequant(const uint8_t *blocks, const uint8_t *scales, uint16_t *out, int64_t E, int64_t N,
                         int64_t K, cudaStream_t stream) {
    if (!blocks || !scales || !out) return MOE_ERR_INVALID_ARG;
    if (E < 1 || N < 1 || K < 32 || K % 32 != 0) return MOE_ERR_INVALID_ARG;
    if (!aligned(blocks, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
    // one wave of 6 blocks per SM, each owning a contiguous run of whole rounds
    const int64_t n_words = E * N * (K / 8);
    const int64_t rounds = moe::ceil_div(n_words, moe::kDequantWords);
    const int64_t cap = (int64_t)sm_count() * 6;
    const int grid = (int)(rounds < cap ? rounds : cap);
    const int64_t words_per_block = moe::ceil_div(rounds, grid) * moe::kDequantWords;
    StageScope scope(MOE_STAGE_DEQUANT, stream);
    moe::mxfp4_dequant_kernel<kHostSrc><<<grid, moe::kDequantThreads, 0, stream>>>(
        reinterpret_cast<const uint32_t *>(blocks), scales, reinterpret_cast<uint4 *>(out), n_words, words_per_block);
    return launch_check();
}

template <bool kHostSrc>
int launch_nvfp4_dequant(const uint8_t *blocks, const uint8_t *scales, const float *scale2, uint16_t *out,
                         int64_t E, int64_t N, int64_t K, cudaStream_t stream) {
    if (!blocks || !scales || !out) return MOE_ERR_INVALID_ARG;
    if (E < 1 || N < 1 || K < 16 || K % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (!aligned(blocks, 16) || !aligned(out, 16) || !aligned(scale2, 4)) return MOE_ERR_INVALID_ARG;
    const int64_t words_per_expert = N * (K / 8);
    const int threads = 256;
    // one wave: as many blocks as the SMs hold at once, spread over the experts
    static int per_sm = 0;
    if (per_sm == 0 &&
        (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, moe::nvfp4_dequant_kernel<kHostSrc>, threads, 0) !=
             cudaSuccess || per_sm < 1))
        per_sm = 4;
    const int64_t target = (int64_t)sm_count() * per_sm;
    const int64_t gy = E < 65535 ? E : 65535;
    int64_t gx = target / gy;
    const int64_t need_x = moe::ceil_div(words_per_expert, threads);
    if (gx > need_x) gx = need_x;
    if (gx < 1) gx = 1;
    StageScope scope(MOE_STAGE_DEQUANT, stream);
    moe::nvfp4_dequant_kernel<kHostSrc><<<dim3((unsigned)gx, (unsigned)gy), threads, 0, stream>>>(
        reinterpret_cast<const uint32_t *>(blocks), scales, scale2, reinterpret_cast<uint4 *>(out),
        words_per_expert, E);
    return launch_check();
}

// Dequant-on-copy from host memory (MoE-Infinity PR #152: fetched packed experts are
// dequantised on copy): the device address of `bytes` of page-locked host memory, or
// an error when the first or the last byte is not host memory the current device can
// address, or the two are not mapped contiguously.
int device_view_of_host(const void *host, int64_t bytes, const void **dev) {
    if (!host || bytes < 1) return MOE_ERR_INVALID_ARG;
    const char *first = static_cast<const char *>(host);
    const char *last = first + (bytes - 1);
    cudaPointerAttributes a, b;
    if (cudaPointerGetAttributes(&a, first) != cudaSuccess || cudaPointerGetAttributes(&b, last) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_INVALID_ARG;
    }
    if (a.type != cudaMemoryTypeHost || b.type != cudaMemoryTypeHost || !a.devicePointer || !b.devicePointer)
        return MOE_ERR_INVALID_ARG;
    if (static_cast<const char *>(b.devicePointer) != static_cast<const char *>(a.devicePointer) + (bytes - 1))
        return MOE_ERR_INVALID_ARG;
    *dev = a.devicePointer;
    return MOE_OK;
}

bool bank_sizes_ok(int64_t E, int64_t N, int64_t K, int64_t block) {
    return E >= 1 && N >= 1 && K >= block && K % block == 0 && E <= (int64_t(1) << 40) / N / K;
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
    NvtxRange nvtx("mxfp4_dequantize");
    return launch_mxfp4_dequant<false>(blocks, scales, out, E, N, K, (cudaStream_t)stream);
}

int nvfp4_dequantize(const uint8_t *blocks, const uint8_t *scales, const float *scale2, uint16_t *out,
                     int64_t E, int64_t N, int64_t K, void *stream) {
    NvtxRange nvtx("nvfp4_dequantize");
    return launch_nvfp4_dequant<false>(blocks, scales, scale2, out, E, N, K, (cudaStream_t)stream);
}

int mxfp4_dequantize_from_host(const uint8_t *host_blocks, const uint8_t *host_scales, uint16_t *out,
                               int64_t E, int64_t N, int64_t K, void *stream) {
    NvtxRange nvtx("mxfp4_dequantize_from_host");
    if (!host_blocks || !host_scales || !out || !bank_sizes_ok(E, N, K, 32)) return MOE_ERR_INVALID_ARG;
    const void *db = nullptr, *ds = nullptr;
    int rc = device_view_of_host(host_blocks, E * N * (K / 2), &db);
    if (rc == MOE_OK) rc = device_view_of_host(host_scales, E * N * (K / 32), &ds);
    if (rc != MOE_OK) return rc;
    return launch_mxfp4_dequant<true>(static_cast<const uint8_t *>(db), static_cast<const uint8_t *>(ds), out, E,
                                      N, K, (cudaStream_t)stream);
}

int nvfp4_dequantize_from_host(const uint8_t *host_blocks, const uint8_t *host_scales,
                               const float *scale2, uint16_t *out, int64_t E, int64_t N, int64_t K,
                               void *stream) {
    NvtxRange nvtx("nvfp4_dequantize_from_host");
    if (!host_blocks || !host_scales || !out || !bank_sizes_ok(E, N, K, 16)) return MOE_ERR_INVALID_ARG;
    const void *db = nullptr, *ds = nullptr;
    int rc = device_view_of_host(host_blocks, E * N * (K / 2), &db);
    if (rc == MOE_OK) rc = device_view_of_host(host_scales, E * N * (K / 16), &ds);
    if (rc != MOE_OK) return rc;
    return launch_nvfp4_dequant<true>(static_cast<const uint8_t *>(db), static_cast<const uint8_t *>(ds), scale2,
                                      out, E, N, K, (cudaStream_t)stream);
}

int moe_route(const float *router_logits, int64_t T, int64_t E, int k, int32_t *ids,
              float *weights, void *stream) {
    NvtxRange nvtx("moe_route");
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

int moe_router_route(const uint16_t *x, const uint16_t *w_router, const float *b_router, int64_t T,
                     int64_t H, int64_t E, int k, float *logits, int32_t *ids, float *weights,
                     void *stream) {
    NvtxRange nvtx("moe_router_route");
    if (!x || !w_router || !ids || !weights) return MOE_ERR_INVALID_ARG;
    if (T < 1 || T > (int64_t)0x7FFFFFFF - moe::rtr::BM) return MOE_ERR_INVALID_ARG;
    if (H < 64 || H % 64 != 0 || H > (int64_t)0x7FFFFFFF) return MOE_ERR_INVALID_ARG;
    if (E < 1 || k < 1 || k > 8 || k > E) return MOE_ERR_INVALID_ARG;
    if (E > 256) return MOE_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(b_router, 4) || !aligned(logits, 4) ||
        !aligned(ids, 4) || !aligned(weights, 4))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    CUtensorMap mx, mw;
    if (!make_act_map(&mx, x, T, H) || !make_act_map(&mw, w_router, E, H)) return MOE_ERR_CUDA;
    const int slots = moe::rtr::ring_slots((int)E);
    const uint32_t smem = moe::rtr::smem_bytes((int)E, slots);
    if ((int)smem > max_smem_optin()) return MOE_ERR_UNSUPPORTED;
    // the split-K partials reuse the ring once the K loop is done
    if (moe::rtr::partial_bytes((int)E) > (uint32_t)slots * moe::rtr::stage_bytes((int)E)) return MOE_ERR_UNSUPPORTED;
    auto kernel = k <= 4 ? (slots == 8   ? moe::rtr::router_route_kernel<8, 4>
                            : slots == 6 ? moe::rtr::router_route_kernel<6, 4>
                                         : moe::rtr::router_route_kernel<4, 4>)
                         : (slots == 8   ? moe::rtr::router_route_kernel<8, 8>
                            : slots == 6 ? moe::rtr::router_route_kernel<6, 8>
                                         : moe::rtr::router_route_kernel<4, 8>);
    if (!ensure_smem_attr(reinterpret_cast<const void *>(kernel), (int)smem))
        return MOE_ERR_CUDA;
    // K split over a cluster of up to 8 CTAs per 128-token tile, so that small T still
    // spreads over the SMs (and no split once the tiles alone fill them)
    const int64_t tiles = moe::ceil_div(T, moe::rtr::BM);
    // (a power of two: a token's threads are adjacent lanes of one warp)
    int64_t ksplit = 1;
    while (ksplit < 8 && tiles * ksplit * 2 <= sm_count() && ksplit * 2 <= H / moe::rtr::BK) ksplit *= 2;
    if (tiles * ksplit > (int64_t)0x7FFFFFFF) return MOE_ERR_INVALID_ARG;
    StageScope scope(MOE_STAGE_ROUTE, s);
    launch_pdl_cluster(kernel, dim3((unsigned)(tiles * ksplit)), dim3(moe::rtr::kThreads), smem, (unsigned)ksplit, s,
                       mx, mw, b_router, (int)T, (int)H, (int)E, k, (int)ksplit, logits, ids, weights);
    return launch_check();
}

int moe_gather_pairs(const uint16_t *x, int64_t T, int64_t H, int k, const int32_t *ids, const float *weights,
                     const int32_t *sorted_pairs, const int32_t *offsets, int64_t E, uint16_t *x_rows,
                     int32_t *row_ids, float *row_weights, void *stream) {
    NvtxRange nvtx("moe_gather_pairs");
    if (!x || !ids || !weights || !sorted_pairs || !offsets || !x_rows || !row_ids || !row_weights)
        return MOE_ERR_INVALID_ARG;
    if (T < 1 || k < 1 || k > 8 || E < 1 || E > 256 || H < 8 || H % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (T * k >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(x_rows, 16)) return MOE_ERR_INVALID_ARG;
    const int64_t P = T * k;
    const int64_t grid = moe::ceil_div(P, 8) < sm_count() * 8 ? moe::ceil_div(P, 8) : sm_count() * 8;
    cudaStream_t s = (cudaStream_t)stream;
    StageScope sg(MOE_STAGE_GATHER, s);
    launch_pdl(moe::gather_rows_kernel, dim3((unsigned)grid), dim3(256), 0, s, x, weights, sorted_pairs, offsets,
               (int)E, k, H, 0, x_rows, ids, row_ids, row_weights, P);
    return launch_check();
}

int moe_mxfp4_expert_rows(const uint16_t *x_rows, int64_t R, int64_t H, int64_t I, int64_t E, int64_t expert_base,
                          const int32_t *row_ids, const float *row_weights, const uint8_t *gate_up_blocks,
                          const uint8_t *gate_up_scales, const float *gate_up_bias,
                          const uint8_t *down_blocks, const uint8_t *down_scales, const float *down_bias,
                          float alpha, float limit, float *y_rows, uint32_t flags, void *workspace,
                          size_t workspace_bytes, void *stream) {
    NvtxRange nvtx("moe_mxfp4_expert_rows");
    if (!y_rows) return MOE_ERR_INVALID_ARG;
    return forward_layer(false, x_rows, R, H, I, E, 1, row_ids, row_weights, gate_up_blocks, gate_up_scales,
                         nullptr, gate_up_bias, down_blocks, down_scales, nullptr, down_bias, alpha, limit,
                         nullptr, flags, workspace, workspace_bytes, stream, expert_base, y_rows);
}

int moe_combine_pairs(const float *y_rows, const int32_t *pair_rows, int64_t T, int k, int64_t H, uint16_t *out,
                      void *stream) {
    NvtxRange nvtx("moe_combine_pairs");
    if (!y_rows || !pair_rows || !out) return MOE_ERR_INVALID_ARG;
    if (T < 1 || k < 1 || k > 8 || H < 4 || H % 4 != 0) return MOE_ERR_INVALID_ARG;
    if (!aligned(y_rows, 16) || !aligned(out, 8)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t n4 = T * (H / 4);
    const int64_t cgrid = moe::ceil_div(n4, 256) < sm_count() * 16 ? moe::ceil_div(n4, 256) : sm_count() * 16;
    StageScope sc(MOE_STAGE_COMBINE, s);
    launch_pdl(moe::combine_pair_rows_kernel, dim3((unsigned)cgrid), dim3(256), 0, s, y_rows, pair_rows, T, k, H,
               out);
    return launch_check();
}

int moe_permute(const int32_t *ids, int64_t T, int k, int64_t E, int tile_rows, int32_t *counts,
                int32_t *offsets, int32_t *tile_offsets, int32_t *sorted_pairs, int32_t *pair_rows,
                void *stream) {
    NvtxRange nvtx("moe_permute");
    if (!ids || !counts || !offsets || !tile_offsets || !sorted_pairs) return MOE_ERR_INVALID_ARG;
    if (T < 1 || k < 1 || k > 8 || E < 1 || E > 256 || tile_rows < 1) return MOE_ERR_INVALID_ARG;
    if (T * k >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
    return launch_permute(ids, 0, T * k, E, tile_rows, counts, offsets, tile_offsets, sorted_pairs, pair_rows,
                          (cudaStream_t)stream);
}

int moe_token_tile_rows(int64_t T, int64_t H, int64_t I, int64_t E, int k, int nvfp4) {
    if (!forward_sizes_ok(T, H, I, E, k)) return MOE_ERR_INVALID_ARG;
    return config_tok(pick_config(T * k, H, I, E, nvfp4 != 0));
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
    NvtxRange nvtx("moe_mxfp4_forward_ex");
    return forward_layer(false, x, T, H, I, E, k, ids, weights, gate_up_blocks, gate_up_scales, nullptr,
                         gate_up_bias, down_blocks, down_scales, nullptr, down_bias, alpha, limit, out,
                         flags, workspace, workspace_bytes, stream);
}

int moe_nvfp4_forward_ex(const uint16_t *x, int64_t T, int64_t H, int64_t I, int64_t E, int k,
                         const int32_t *ids, const float *weights,
                         const uint8_t *gate_up_blocks, const uint8_t *gate_up_scales,
                         const float *gate_up_scale2, const float *gate_up_bias,
                         const uint8_t *down_blocks, const uint8_t *down_scales,
                         const float *down_scale2, const float *down_bias, float alpha,
                         float limit, uint16_t *out, uint32_t flags, void *workspace,
                         size_t workspace_bytes, void *stream) {
    NvtxRange nvtx("moe_nvfp4_forward_ex");
    return forward_layer(true, x, T, H, I, E, k, ids, weights, gate_up_blocks, gate_up_scales,
                         gate_up_scale2, gate_up_bias, down_blocks, down_scales, down_scale2, down_bias,
                         alpha, limit, out, flags, workspace, workspace_bytes, stream);
}

int moe_mxfp4_forward(const uint16_t *x, int64_t T, int64_t H, int64_t I, int64_t E, int k,
                      const int32_t *ids, const float *weights, const uint8_t *gate_up_blocks,
                      const uint8_t *gate_up_scales, const float *gate_up_bias,
                      const uint8_t *down_blocks, const uint8_t *down_scales,
                      const float *down_bias, float alpha, float limit, uint16_t *out,
                      void *stream) {
    NvtxRange nvtx("moe_mxfp4_forward");
    return moe_mxfp4_forward_ex(x, T, H, I, E, k, ids, weights, gate_up_blocks, gate_up_scales,
                                gate_up_bias, down_blocks, down_scales, down_bias, alpha, limit,
                                out, 0u, nullptr, 0, stream);
}

int moe_profile_enable(int on) {
    g_prof.timed_stages = on ? (1u << MOE_PROFILE_STAGES) - 1u : 0u;
    return MOE_OK;
}

int moe_profile_enable_stages(uint32_t stage_mask) {
    if (stage_mask >> MOE_PROFILE_STAGES) return MOE_ERR_INVALID_ARG;
    g_prof.timed_stages = stage_mask;
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
