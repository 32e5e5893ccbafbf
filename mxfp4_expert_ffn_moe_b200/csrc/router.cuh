// router.cuh -- the router linear layer fused with top-k routing.
//
//   logits[t, e] = x[t] . W_r[e] + b_r[e]          (bf16 operands, fp32 accumulate)
//   ids[t, :]    = the k largest logits (value descending, ties to the lower index)
//   weights[t,j] = exp(l_j - l_max) / sum_i exp(l_i - l_max) over the k chosen
// The gpt-oss router is the linear module mlp.router with a bias (FreeToken PR #838,
// "What it does" and the loader notes); its output feeds the routing that the MXFP4
// experts consume as ids + weights (transformers PR #49431).
//
// One CTA per 128-token tile, tokens on the MMA's M side (TMEM lane = token), the E
// router rows (padded to a multiple of 32, at most 256) on N, so the whole logit row
// of a token ends up in one thread's TMEM lane:
//   warp 0     TMA: per K step of 64, the token tile (32-row boxes, 128-byte swizzle)
//              and the router rows (same boxes), into an S-slot ring (S = 8, 6, 4 for
//              E up to 64, 128, 256: about 192 KB, enough loads in flight to cover
//              the HBM round trip of the small per-step boxes)
//   warp 1     TMEM owner and MMA issuer: 4 x tcgen05.mma 128 x E_pad x 16 per step
//   warps 2-5  epilogue, one token per thread (TMEM lane quarter = warp % 4): reads
//              its logits 32 columns at a time, adds the bias, optionally stores the
//              logits, keeps a running top-k (k <= 8) in registers, then the softmax
// Every mbarrier wait is bounded; on a timeout the roles fall through to teardown.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace rtr {

constexpr int BM = 128;                          // tokens per tile (TMEM lanes)
constexpr int BK = 64;                           // K elements per step (128-byte rows)
constexpr int kThreads = 192;
constexpr uint32_t BOX_ROWS = 32;
constexpr uint32_t BOX_BYTES = BOX_ROWS * BK * 2;   // 4096
constexpr uint32_t A_BYTES = BM * BK * 2;           // 16384
constexpr int kMaxK = 8;

__host__ __device__ constexpr int e_pad(int E) { return (E + 31) / 32 * 32; }
__host__ __device__ constexpr uint32_t stage_bytes(int E) { return A_BYTES + (uint32_t)e_pad(E) * BK * 2; }
__host__ __device__ constexpr uint32_t tmem_cols(int E) {
    return e_pad(E) <= 32 ? 32u : e_pad(E) <= 64 ? 64u : e_pad(E) <= 128 ? 128u : 256u;
}
__host__ __device__ constexpr int ring_slots(int E) { return e_pad(E) <= 64 ? 8 : e_pad(E) <= 128 ? 6 : 4; }
// ring + barriers (2 S + 1) + TMEM holder + 1 KB alignment slack
__host__ __device__ constexpr uint32_t smem_bytes(int E, int S) { return S * stage_bytes(E) + 8 * (2 * S + 2) + 1024; }

template <int S>
__global__ void __launch_bounds__(kThreads, 1)
    router_route_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                        const float *__restrict__ bias, int T, int H, int E, int k,
                        float *__restrict__ logits, int32_t *__restrict__ ids,
                        float *__restrict__ weights) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const gbase = smem_raw + (base - raw);
    const int EP = e_pad(E);
    const uint32_t SB = stage_bytes(E);
    auto a_stage = [&](int s) { return base + s * SB; };
    auto b_stage = [&](int s) { return base + s * SB + A_BYTES; };
    const uint32_t bars = base + S * SB;
    auto full = [&](int s) { return bars + 8u * s; };
    auto empty = [&](int s) { return bars + 8u * (S + s); };
    const uint32_t acc_full = bars + 8u * (2 * S);
    const uint32_t tmem_holder = bars + 8u * (2 * S + 1);
    const uint32_t ncols = tmem_cols(E);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = blockIdx.x * BM;
    const int k_iters = H / BK;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), 1);
        }
        ptx::mbar_init(acc_full, 1);
        ptx::fence_mbarrier_init();
        ptx::prefetch_tmap(&tmap_x);
        ptx::prefetch_tmap(&tmap_w);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, ncols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    pdl_wait();
    pdl_trigger();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(gbase + (tmem_holder - base));

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        const int ntok = min(BM, T - row0);
        const int abox = (ntok + (int)BOX_ROWS - 1) / (int)BOX_ROWS;   // rows past T are never read
        const int bbox = EP / (int)BOX_ROWS;                            // rows past E: zero fill
        for (int kb = 0; kb < k_iters; ++kb) {
            const int s = kb % S;
            if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(empty(s), ((kb / S) & 1) ^ 1))) break;
            if (ptx::elect_one()) {
                ptx::mbar_arrive_expect_tx(full(s), (uint32_t)(abox + bbox) * BOX_BYTES);
                for (int b = 0; b < abox; ++b)
                    ptx::tma_load_2d(a_stage(s) + b * BOX_BYTES, &tmap_x, kb * BK, row0 + b * (int)BOX_ROWS, full(s));
                for (int b = 0; b < bbox; ++b)
                    ptx::tma_load_2d(b_stage(s) + b * BOX_BYTES, &tmap_w, kb * BK, b * (int)BOX_ROWS, full(s));
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        const uint32_t idesc = ptx::idesc_bf16_f32(BM, EP);
        bool ok = true;
        for (int kb = 0; kb < k_iters; ++kb) {
            const int s = kb % S;
            if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(full(s), (kb / S) & 1)))) break;
            ptx::tc_fence_after();
            if (ptx::elect_one()) {
                const uint64_t ad = ptx::sw128_kmajor_desc(a_stage(s));
                const uint64_t bd = ptx::sw128_kmajor_desc(b_stage(s));
#pragma unroll
                for (int j = 0; j < BK / 16; ++j)   // +32 B per 16-element K step
                    ptx::mma_bf16(tmem_base, ad + 2u * j, bd + 2u * j, idesc, (kb > 0 || j > 0) ? 1u : 0u);
                ptx::mma_commit(empty(s));
            }
            __syncwarp();
        }
        if (ok && ptx::elect_one()) ptx::mma_commit(acc_full);
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int t = row0 + 32 * q + lane;
        const bool live = t < T;
        if (__all_sync(0xFFFFFFFFu, ptx::mbar_wait(acc_full, 0))) {
            ptx::tc_fence_after();
            float topv[kMaxK];
            int topi[kMaxK];
#pragma unroll
            for (int j = 0; j < kMaxK; ++j) {
                topv[j] = -INFINITY;
                topi[j] = 0x7FFFFFFF;
            }
            for (int c0 = 0; c0 < EP; c0 += 32) {
                uint32_t v[32];
                ptx::tmem_ld_32x32b_x32(tmem_base + (uint32_t)c0 + ((uint32_t)(32 * q) << 16), v);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = c0 + i;
                    if (e >= E) break;                                   // uniform over the warp
                    float cv = __uint_as_float(v[i]) + (bias ? __ldg(bias + e) : 0.0f);
                    if (live && logits) logits[(int64_t)t * E + e] = cv;
                    // insertion into the list ordered by (value descending, index
                    // ascending), the routing kernel's rule; empty slots hold
                    // (-inf, INT_MAX), so a -inf logit still takes one
                    int ci = e;
#pragma unroll
                    for (int j = 0; j < kMaxK; ++j) {
                        if (cv > topv[j] || (cv == topv[j] && ci < topi[j])) {
                            const float tv = topv[j];
                            const int ti = topi[j];
                            topv[j] = cv;
                            topi[j] = ci;
                            cv = tv;
                            ci = ti;
                        }
                    }
                }
            }
            if (live) {
                // softmax over the k chosen, as the standalone routing kernel computes it;
                // a NaN logit never enters the list, so with fewer than k others a slot
                // stays empty: id -1, weight 0, MOE_DEVERR_BAD_LOGIT
                const float m = topv[0];
                float ex[kMaxK], sum = 0.0f;
#pragma unroll
                for (int j = 0; j < kMaxK; ++j) {
                    ex[j] = (j < k && topi[j] < E) ? expf(topv[j] - m) : 0.0f;
                    sum += ex[j];
                }
                const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
#pragma unroll
                for (int j = 0; j < kMaxK; ++j) {
                    if (j < k) {
                        const bool valid = topi[j] < E;
                        if (!valid) raise_device_error(MOE_DEVERR_BAD_LOGIT);
                        ids[(int64_t)t * k + j] = valid ? topi[j] : -1;
                        weights[(int64_t)t * k + j] = ex[j] * inv;
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, ncols);
    }
}

}  // namespace rtr
}  // namespace moe
