// router.cuh -- the router linear layer fused with top-k routing.
//
//   logits[t, e] = x[t] . W_r[e] + b_r[e]          (bf16 operands, fp32 accumulate)
//   ids[t, :]    = the k largest logits (value descending, ties to the lower index)
//   weights[t,j] = exp(l_j - l_max) / sum_i exp(l_i - l_max) over the k chosen
// The gpt-oss router is the linear module mlp.router with a bias (FreeToken PR #838,
// "What it does" and the loader notes); its output feeds the routing that the MXFP4
// experts consume as ids + weights (transformers PR #49431).
//
// Each 128-token tile is computed by a cluster of `ksplit` CTAs (1 to 8), CTA r of the
// cluster taking K steps [r K/ksplit, (r+1) K/ksplit): with few tokens one CTA walking
// all of K would leave the GPU idle and pay every step's load latency in turn.  Tokens
// sit on the MMA's M side (TMEM lane = token), the E router rows (padded to a multiple
// of 32, at most 256) on N, so a token's whole logit row ends up in one TMEM lane.
// After the K loop every CTA writes its partial logits into its own shared memory (the
// ring, idle by then); after a cluster barrier CTA r finishes its slice of the tile's
// tokens, adding the CTAs' partials in rank order (a fixed order: the result does not
// depend on timing) through distributed shared memory; a second cluster barrier keeps
// every CTA's shared memory alive until all have read it.  Roles per CTA:
//   warp 0     TMA: per K step of 64, the token tile (32-row boxes, 128-byte swizzle)
//              and the router rows (same boxes), into an S-slot ring (S = 8, 6, 4 for
//              E up to 64, 128, 256: about 192 KB, enough loads in flight to cover
//              the HBM round trip of the small per-step boxes)
//   warp 1     TMEM owner and MMA issuer: 4 x tcgen05.mma 128 x E_pad x 16 per step
//   warps 2-5  epilogue: the partial logits out of TMEM (TMEM lane quarter =
//              warp % 4), then, with ksplit threads per token of the CTA's slice, the
//              sum of the partials, the bias, the optional logits store, a top-k
//              (k <= 8) per thread merged across the token's threads, the softmax
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

__host__ __device__ constexpr int e_pad(int E) { return (E + 31) / 32 * 32; }
__host__ __device__ constexpr uint32_t stage_bytes(int E) { return A_BYTES + (uint32_t)e_pad(E) * BK * 2; }
__host__ __device__ constexpr uint32_t tmem_cols(int E) {
    return e_pad(E) <= 32 ? 32u : e_pad(E) <= 64 ? 64u : e_pad(E) <= 128 ? 128u : 256u;
}
__host__ __device__ constexpr int ring_slots(int E) { return e_pad(E) <= 64 ? 8 : e_pad(E) <= 128 ? 6 : 4; }
// ring + barriers (2 S + 1) + TMEM holder + 1 KB alignment slack
__host__ __device__ constexpr uint32_t smem_bytes(int E, int S) { return S * stage_bytes(E) + 8 * (2 * S + 2) + 1024; }

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster (release / acquire: shared-memory writes
// before it are visible to the cluster's reads after it).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The shared address `a` of this CTA mapped to CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    return ra;
}

// Four floats at a cluster shared address (16-byte aligned).
__device__ __forceinline__ float4 ld_cluster_v4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(a)
                 : "memory");
    return v;
}

// Partial logits of a CTA: token-major rows of E_pad floats, padded by 4 floats so that
// the 16-byte stores and loads of eight consecutive tokens fall in distinct banks.
__host__ __device__ constexpr int partial_stride(int E) { return e_pad(E) + 4; }
__host__ __device__ constexpr uint32_t partial_bytes(int E) { return (uint32_t)partial_stride(E) * BM * 4; }

// (value, index) a ranks before (value, index) b in the top-k order: value descending,
// index ascending (a NaN value never ranks before anything).
__device__ __forceinline__ bool ranks_before(float av, int ai, float bv, int bi) {
    return av > bv || (av == bv && ai < bi);
}

// KMAX: top-k list length (4 for k <= 4, else 8).
template <int S, int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
    router_route_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                        const float *__restrict__ bias, int T, int H, int E, int k, int ksplit,
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
    const uint32_t rank = cluster_rank();
    const int row0 = (blockIdx.x / ksplit) * BM;
    const int kall = H / BK;
    const int kbeg = (int)rank * kall / ksplit, k_iters = ((int)rank + 1) * kall / ksplit - kbeg;
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
                const int kx = (kbeg + kb) * BK;
                for (int b = 0; b < abox; ++b)
                    ptx::tma_load_2d(a_stage(s) + b * BOX_BYTES, &tmap_x, kx, row0 + b * (int)BOX_ROWS, full(s));
                for (int b = 0; b < bbox; ++b)
                    ptx::tma_load_2d(b_stage(s) + b * BOX_BYTES, &tmap_w, kx, b * (int)BOX_ROWS, full(s));
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
        // ---------------------------------------------------------------- partials
        // this CTA's partial logits (TMEM lane = token) into its shared memory
        const int q = warp & 3;
        const int tok = 32 * q + lane;
        const int PST = partial_stride(E);
        if (__all_sync(0xFFFFFFFFu, ptx::mbar_wait(acc_full, 0))) {
            ptx::tc_fence_after();
            for (int c0 = 0; c0 < EP; c0 += 32) {
                uint32_t v[32];
                ptx::tmem_ld_32x32b_x32(tmem_base + (uint32_t)c0 + ((uint32_t)(32 * q) << 16), v);
                ptx::tmem_ld_wait();
                float4 *row = reinterpret_cast<float4 *>(reinterpret_cast<float *>(gbase) + tok * PST + c0);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    row[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                         __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
        }
    }
    // every CTA's partials are in place
    cluster_sync();
    if (warp >= 2) {
        // ---------------------------------------------------------------- epilogue
        // CTA r of the cluster finishes tokens [r BM/ksplit, (r+1) BM/ksplit) of the tile
        // with ksplit threads per token (adjacent lanes); a thread owns E_pad/ksplit
        // consecutive logit columns: it adds the ranks' partials in rank order (all
        // loads of a chunk in flight before the adds), adds the bias, keeps a top-k
        // list of its columns; the token's threads then merge their lists by shuffles.
        // The order (value descending, index ascending) is total over the non-NaN
        // logits, so the merged list is the one a single pass over all columns keeps.
        const int et = threadIdx.x - 64;
        const int tl = (int)rank * (BM / ksplit) + et / ksplit;    // token within the tile
        const int sub = et % ksplit;
        const int t = row0 + tl;
        const bool live = t < T;
        const int ncol = EP / ksplit;                              // a multiple of 4
        const int cbeg = sub * ncol;
        const int PST = partial_stride(E);
        float topv[KMAX];
        int topi[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            topv[j] = -INFINITY;
            topi[j] = 0x7FFFFFFF;
        }
        // insertion into the list ordered by (value descending, index ascending), the
        // routing kernel's rule; empty slots hold (-inf, INT_MAX), so a -inf logit
        // still takes one and a NaN never does
        auto insert = [&](float cv, int ci) {
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (ranks_before(cv, ci, topv[j], topi[j])) {
                    const float tv = topv[j];
                    const int ti = topi[j];
                    topv[j] = cv;
                    topi[j] = ci;
                    cv = tv;
                    ci = ti;
                }
            }
        };
        const uint32_t prow = base + (uint32_t)((tl * PST + cbeg) * 4);
        for (int cc = 0; cc < ncol; cc += 32) {
            const int w = min(32, ncol - cc);
            float f[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) f[i] = 0.0f;
            // the chunk's bias values, all loads issued before any use (columns past E
            // read a valid element and are never inserted)
            float bv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                bv[i] = (bias && i < w) ? __ldg(bias + min(cbeg + cc + i, E - 1)) : 0.0f;
            for (int r = 0; r < ksplit; ++r) {
                const uint32_t ra = peer_addr(prow + (uint32_t)(cc * 4), (uint32_t)r);
                float4 pv[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (4 * i < w) pv[i] = ld_cluster_v4(ra + 16u * i);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (4 * i < w) {
                        f[4 * i] += pv[i].x;
                        f[4 * i + 1] += pv[i].y;
                        f[4 * i + 2] += pv[i].z;
                        f[4 * i + 3] += pv[i].w;
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int e = cbeg + cc + i;
                if (i >= w || e >= E) break;
                const float cv = f[i] + bv[i];
                if (live && logits) logits[(int64_t)t * E + e] = cv;
                insert(cv, e);
            }
        }
        // merge the lists of the token's ksplit threads (butterfly over adjacent lanes):
        // the better of own entry j and the partner's entry KMAX-1-j is the top KMAX of
        // both lists as a bitonic sequence, which half-cleaners then sort
        for (int m = 1; m < ksplit; m <<= 1) {
            float pv[KMAX];
            int pi[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                pv[j] = __shfl_xor_sync(0xFFFFFFFFu, topv[KMAX - 1 - j], m);
                pi[j] = __shfl_xor_sync(0xFFFFFFFFu, topi[KMAX - 1 - j], m);
            }
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (ranks_before(pv[j], pi[j], topv[j], topi[j])) {
                    topv[j] = pv[j];
                    topi[j] = pi[j];
                }
            }
#pragma unroll
            for (int d = KMAX / 2; d >= 1; d >>= 1) {
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if ((j & d) == 0 && ranks_before(topv[j + d], topi[j + d], topv[j], topi[j])) {
                        const float tv = topv[j];
                        const int ti = topi[j];
                        topv[j] = topv[j + d];
                        topi[j] = topi[j + d];
                        topv[j + d] = tv;
                        topi[j + d] = ti;
                    }
                }
            }
        }
        if (live && sub == 0) {
            // softmax over the k chosen, as the standalone routing kernel computes it;
            // with fewer than k non-NaN logits a slot stays empty: id -1, weight 0,
            // MOE_DEVERR_BAD_LOGIT
            const float m = topv[0];
            float ex[KMAX], sum = 0.0f;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                ex[j] = (j < k && topi[j] < E) ? expf(topv[j] - m) : 0.0f;
                sum += ex[j];
            }
            const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < k) {
                    const bool valid = topi[j] < E;
                    if (!valid) raise_device_error(MOE_DEVERR_BAD_LOGIT);
                    ids[(int64_t)t * k + j] = valid ? topi[j] : -1;
                    weights[(int64_t)t * k + j] = ex[j] * inv;
                }
            }
        }
    }
    // every CTA has read the partials it needs
    cluster_sync();

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, ncols);
    }
}

}  // namespace rtr
}  // namespace moe
