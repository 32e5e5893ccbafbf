// gemm_tc.cuh -- grouped MXFP4 expert GEMM on the sm_100a tensor cores (tcgen05).
//
// For every (expert e, 128-row M tile, 192-row N tile) of a projection:
//   acc[m, n] = sum_k A[row0 + m, k] * W[e, n0 + n, k]         (bf16 x bf16 -> fp32)
// with W decoded from MXFP4 (E2M1 codes, element 2j in the low nibble of byte j,
// one E8M0 byte per 32 elements of a row) inside shared memory, then
//   gate_up epilogue: h = acc + b_gu[e]; gate = h[2i], up = h[2i+1];
//                     act[row, i] = bf16(clamped SwiGLU(gate, up))
//   down epilogue:    yp[p, n] = w[p] * (acc + b_d[e])   (router weight on output)
//                     yp[p, n] = acc                     (router weight on input)
// (MoE-Infinity PR #152, Changes: dequant-on-copy of fetched packed experts,
// [N, K//2] layout, scales, bias, gate/up split, clamped SwiGLU, fp32 accumulate;
// FreeToken PR #838: gate_up bias before the gated activation, down bias before
// the routing weight, sum w*(y + b).)
//
// One persistent CTA per SM, warp-specialised:
//   warp 0        TMA producer: activation tile (128 x 64 bf16, 128-byte swizzle)
//                 and packed weight tile (192 rows x 32 bytes) per K step
//   warp 1        TMEM owner and MMA issuer: 4 x tcgen05.mma 128x192x16 per K step
//                 into one of two 192-column fp32 accumulators
//   warps 2..5    epilogue: tcgen05.ld of the accumulator rows, fused bias and
//                 SwiGLU / routing weight, global stores
//   warps 6..17   converters: packed E2M1 + E8M0 -> bf16 in the 128-byte swizzled
//                 K-major layout the MMA reads, one 32-element block per thread
// Stage ring of 4 (A tile, packed W tile, bf16 W tile); two TMEM accumulators
// let the epilogue of one tile overlap the main loop of the next.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;              // rows (token slots) per tile, TMEM lanes
constexpr int BN = 192;              // weight rows per tile, accumulator columns
constexpr int BK = 64;               // K elements per stage (one 128-byte swizzle row)
constexpr int STAGES = 4;
constexpr int ACC_STRIDE = 256;      // TMEM columns between the two accumulators
constexpr int TMEM_COLS = 512;
constexpr int kConvWarps = 12;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps + kConvWarps);   // 576
constexpr int kFirstEpiWarp = 2;
constexpr int kFirstConvWarp = 2 + kEpiWarps;

constexpr uint32_t A_BYTES = BM * BK * 2;        // 16384
constexpr uint32_t BP_BYTES = BN * BK / 2;       // 6144 packed codes
constexpr uint32_t BB_BYTES = BN * BK * 2;       // 24576 bf16
constexpr uint32_t STAGE_BYTES = A_BYTES + BB_BYTES + BP_BYTES;
constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*barriers*/ + 1024 /*align slack*/;
static_assert(A_BYTES % 1024 == 0 && BB_BYTES % 1024 == 0 && BP_BYTES % 1024 == 0, "1 KB aligned");
static_assert(BN * 2 == kConvWarps * 32, "one converter thread per 32-element block");

struct Params {
    const int32_t *counts;        // [E]
    const int32_t *offsets;       // [E + 1]
    const int32_t *tile_offsets;  // [E + 1] in BM-row tiles
    const uint8_t *wscales;       // [E, N, K/32]
    const float *bias;            // [E, N] or null
    int E, N, K;
    // gate_up epilogue
    uint16_t *act;                // [rows, N/2] bf16
    float alpha, limit;
    // down epilogue
    float *yp;                    // [T*k, N] fp32, indexed by pair
    const int32_t *sorted_pairs;  // [rows]
    const float *weights;         // [T*k]
    int weight_on_input;
};

__device__ __forceinline__ int tile_expert(const int32_t *__restrict__ tile_offsets, int E, int m) {
    int lo = 0, hi = E - 1;  // largest e with tile_offsets[e] <= m
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(tile_offsets + mid) <= m)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

struct TileInfo {
    int e, row0, mrows, n0;
};

__device__ __forceinline__ TileInfo decode_tile(const Params &p, int tile, int n_tiles) {
    TileInfo t;
    const int m = tile / n_tiles;
    const int nt = tile - m * n_tiles;
    t.e = tile_expert(p.tile_offsets, p.E, m);
    const int mt = m - __ldg(p.tile_offsets + t.e);
    t.row0 = __ldg(p.offsets + t.e) + mt * BM;
    t.mrows = min(BM, __ldg(p.counts + t.e) - mt * BM);
    t.n0 = nt * BN;
    return t;
}

// Eight E2M1 codes -> four bf16x2 words holding E2M1(code) * 2^-126: sign bit to
// bit 15 of its half, the three magnitude bits (exponent bits and mantissa msb)
// to bits 8..6.  Code 1 (0.5) becomes the bf16 subnormal 2^-127, still exact.
// Element order is natural: word j holds elements 2j (low half) and 2j + 1.
__device__ __forceinline__ void e2m1x8_to_bf16_rep(uint32_t q, uint32_t &r0, uint32_t &r1,
                                                   uint32_t &r2, uint32_t &r3) {
    const uint32_t lo = q & 0x0F0F0F0Fu;          // even elements, one per byte
    const uint32_t hi = (q >> 4) & 0x0F0F0F0Fu;   // odd elements
    // [code 2j, 0, code 2j+1, 0] (selector 8 copies the zero msb of a small byte)
    r0 = (ptx::prmt(lo, hi, 0x8480u) * 0x1040u) & 0x81C081C0u;
    r1 = (ptx::prmt(lo, hi, 0x8581u) * 0x1040u) & 0x81C081C0u;
    r2 = (ptx::prmt(lo, hi, 0x8682u) * 0x1040u) & 0x81C081C0u;
    r3 = (ptx::prmt(lo, hi, 0x8783u) * 0x1040u) & 0x81C081C0u;
}

template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_mxfp4_tc_kernel(const __grid_constant__ CUtensorMap tmap_a,
                            const __grid_constant__ CUtensorMap tmap_w, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    auto stage_a = [&](int s) { return base + s * STAGE_BYTES; };
    auto stage_bb = [&](int s) { return base + s * STAGE_BYTES + A_BYTES; };
    auto stage_bp = [&](int s) { return base + s * STAGE_BYTES + A_BYTES + BB_BYTES; };
    const uint32_t bars = base + STAGES * STAGE_BYTES;
    auto full_tma = [&](int s) { return bars + 8u * s; };
    auto full_conv = [&](int s) { return bars + 8u * (STAGES + s); };
    auto empty = [&](int s) { return bars + 8u * (2 * STAGES + s); };
    auto tmem_full = [&](int b) { return bars + 8u * (3 * STAGES + b); };
    auto tmem_empty = [&](int b) { return bars + 8u * (3 * STAGES + 2 + b); };
    const uint32_t tmem_holder = bars + 8u * (3 * STAGES + 4);
    uint8_t *smem_generic = smem_raw + (base - raw);
    volatile uint32_t *tmem_holder_ptr =
        reinterpret_cast<volatile uint32_t *>(smem_generic + (tmem_holder - base));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(full_tma(s), 1);
            ptx::mbar_init(full_conv(s), kConvWarps);
            ptx::mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(tmem_full(b), 1);
            ptx::mbar_init(tmem_empty(b), kEpiWarps);
        }
        ptx::fence_mbarrier_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_w);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_holder_ptr;

    const int n_tiles = (p.N + BN - 1) / BN;
    const int total = __ldg(p.tile_offsets + p.E) * n_tiles;
    const int k_iters = p.K / BK;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileInfo t = decode_tile(p, tile, n_tiles);
                for (int kb = 0; kb < k_iters; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!(ok = ptx::mbar_wait(empty(s), ph ^ 1u))) break;
                    ptx::mbar_arrive_expect_tx(full_tma(s), A_BYTES + BP_BYTES);
                    ptx::tma_load_2d(stage_a(s), &tmap_a, kb * BK, t.row0, full_tma(s));
                    ptx::tma_load_3d(stage_bp(s), &tmap_w, kb * (BK / 2), t.n0, t.e, full_tma(s));
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, BN);
            uint32_t it = 0, local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++local) {
                const int b = local & 1;
                const uint32_t tph = (local >> 1) & 1u;
                if (!(ok = ptx::mbar_wait(tmem_empty(b), tph ^ 1u))) break;
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * ACC_STRIDE;
                for (int kb = 0; kb < k_iters; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!(ok = ptx::mbar_wait(full_conv(s), ph))) break;
                    if (!(ok = ptx::mbar_wait(full_tma(s), ph))) break;
                    ptx::tc_fence_after();
#pragma unroll
                    for (int j = 0; j < BK / 16; ++j) {
                        const uint64_t ad = ptx::sw128_kmajor_desc(stage_a(s) + 32u * j);
                        const uint64_t bd = ptx::sw128_kmajor_desc(stage_bb(s) + 32u * j);
                        ptx::mma_bf16(d_tmem, ad, bd, idesc, (kb > 0 || j > 0) ? 1u : 0u);
                    }
                    ptx::mma_commit(empty(s));
                }
                if (ok) ptx::mma_commit(tmem_full(b));
            }
        }
    } else if (warp < kFirstConvWarp) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int r = q * 32 + lane;             // accumulator row of this thread
        uint32_t local = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
            const TileInfo t = decode_tile(p, tile, n_tiles);
            const int b = local & 1;
            const uint32_t tph = (local >> 1) & 1u;
            if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(tmem_full(b), tph))) break;
            ptx::tc_fence_after();
            const bool valid = r < t.mrows;
            const int64_t grow = (int64_t)t.row0 + r;
            int pair = 0;
            float wgt = 1.0f;
            if (!kGateUp && valid) {
                pair = __ldg(p.sorted_pairs + grow);
                if (!p.weight_on_input) wgt = __ldg(p.weights + pair);
            }
            const float *bias = p.bias ? p.bias + (int64_t)t.e * p.N : nullptr;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t v[32];
                ptx::tmem_ld_32x32b_x32(tmem_base + b * ACC_STRIDE + c0 + ((uint32_t)(q * 32) << 16), v);
                ptx::tmem_ld_wait();
                const int n = t.n0 + c0;
                if (!valid || n >= p.N) continue;
                if (kGateUp) {
                    uint32_t packed[8];
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        float a2[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int c = 2 * (i + h);
                            float gate = __uint_as_float(v[c]);
                            float up = __uint_as_float(v[c + 1]);
                            if (bias) {
                                gate += __ldg(bias + n + c);
                                up += __ldg(bias + n + c + 1);
                            }
                            a2[h] = clamped_swiglu(gate, up, p.alpha, p.limit);
                        }
                        packed[i / 2] = pack_bf16x2(a2[0], a2[1]);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(p.act + grow * (p.N / 2) + n / 2);
                    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(p.yp + (int64_t)pair * p.N + n);
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        float4 o;
                        o.x = __uint_as_float(v[c + 0]);
                        o.y = __uint_as_float(v[c + 1]);
                        o.z = __uint_as_float(v[c + 2]);
                        o.w = __uint_as_float(v[c + 3]);
                        if (bias) {
                            const float4 bb = __ldg(reinterpret_cast<const float4 *>(bias + n + c));
                            o.x += bb.x;
                            o.y += bb.y;
                            o.z += bb.z;
                            o.w += bb.w;
                        }
                        o.x *= wgt;
                        o.y *= wgt;
                        o.z *= wgt;
                        o.w *= wgt;
                        dst[c / 4] = o;
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(tmem_empty(b));
        }
    } else {
        // ------------------------------------------------------------ converters
        const int ct = threadIdx.x - 32 * kFirstConvWarp;   // 0 .. 383
        const int row = ct >> 1;                              // weight row in the tile
        const int blk = ct & 1;                               // 32-element half of the K step
        const uint32_t sw = (uint32_t)(row & 7);
        const int kblocks = p.K / 32;
        uint32_t it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            const TileInfo t = decode_tile(p, tile, n_tiles);
            const int n = t.n0 + row;
            const bool in_range = n < p.N;
            const uint8_t *srow = p.wscales + ((int64_t)t.e * p.N + (in_range ? n : 0)) * kblocks + blk;
            uint32_t s_next = in_range ? __ldg(srow) : 127u;
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1u;
                const uint32_t sc = s_next;
                if (kb + 1 < k_iters) s_next = in_range ? __ldg(srow + 2 * (kb + 1)) : 127u;
                // multiplier(s): bf16 2^(s-1) when it fits, else 2^126 then 2^(s-127)
                uint32_t m1, m2 = 0;
                if (sc == 255u) {
                    raise_device_error(MOE_DEVERR_BAD_SCALE);
                    m1 = 0x7FC07FC0u;
                } else if (sc <= 128u) {
                    m1 = ((sc + 126u) << 7) * 0x10001u;
                } else {
                    m1 = 0x7E807E80u;
                    m2 = (sc << 7) * 0x10001u;
                }
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(full_tma(s), ph)))) break;
                const uint4 q4 = ptx::ld_shared_v4(stage_bp(s) + row * 32 + blk * 16);
                const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
                const uint32_t dst_row = stage_bb(s) + row * 128;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t r0, r1, r2, r3;
                    e2m1x8_to_bf16_rep(qw[w], r0, r1, r2, r3);
                    r0 = ptx::hmul2_bf16(r0, m1);
                    r1 = ptx::hmul2_bf16(r1, m1);
                    r2 = ptx::hmul2_bf16(r2, m1);
                    r3 = ptx::hmul2_bf16(r3, m1);
                    if (m2) {
                        r0 = ptx::hmul2_bf16(r0, m2);
                        r1 = ptx::hmul2_bf16(r1, m2);
                        r2 = ptx::hmul2_bf16(r2, m2);
                        r3 = ptx::hmul2_bf16(r3, m2);
                    }
                    const uint32_t chunk = (uint32_t)(blk * 4 + w);
                    ptx::st_shared_v4(dst_row + ((chunk ^ sw) << 4), r0, r1, r2, r3);
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(full_conv(s));
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace moe
