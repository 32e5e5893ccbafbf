// gemm_swap.cuh -- grouped MXFP4 expert GEMM on sm_100a tensor cores, weights on
// the MMA's M side.
//
// For every (expert e, token tile of up to TOK rows of that expert, 128-row weight
// tile) of a projection:
//   acc[n, t] = sum_k W[e, m0 + n, k] * A[row0 + t, k]          (bf16 x bf16 -> fp32)
// with W decoded from MXFP4 (E2M1 codes, element 2j in the low nibble of byte j,
// one E8M0 byte per 32 elements of a row) inside shared memory, then
//   gate_up epilogue: h = acc + b_gu[e]; gate = h[2i], up = h[2i+1] (adjacent
//                     TMEM lanes); act[row, i] = bf16(clamped SwiGLU(gate, up))
//   down epilogue:    yp[p, n] = w[p] * (acc + b_d[e])   (router weight on output)
//                     yp[p, n] = acc                     (router weight on input)
// (MoE-Infinity PR #152, Changes: dequant-on-copy of fetched packed experts,
// [N, K//2] layout, scales, bias, gate/up split, clamped SwiGLU, fp32 accumulate;
// FreeToken PR #838: gate_up bias before the gated activation, down bias before
// the routing weight, sum w*(y + b).)
//
// NVFP4 experts (kNv): the same codes with one E4M3 scale per 16 elements decode to
// E2M1 * E4M3 (exact in bf16: at most 6 significant bits), and the per-expert fp32
// weight_scale_2 s multiplies the accumulator before the bias, h = s*acc + b and
// y = s*acc + b, with one s for the gate rows and one for the up rows of gate_up
// (FreeToken PR #838, review item "NVFP4 down scale vs. down bias": sum w*(s*y + b)).
//
// Why weights on M: one tcgen05.mma 128 x TOK x 16 applies every decoded weight
// element to TOK token rows, so the in-smem decode work per MAC is 1/TOK (1/256 for
// prefill tiles), and a tile's token count sets the MMA's N, so small decode
// batches cost MMA time in proportion to their tokens.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0        token TMA: per K step the token tile (32-row boxes, 128-byte
//                 swizzle), into the ring slot the MMA freed
//   warp 22       packed-weight TMA: per K step the weight tile (128 rows x 32 B,
//                 3-D map, out-of-range rows zero-filled), into a deeper ring the
//                 converters free as soon as they have read it
//   warp 1        TMEM owner and MMA issuer (4 x 128 x N x 16 per K step)
//   warps 2..5    epilogue (TMEM lane quarter = warp % 4)
//   warps 6..21   converters in 4 groups; group g converts the K steps with
//                 index % 4 == g (two 32-element blocks per thread per step)
// Rings: token and converted-weight slots released together by the MMA; packed
// weight slots released by the converters; two TMEM accumulators.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace swp {

constexpr int BM = 128;              // weight rows per tile (TMEM lanes)
constexpr int BK = 64;               // K elements per stage (one 128-byte swizzle row)
constexpr int TMEM_COLS = 512;
#ifndef MOE_CONV_WARPS
#define MOE_CONV_WARPS 16
#endif
#ifndef MOE_CONV_GROUPS
#define MOE_CONV_GROUPS 4
#endif
constexpr int kConvWarps = MOE_CONV_WARPS;
// Converter warps form kConvGroups groups; group g converts the K steps with
// step index % kConvGroups == g, so that several steps (each ending in a proxy
// fence) are converted at once.
constexpr int kConvGroups = MOE_CONV_GROUPS;
constexpr int kGroupThreads = 32 * kConvWarps / kConvGroups;
constexpr int kBlocksPerThread = 2 * 128 / kGroupThreads;   // 32-element blocks per step
constexpr int kEpiWarps = 4;
constexpr int kWpWarp = 2 + kEpiWarps + kConvWarps;          // packed-weight TMA producer
constexpr int kThreads = 32 * (3 + kEpiWarps + kConvWarps);
constexpr int kFirstConvWarp = 2 + kEpiWarps;
constexpr uint32_t WP_BYTES = BM * BK / 2;                     // 4096 packed codes
constexpr uint32_t WB_BYTES = BM * BK * 2;                     // 16384 bf16
constexpr uint32_t XBOX_ROWS = 32;                             // token rows per TMA box
constexpr uint32_t XBOX_BYTES = XBOX_ROWS * BK * 2;            // 4096
static_assert(kBlocksPerThread * kGroupThreads == BM * 2, "blocks of a step spread over a group");

// Tile shapes: TOK token rows per tile; S slots of the token ring and of the
// converted-weight ring (freed together by the MMA), PS slots of the packed-weight
// ring (freed by the converters as soon as they have read a slot).  Two TMEM
// accumulators of max(TOK, 32) fp32 columns each let the epilogue of one tile
// overlap the MMAs of the next.
template <int TOK_, int S_, int PS_>
struct Config {
    static constexpr int TOK = TOK_;
    static constexpr int S = S_;
    static constexpr int PS = PS_;
    static constexpr int NACC = 2;
    static constexpr uint32_t ACC_STRIDE = TOK < 32 ? 32 : TOK;
    static constexpr uint32_t X_BYTES = TOK * BK * 2;
    static constexpr uint32_t OFF_WB = 0;                       // S x 16 KB converted weights
    static constexpr uint32_t OFF_X = OFF_WB + S * WB_BYTES;    // S x tokens
    static constexpr uint32_t OFF_WP = OFF_X + S * X_BYTES;     // PS x 4 KB packed weights
    static constexpr uint32_t OFF_EPI = OFF_WP + PS * WP_BYTES; // epilogue staging, 4 KB / warp
    // the tile offsets (E <= 256) staged per CTA for the item -> expert search
    static constexpr uint32_t OFF_TOFF = OFF_EPI + 4096 * kEpiWarps;
    static constexpr uint32_t OFF_BAR = (OFF_TOFF + 4 * 257 + 15u) & ~15u;   // mbarriers: 8-byte aligned
    static_assert(OFF_BAR % 16 == 0, "barrier alignment");
    static constexpr uint32_t BAR_BYTES = 8 * (2 * S + 2 * PS + 2 * NACC) + 16;
    // + slack for aligning the base to 1 KB
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
    static_assert(X_BYTES % 1024 == 0, "1 KB aligned stages");
    // a ring slot is only ever used by one converter group, so that the parity
    // waits and the per-group arrival counts never mix two groups' steps
    static_assert(S % kConvGroups == 0 && PS % kConvGroups == 0, "rings split over groups");
    static_assert(NACC * ACC_STRIDE <= TMEM_COLS, "TMEM columns");
    static_assert(TOK % 32 == 0 && TOK <= 256, "token tile");
    __host__ __device__ static constexpr uint32_t smem_bytes(int /*kblocks*/) { return SMEM_BYTES; }
};
using PrefillCfg = Config<256, 4, 4>;
using DecodeCfg = Config<32, 8, 8>;

struct Params {
    const int32_t *counts;        // [E]
    const int32_t *offsets;       // [E + 1]
    const int32_t *tile_offsets;  // [E + 1] in TOK-row token tiles
    const uint8_t *wscales;       // E8M0 [E, N, K/32] (MXFP4) or E4M3 [E, N, K/16] (NVFP4)
    const float *bias;            // [E, N] or null
    const float *scale2;          // NVFP4 weight_scale_2: gate_up [E, 2] (gate, up), down [E]; or null
    int E, N, K;
    int rows_cap;                 // rows of the A, act and yp buffers (bounds-checked builds)
    // gate_up epilogue
    uint16_t *act;                // [rows, N/2] bf16
    float alpha, limit;
    // down epilogue
    float *yp;                    // [T*k, N] fp32, indexed by pair
    const int32_t *sorted_pairs;  // [rows]
    const float *weights;         // [T*k]
    int weight_on_input;
};

// s_toff: the tile offsets staged in shared memory
__device__ __forceinline__ int tile_expert(const int *s_toff, int E, int m) {
    int lo = 0, hi = E - 1;  // largest e with tile_offsets[e] <= m
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_toff[mid] <= m)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

struct Tile {
    int e;       // expert
    int row0;    // first expert-ordered row (token slot) of the token tile
    int ntok;    // token rows in the tile (1..TOK)
    int m0;      // first weight row
    int mrows;   // weight rows in range (64 or 128)
};

// Work item -> tile.  Items enumerate (token tile, weight tile) with the weight
// tile fastest, so the CTAs running at one time share token tiles through L2.
template <int TOK>
__device__ __forceinline__ Tile decode_tile(const Params &p, const int *s_toff, int item, int w_tiles) {
    Tile t;
    const int g = item / w_tiles;
    const int wt = item - g * w_tiles;
    t.e = tile_expert(s_toff, p.E, g);
    const int tt = g - s_toff[t.e];
    t.row0 = __ldg(p.offsets + t.e) + tt * TOK;
    t.ntok = min(TOK, __ldg(p.counts + t.e) - tt * TOK);
    t.m0 = wt * BM;
    t.mrows = min(BM, p.N - t.m0);
    // bounds-checked builds report an inconsistent schedule (the stores below are checked)
    range_in_bounds(t.row0, (int64_t)t.row0 + t.ntok, p.rows_cap);
    in_bounds(t.e, p.E);
    return t;
}

// Eight E2M1 codes -> four bf16x2 words holding E2M1(code) * 2^-126 (see the
// converter below); element order is natural (word j = elements 2j, 2j + 1).
__device__ __forceinline__ void e2m1x8_to_bf16_rep(uint32_t q, uint32_t &r0, uint32_t &r1,
                                                   uint32_t &r2, uint32_t &r3) {
    const uint32_t lo = q & 0x0F0F0F0Fu;          // even elements, one per byte
    const uint32_t hi = (q >> 4) & 0x0F0F0F0Fu;   // odd elements
    r0 = (ptx::prmt(lo, hi, 0x8480u) * 0x1040u) & 0x81C081C0u;
    r1 = (ptx::prmt(lo, hi, 0x8581u) * 0x1040u) & 0x81C081C0u;
    r2 = (ptx::prmt(lo, hi, 0x8682u) * 0x1040u) & 0x81C081C0u;
    r3 = (ptx::prmt(lo, hi, 0x8783u) * 0x1040u) & 0x81C081C0u;
}

// An E4M3 scale byte as a bf16 pair (exact: 4 significant bits, exponents within
// bf16's normal range); S.1111.111 is NaN and flags the device error word.
__device__ __forceinline__ uint32_t e4m3_to_bf16x2(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u, sign = (b & 0x80u) << 8;
    uint32_t h;
    if (e == 15u && m == 7u) {
        raise_device_error(MOE_DEVERR_BAD_SCALE);
        h = 0x7FC0u;
    } else if (e) {
        h = sign | ((e + 120u) << 7) | (m << 4);
    } else {
        h = sign | (__float_as_uint((float)m * 0x1p-9f) >> 16);   // subnormal m/8 * 2^-6
    }
    return h * 0x10001u;
}

// The epilogue of one work item, run by the four epilogue warps: TMEM accumulator
// columns [acc, acc + ntok) of lane quarter q (weight rows 32 q .. 32 q + 31 of the
// tile) -> the act rows (gate_up: bias, gate/up pairing, clamped SwiGLU, bf16) or
// the yp rows (down: bias, routing weight, fp32).  stg is this warp's 4 KB of
// shared-memory staging.
template <int TOK, bool kGateUp, bool kNv>
__device__ __forceinline__ void epilogue_tile(const Params &p, const Tile &t, uint32_t acc, uint8_t *stg_bytes,
                                              int q, int lane) {
    const int r = q * 32 + lane;             // weight row within the tile
    const bool row_ok = r < t.mrows;
    const int n = t.m0 + r;                             // output feature of this thread
    const float bias = (p.bias && row_ok) ? __ldg(p.bias + (int64_t)t.e * p.N + n) : 0.0f;
    // NVFP4 weight_scale_2 of this row (gate rows are even), applied before the bias;
    // the down projection's is one per expert and is loaded per chunk below
    const float rs = (kNv && kGateUp && p.scale2 && row_ok) ? __ldg(p.scale2 + 2 * t.e + (n & 1)) : 1.0f;
    // down: lane i holds the pair index and routing weight of token 32 j + i
    int pairs[TOK / 32];
    float wts[TOK / 32];
    if (!kGateUp) {
#pragma unroll
        for (int j = 0; j < TOK / 32; ++j) {
            const int tok = 32 * j + lane;
            pairs[j] = (tok < t.ntok && in_bounds(t.row0 + tok, p.rows_cap)) ? __ldg(p.sorted_pairs + t.row0 + tok) : 0;
            wts[j] = (tok < t.ntok && !p.weight_on_input) ? __ldg(p.weights + pairs[j]) : 1.0f;
        }
    }
    for (int c0 = 0; c0 < t.ntok; c0 += 32) {
        const uint32_t taddr = acc + c0 + ((uint32_t)(q * 32) << 16);
        uint32_t v[32];
        if (kGateUp || !kNv) {
            ptx::tmem_ld_32x32b_x32(taddr, v);
            ptx::tmem_ld_wait();
        }
        const int nvalid = min(32, t.ntok - c0);
        if (kGateUp) {
            // lanes 2i (gate row) and 2i+1 (up row) hold one output feature; the
            // even lane finishes tokens 0..15 of the chunk, the odd lane 16..31.
            // The warp's 16 features x 32 tokens go through a 1 KB staging tile
            // so that every lane then stores whole 16-byte pieces of act rows.
            const bool odd = lane & 1;
            const float pb = __shfl_xor_sync(0xFFFFFFFFu, bias, 1);
            const float bg = odd ? pb : bias, bu = odd ? bias : pb;
            uint16_t *stg = reinterpret_cast<uint16_t *>(stg_bytes);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float lo_v = rs * __uint_as_float(v[i]), hi_v = rs * __uint_as_float(v[16 + i]);
                const float mine = odd ? hi_v : lo_v;
                const float other = __shfl_xor_sync(0xFFFFFFFFu, odd ? lo_v : hi_v, 1);
                const float gate = (odd ? other : mine) + bg;
                const float up = (odd ? mine : other) + bu;
                const float a = clamped_swiglu(gate, up, p.alpha, p.limit);
                stg[(odd ? 16 + i : i) * 16 + (lane >> 1)] = (uint16_t)(pack_bf16x2(a, 0.0f) & 0xFFFFu);
            }
            __syncwarp();
            const int64_t fbase = (t.m0 + 32 * q) >> 1;     // first feature of the warp
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int piece = lane + 32 * h;            // 64 pieces of 16 bytes
                const int tok = piece >> 1;
                if (tok < nvalid && in_bounds(t.row0 + c0 + tok, p.rows_cap) &&
                    range_in_bounds(fbase + (piece & 1) * 8, fbase + (piece & 1) * 8 + 8, p.N / 2)) {
                    const uint4 val = *reinterpret_cast<const uint4 *>(stg + tok * 16 + (piece & 1) * 8);
                    *reinterpret_cast<uint4 *>(p.act + (int64_t)(t.row0 + c0 + tok) * (p.N / 2) +
                                               fbase + (piece & 1) * 8) = val;
                }
            }
            __syncwarp();
        } else {
            // w * (acc + bias) for 32 tokens x the warp's 32 features, staged
            // so that each pair's row segment leaves as 16-byte stores
            float *stg = reinterpret_cast<float *>(stg_bytes);
            if constexpr (kNv) {
                // w * (s * acc + bias), s the expert's down weight_scale_2; the
                // accumulator comes in two 16-column pieces (register budget)
                const float ds = p.scale2 ? __ldg(p.scale2 + t.e) : 1.0f;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t u[16];
                    ptx::tmem_ld_32x32b_x16(taddr + 16u * hf, u);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float wi = __shfl_sync(0xFFFFFFFFu, wts[c0 >> 5], 16 * hf + i);
                        stg[(16 * hf + i) * 32 + lane] = wi * fmaf(ds, __uint_as_float(u[i]), bias);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float wi = __shfl_sync(0xFFFFFFFFu, wts[c0 >> 5], i);
                    stg[i * 32 + lane] = wi * (__uint_as_float(v[i]) + bias);
                }
            }
            __syncwarp();
            if (32 * q < t.mrows) {                      // warp-uniform
#pragma unroll
                for (int rd = 0; rd < 8; ++rd) {
                    const int piece = rd * 32 + lane;    // 32 tokens x 8 pieces of 16 B
                    const int tok = piece >> 3, part = piece & 7;
                    const int pi = __shfl_sync(0xFFFFFFFFu, pairs[c0 >> 5], tok);
                    if (tok < nvalid && in_bounds(pi, p.rows_cap) &&
                        range_in_bounds(t.m0 + 32 * q + part * 4, t.m0 + 32 * q + part * 4 + 4, p.N)) {
                        const float4 val = *reinterpret_cast<const float4 *>(stg + tok * 32 + part * 4);
                        *reinterpret_cast<float4 *>(p.yp + (int64_t)pi * p.N + t.m0 + 32 * q + part * 4) = val;
                    }
                }
            }
            __syncwarp();
        }
    }
}

template <class Cfg, bool kGateUp, bool kNv = false>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_mxfp4_swap_kernel(const __grid_constant__ CUtensorMap tmap_x,
                              const __grid_constant__ CUtensorMap tmap_w, const Params p) {
    constexpr int TOK = Cfg::TOK, S = Cfg::S, PS = Cfg::PS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const gbase = smem_raw + (base - raw);
    auto wb_stage = [&](int c) { return base + Cfg::OFF_WB + c * WB_BYTES; };
    auto x_stage = [&](int s) { return base + Cfg::OFF_X + s * Cfg::X_BYTES; };
    auto wp_stage = [&](int s) { return base + Cfg::OFF_WP + s * WP_BYTES; };
    const int kblocks = p.K / 32;
    const uint32_t bars = base + Cfg::OFF_BAR;
    // ready(s): the token tile landed (producer arrival + transaction bytes) and
    // every converter warp of the step's group stored its weights
    auto ready = [&](int s) { return bars + 8u * s; };
    auto empty = [&](int s) { return bars + 8u * (S + s); };   // MMA done with slot s
    auto wp_full = [&](int s) { return bars + 8u * (2 * S + s); };
    auto wp_empty = [&](int s) { return bars + 8u * (2 * S + PS + s); };
    auto a_full = [&](int b) { return bars + 8u * (2 * S + 2 * PS + b); };
    auto a_empty = [&](int b) { return bars + 8u * (2 * S + 2 * PS + Cfg::NACC + b); };
    const uint32_t tmem_holder = bars + 8u * (2 * S + 2 * PS + 2 * Cfg::NACC);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(ready(s), 1 + kConvWarps / kConvGroups);
            ptx::mbar_init(empty(s), 1);
        }
        for (int s = 0; s < PS; ++s) {
            ptx::mbar_init(wp_full(s), 1);
            ptx::mbar_init(wp_empty(s), kConvWarps / kConvGroups);
        }
        for (int b = 0; b < Cfg::NACC; ++b) {
            ptx::mbar_init(a_full(b), 1);
            ptx::mbar_init(a_empty(b), kEpiWarps);
        }
        ptx::fence_mbarrier_init();
        ptx::prefetch_tmap(&tmap_x);
        ptx::prefetch_tmap(&tmap_w);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    // barriers and TMEM are set up; wait for the producer of this kernel's inputs, then
    // stage the tile offsets it wrote
    pdl_wait();
    pdl_trigger();
    int *const s_toff = reinterpret_cast<int *>(gbase + Cfg::OFF_TOFF);
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) s_toff[i] = __ldg(p.tile_offsets + i);
    __syncthreads();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(gbase + (tmem_holder - base));

    const int w_tiles = (p.N + BM - 1) / BM;
    const int total = s_toff[p.E] * w_tiles;
    const int k_iters = p.K / BK;

    if (warp == 0) {
        // ------------------------------------------------------------ token TMA
        // The whole warp runs the loop (uniform control flow keeps the operands in
        // uniform registers); one elected lane issues the asynchronous copies.
        uint32_t it = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const Tile t = decode_tile<TOK>(p, s_toff, item, w_tiles);
            const int nbox = (t.ntok + (int)XBOX_ROWS - 1) / (int)XBOX_ROWS;
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int s = it % S;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(empty(s), ((it / S) & 1u) ^ 1u)))) break;
                if (ptx::elect_one()) {
                    ptx::mbar_arrive_expect_tx(ready(s), nbox * XBOX_BYTES);
                    for (int b = 0; b < nbox; ++b)
                        ptx::tma_load_2d(x_stage(s) + b * XBOX_BYTES, &tmap_x, kb * BK,
                                         t.row0 + b * (int)XBOX_ROWS, ready(s));
                }
                __syncwarp();
            }
        }
    } else if (warp == kWpWarp) {
        // ------------------------------------------------------------ packed-weight TMA
        uint32_t it = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const Tile t = decode_tile<TOK>(p, s_toff, item, w_tiles);
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int s = it % PS;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(wp_empty(s), ((it / PS) & 1u) ^ 1u)))) break;
                if (ptx::elect_one()) {
                    ptx::mbar_arrive_expect_tx(wp_full(s), WP_BYTES);
                    ptx::tma_load_3d(wp_stage(s), &tmap_w, kb * (BK / 2), t.m0, t.e, wp_full(s));
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Warp-wide loop, one elected lane issues the MMAs and commits.
        uint32_t it = 0, local = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++local) {
            const Tile t = decode_tile<TOK>(p, s_toff, item, w_tiles);
            const int nmma = max(16, (t.ntok + 15) & ~15);
            const uint32_t idesc = ptx::idesc_bf16_f32(BM, nmma);
            const int b = local % Cfg::NACC;
            const uint32_t use = local / Cfg::NACC;
            if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(a_empty(b), (use & 1u) ^ 1u)))) break;
            ptx::tc_fence_after();
            const uint32_t d_tmem = tmem_base + b * Cfg::ACC_STRIDE;
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int s = it % S;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(ready(s), (it / S) & 1u)))) break;
                ptx::tc_fence_after();
                const uint64_t bd = ptx::sw128_kmajor_desc(x_stage(s));
                if (ptx::elect_one()) {
                    const uint64_t ad = ptx::sw128_kmajor_desc(wb_stage(s));
#pragma unroll
                    for (int j = 0; j < BK / 16; ++j)   // +32 B per 16-element K step (start address >> 4)
                        ptx::mma_bf16(d_tmem, ad + 2u * j, bd + 2u * j, idesc, (kb > 0 || j > 0) ? 1u : 0u);
                    ptx::mma_commit(empty(s));
                }
                __syncwarp();
            }
            if (ok && ptx::elect_one()) ptx::mma_commit(a_full(b));
            __syncwarp();
        }
    } else if (warp < kFirstConvWarp) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        uint32_t local = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x, ++local) {
            const Tile t = decode_tile<TOK>(p, s_toff, item, w_tiles);
            const int b = local % Cfg::NACC;
            if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(a_full(b), (local / Cfg::NACC) & 1u))) break;
            ptx::tc_fence_after();
            epilogue_tile<TOK, kGateUp, kNv>(p, t, tmem_base + b * Cfg::ACC_STRIDE,
                                             gbase + Cfg::OFF_EPI + 4096 * q, q, lane);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(a_empty(b));
        }
    } else {
        // ------------------------------------------------------------ converters
        // Each thread turns kBlocksPerThread 32-element blocks (16 bytes of codes
        // each) of the step's weight rows into bf16: the codes become E2M1 * 2^-126
        // bit patterns (sign to bit 15, exponent bits and mantissa msb to bits 8..6;
        // code 1 = 0.5 is the bf16 subnormal 2^-127), then one bf16 multiply by
        // 2^(s-1) (two, by 2^126 and 2^(s-127), when 2^(s-1) is not a bf16) gives
        // E2M1 * 2^(s-127) exactly; the result goes to the 128-byte swizzled
        // K-major layout the MMA reads.  The E8M0 bytes a thread needs for its
        // group's next step are loaded from global memory one step ahead, and the
        // next step is converted into registers while the MMA still reads the slot.
        // NVFP4: a block's two E4M3 bytes (one per 16 elements) come as one 16-bit
        // load; the codes are multiplied by 2^126 (exact E2M1) and then by the
        // E4M3 scale of their half as a bf16 (exact products).
        const int ct = threadIdx.x - 32 * kFirstConvWarp;
        const int grp = ct / kGroupThreads;
        const int gt = ct % kGroupThreads;                    // thread within its group
        uint32_t it = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const Tile t = decode_tile<TOK>(p, s_toff, item, w_tiles);
            const uint8_t *srow[kBlocksPerThread];
            bool rok[kBlocksPerThread];
#pragma unroll
            for (int bi = 0; bi < kBlocksPerThread; ++bi) {
                const int blkid = gt + bi * kGroupThreads;
                const int row = blkid >> 1;
                rok[bi] = row < t.mrows;
                srow[bi] = kNv ? p.wscales + ((int64_t)t.e * p.N + t.m0 + (rok[bi] ? row : 0)) * (2 * kblocks) +
                                     2 * (blkid & 1)
                               : p.wscales + ((int64_t)t.e * p.N + t.m0 + (rok[bi] ? row : 0)) * kblocks + (blkid & 1);
            }
            // scale bits of block bi at step kbi (a block past the tile's rows reads 1.0)
            constexpr uint32_t kOne = kNv ? 0x3838u : 127u;
            auto load_sc = [&](int bi, int kbi) -> uint32_t {
                if constexpr (kNv)
                    return (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(srow[bi] + 4 * kbi));
                else
                    return (uint32_t)__ldg(srow[bi] + 2 * kbi);
            };
            // first step of this tile that belongs to this group
            int kb = (int)((grp - (int)(it % kConvGroups) + kConvGroups) % kConvGroups);
            uint32_t nxt[kBlocksPerThread];     // scale bits of the next step to decode
#pragma unroll
            for (int bi = 0; bi < kBlocksPerThread; ++bi)
                nxt[bi] = (rok[bi] && kb < k_iters) ? load_sc(bi, kb) : kOne;
            // The group's steps are software-pipelined: step kb + kConvGroups is decoded
            // into registers as soon as step kb is stored, so that once a stage slot is
            // free only the stores remain.
            uint32_t cv[kBlocksPerThread][16];
            auto decode_step = [&](int kbi) -> bool {
                const uint32_t gix = it + (uint32_t)kbi;
                const int ps = gix % PS;
                if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(wp_full(ps), (gix / PS) & 1u))) return false;
#pragma unroll
                for (int bi = 0; bi < kBlocksPerThread; ++bi) {
                    const int blkid = gt + bi * kGroupThreads;
                    const uint4 q4 = ptx::ld_shared_v4(wp_stage(ps) + (blkid >> 1) * 32 + (blkid & 1) * 16);
                    const uint32_t sc = nxt[bi];
                    uint32_t m1, m2 = 0, m2b = 0;   // m2: words 0-1 (first 16 elements), m2b: words 2-3
                    if (kNv) {
                        m1 = 0x7E807E80u;
                        m2 = e4m3_to_bf16x2(sc & 0xFFu);
                        m2b = e4m3_to_bf16x2(sc >> 8);
                    } else if (sc == 255u) {
                        raise_device_error(MOE_DEVERR_BAD_SCALE);
                        m1 = 0x7FC07FC0u;
                    } else if (sc <= 128u) {
                        m1 = ((sc + 126u) << 7) * 0x10001u;
                    } else {
                        m1 = 0x7E807E80u;
                        m2 = (sc << 7) * 0x10001u;
                    }
                    if (!kNv) m2b = m2;
                    const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint32_t r0, r1, r2, r3;
                        e2m1x8_to_bf16_rep(qw[w], r0, r1, r2, r3);
                        r0 = ptx::hmul2_bf16(r0, m1);
                        r1 = ptx::hmul2_bf16(r1, m1);
                        r2 = ptx::hmul2_bf16(r2, m1);
                        r3 = ptx::hmul2_bf16(r3, m1);
                        const uint32_t mw = w < 2 ? m2 : m2b;
                        if (kNv || mw) {
                            r0 = ptx::hmul2_bf16(r0, mw);
                            r1 = ptx::hmul2_bf16(r1, mw);
                            r2 = ptx::hmul2_bf16(r2, mw);
                            r3 = ptx::hmul2_bf16(r3, mw);
                        }
                        cv[bi][4 * w] = r0;
                        cv[bi][4 * w + 1] = r1;
                        cv[bi][4 * w + 2] = r2;
                        cv[bi][4 * w + 3] = r3;
                    }
                }
                // every lane has consumed its packed words, so the TMA may refill the slot
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(wp_empty(ps));
#pragma unroll
                for (int bi = 0; bi < kBlocksPerThread; ++bi)
                    nxt[bi] = (rok[bi] && kbi + kConvGroups < k_iters) ? load_sc(bi, kbi + kConvGroups) : kOne;
                return true;
            };
            if (kb < k_iters) ok = decode_step(kb);
            for (; kb < k_iters && ok; kb += kConvGroups) {
                const uint32_t gi = it + (uint32_t)kb;         // global step index
                const int c = gi % S;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(empty(c), ((gi / S) & 1u) ^ 1u)))) break;
#pragma unroll
                for (int bi = 0; bi < kBlocksPerThread; ++bi) {
                    const int blkid = gt + bi * kGroupThreads;    // 0 .. 255 within the step
                    const int row = blkid >> 1, blk = blkid & 1;
                    const uint32_t dst_row = wb_stage(c) + row * 128;
                    const uint32_t sw = (uint32_t)(row & 7);
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t chunk = (uint32_t)(blk * 4 + w);
                        ptx::st_shared_v4(dst_row + ((chunk ^ sw) << 4), cv[bi][4 * w], cv[bi][4 * w + 1],
                                          cv[bi][4 * w + 2], cv[bi][4 * w + 3]);
                    }
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ready(c));
                if (kb + kConvGroups < k_iters) ok = decode_step(kb + kConvGroups);
            }
            it += (uint32_t)k_iters;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace swp
}  // namespace moe
