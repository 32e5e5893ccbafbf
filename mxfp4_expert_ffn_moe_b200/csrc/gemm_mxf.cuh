// gemm_mxf.cuh -- grouped MXFP4 expert GEMM on the sm_100a block-scaled tensor-core
// path (tcgen05.mma kind::mxf8f6f4): the tensor core reads the E2M1 weight codes and
// their E8M0 block scales directly, against activations split exactly into two E4M3
// terms (split.cuh).
//
// For every (expert e, token tile of up to TOK rows of that expert, 128-row weight
// tile) of a projection, with h = ntok rounded up to 16:
//   B rows 0 .. h-1   = hi terms of the tile's token rows, B rows h .. 2h-1 = lo terms
//   D[n, j] = sum_k W[e, m0 + n, k] * 2^(sw[n, k/32] - 127) * B[j, k] * 2^(sb[j, k/32] - 127)
//   acc[n, t] = D[n, t] + D[n, h + t]                       (fp32)
// i.e. acc = W_dequant x A^T with A the bf16 rows of the tile, then
//   gate_up epilogue: h = acc + b_gu[e]; gate = h[2i], up = h[2i+1] (adjacent lanes);
//                     act[row, i] = bf16(clamped SwiGLU(gate, up)), written split
//                     (two E4M3 terms + E8M0 bytes) as the second projection's B
//   down epilogue:    yp[p, n] = w[p] * (acc + b_d[e])   (router weight on output)
//                     yp[p, n] = acc                     (router weight on input)
// (MoE-Infinity PR #152, Changes: dequant-on-copy of fetched packed experts,
// [N, K//2] layout, E8M0 scales per 32 elements, bias, gate/up split, clamped
// SwiGLU, fp32 accumulate; FreeToken PR #838: gate_up bias before the gated
// activation, down bias before the routing weight, sum w*(y + b).)
//
// The MXF8F6F4 operand layout keeps 4-bit codes "unpacked" in shared memory: each
// 16-byte chunk of a K-major row holds 16 codes in its first 8 bytes (element 2j in
// the low nibble of byte j, as in the packed global layout) and 8 unused bytes, so a
// 128-element K step is one 128-byte row of the usual 128-byte-swizzled layout.
// Scale factors live in tensor memory, one 32-bit column per 32 rows (replicated in
// all four lane quarters); byte j of a column is the scale of the step's K block j,
// selected by the scale-factor ids of the instruction descriptor.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0           token TMA: per K step the hi and lo rows of the token tile
//                    (16-row boxes of the [2][P][K] code bytes, 128-byte swizzle)
//                    and the rows' 16-byte scale slots of the step
//   warp 1           TMEM owner and MMA issuer (4 x 128 x 2h x 32 per K step)
//   warps 2..5       epilogue (TMEM lane quarter = warp % 4)
//   warps 6..6+4G-1  stagers in G groups of four (one per lane quarter); group g
//                    takes the steps with index % G == g: it spreads the step's
//                    packed codes into the unpacked layout and writes the step's
//                    weight and token scale words into tensor memory
//   last warp        packed-weight TMA (128 rows x 128 B = two K steps, 128-byte
//                    swizzle; a full line per row keeps the copy engine's request
//                    count per byte low) and the tile's scale rows (one bulk copy
//                    per tile)
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "split.cuh"

namespace moe {
namespace mxf {

constexpr int BM = 128;                          // weight rows per tile (TMEM lanes)
constexpr int BK = 128;                          // K elements per step
constexpr int KBS = BK / 32;                     // scale blocks per step
#ifndef MOE_MXF_WP_STEPS
#define MOE_MXF_WP_STEPS 2
#endif
// K steps per packed-weight load: 2 (128-byte rows, 128-byte swizzle) or 4 (256-byte
// rows, unswizzled; stagers read a row's chunks in a lane-rotated order)
constexpr int WP_STEPS = MOE_MXF_WP_STEPS;
static_assert(WP_STEPS == 2 || WP_STEPS == 4, "two or four K steps per packed load");
constexpr uint32_t WP_ROW = WP_STEPS * BK / 2;   // packed bytes per weight row and load
constexpr bool WP_SWIZZLED = WP_ROW == 128;
constexpr uint32_t WP_BYTES = BM * WP_ROW;       // packed codes of a load
constexpr uint32_t WA_BYTES = BM * BK;           // unpacked codes of a step
constexpr int XBOX_ROWS = 16;                    // token rows per TMA box
constexpr uint32_t XBOX_BYTES = XBOX_ROWS * BK;  // one E4M3 term of 16 rows
constexpr int kEpiWarps = 4;
constexpr int kFirstStageWarp = 2 + kEpiWarps;
constexpr uint32_t kEpiStage = 2048;             // staging bytes per epilogue warp
constexpr uint32_t kXchBytes = 2 * 4 * 32 * 4;   // per-token block maxima exchanged by warp pairs
constexpr uint32_t kSinkBytes = 128;             // scratch words (see ptx::sink_shared)

// TOK token rows per tile (B has 2 TOK rows: hi and lo terms); S slots of the
// unpacked-weight / token / scale-factor rings (freed together by the MMA); PS slots
// of the packed-weight ring (two K steps each, freed by the stagers of both steps);
// NACC accumulators; G stager groups.
template <int TOK_, int S_, int PS_, int NACC_, int G_>
struct Config {
    static constexpr int TOK = TOK_;
    static constexpr int S = S_;
    static constexpr int PS = PS_;
    static constexpr int NACC = NACC_;
    static constexpr int G = G_;
    static constexpr int NB = 2 * TOK;                      // B rows at most
    static constexpr int NCB = NB / 32;                     // token scale columns
    static constexpr uint32_t ACC_COLS = NB;                // fp32 columns per accumulator
    static constexpr uint32_t SF_STRIDE = (4 + NCB + 3) & ~3u;   // weight (4) + token scale columns
    static constexpr uint32_t SF_COL0 = NACC * ACC_COLS;
    static constexpr uint32_t TMEM_USED = SF_COL0 + S * SF_STRIDE;
    static constexpr uint32_t TMEM_COLS = TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
    static constexpr int kStageWarps = 4 * G;
    static constexpr int kWpWarp = kFirstStageWarp + kStageWarps;
    static constexpr int kThreads = 32 * (kWpWarp + 1);
    static constexpr uint32_t X_DATA = NB * BK;             // code bytes of B
    static constexpr uint32_t X_BYTES = X_DATA + NB * 16;   // + one 16-byte scale slot per B row
    static constexpr uint32_t OFF_A = 0;
    static constexpr uint32_t OFF_X = OFF_A + S * WA_BYTES;
    static constexpr uint32_t OFF_WP = OFF_X + S * X_BYTES;
    static constexpr uint32_t OFF_EPI = OFF_WP + PS * WP_BYTES;
    static constexpr uint32_t OFF_XCH = OFF_EPI + kEpiStage * kEpiWarps;
    static constexpr uint32_t OFF_SINK = OFF_XCH + kXchBytes;
    // the tile schedule (counts, row offsets, tile offsets; E <= 256) staged per CTA
    static constexpr uint32_t OFF_SCHED = OFF_SINK + kSinkBytes;
    static constexpr uint32_t OFF_BAR = (OFF_SCHED + 3 * 4 * 257 + 15u) & ~15u;   // mbarriers: 8-byte aligned
    static_assert(OFF_BAR % 16 == 0, "barrier alignment");
    static constexpr uint32_t BAR_BYTES = 8 * (3 * S + 2 * PS + 2 * NACC + 6) + 16;
    static constexpr uint32_t OFF_SC = (OFF_BAR + BAR_BYTES + 127u) & ~127u;
    static constexpr uint32_t SMEM_FIXED = OFF_SC + 1024;   // + slack for the 1 KB base alignment
    static_assert(TOK % 32 == 0 && TOK <= 128, "token tile: B rows <= 256");
    static_assert(S % G == 0, "a ring slot belongs to one stager group");
    // A stager group may only wait on a packed slot whose previous load it also read
    // (an mbarrier parity wait cannot tell a phase from the one two phases later), so
    // the set of groups reading a packed slot must not change from load to load: the
    // groups read consecutive loads in a fixed rotation of G / WP_STEPS loads, and
    // tiles run a multiple of KALIGN steps.
    static_assert(G <= WP_STEPS ? WP_STEPS % G == 0 : (G % WP_STEPS == 0 && PS % (G / WP_STEPS) == 0),
                  "packed slots read by a fixed set of stager groups");
    static constexpr int KALIGN = G > WP_STEPS ? G : WP_STEPS;
    static_assert(NACC == 1 || NACC == 2, "one or two accumulators");
    static_assert(TMEM_USED <= 512, "TMEM columns");
    static_assert(X_BYTES % 1024 == 0 && WP_BYTES % 1024 == 0, "1 KB aligned stages");
    __host__ __device__ static constexpr uint32_t sc_slot_bytes(int kblocks) {
        return ((uint32_t)(BM * kblocks) + 127u) & ~127u;
    }
    __host__ __device__ static constexpr uint32_t smem_bytes(int kblocks) {
        return SMEM_FIXED + 2 * sc_slot_bytes(kblocks);
    }
};

struct Params {
    const int32_t *counts;        // [E]
    const int32_t *offsets;       // [E + 1]
    const int32_t *tile_offsets;  // [E + 1] in TOK-row token tiles
    const uint8_t *wscales;       // [E, N, K/32] E8M0
    const float *bias;            // [E, N] or null
    int E, N, K, P;
    // gate_up epilogue: the activation, split (split_rows_kernel's layout with K = N/2),
    // as the next projection's B
    uint8_t *actq;                // [2][P][split_row_bytes(N/2)]
    float alpha, limit;
    // down epilogue
    float *yp;                    // [T*k, N] fp32, indexed by pair
    const int32_t *sorted_pairs;  // [rows]
    const float *weights;         // [T*k]
    int weight_on_input;
};

// The schedule a CTA stages in shared memory once, so that each role decodes its
// work items without dependent global loads.
struct Sched {
    const int *counts, *offsets, *tile_offsets;
};

__device__ __forceinline__ int tile_expert(const int *tile_offsets, int E, int m) {
    int lo = 0, hi = E - 1;  // largest e with tile_offsets[e] <= m
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_offsets[mid] <= m)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

struct Tile {
    int e;       // expert
    int row0;    // first expert-ordered row of the token tile
    int ntok;    // token rows in the tile (1..TOK)
    int h;       // ntok rounded up to 16: first B row of the lo terms
    int m0;      // first weight row
    int mrows;   // weight rows in range
};

// Work item -> tile; the weight tile index runs fastest, so the CTAs running at one
// time share token tiles through L2.
template <int TOK>
__device__ __forceinline__ Tile decode_tile(const Params &p, const Sched &sc, int item, int w_tiles) {
    Tile t;
    const int g = item / w_tiles;
    const int wt = item - g * w_tiles;
    t.e = tile_expert(sc.tile_offsets, p.E, g);
    const int tt = g - sc.tile_offsets[t.e];
    t.row0 = sc.offsets[t.e] + tt * TOK;
    t.ntok = min(TOK, sc.counts[t.e] - tt * TOK);
    t.h = (t.ntok + 15) & ~15;
    t.m0 = wt * BM;
    t.mrows = min(BM, p.N - t.m0);
    // bounds-checked builds report an inconsistent schedule (the stores below are checked)
    range_in_bounds(t.row0, (int64_t)t.row0 + t.ntok, p.P);
    in_bounds(t.e, p.E);
    return t;
}

// Instruction descriptor, kind::mxf8f6f4 with E8M0 block scales: A E2M1, B E4M3,
// both K-major, fp32 D, shape M x N; sf_id (bits 29-30 for A, 4-5 for B) added per MMA.
__host__ __device__ constexpr uint32_t idesc_e2m1_e4m3(int M, int N) {
    return (5u << 7)                      // A format E2M1
           | (0u << 10)                   // B format E4M3
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | (1u << 23)                   // scale format E8M0
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// Bytes of `w` for K blocks at or past `kblocks` (block index kb0 + j in byte j)
// become 127 (scale 1 for the zero-filled padding of the last step).
__device__ __forceinline__ uint32_t mask_pad_blocks(uint32_t w, int kb0, int kblocks) {
    const int valid = kblocks - kb0;
    if (valid >= 4) return w;
    const uint32_t keep = valid <= 0 ? 0u : (0xFFFFFFFFu >> (8 * (4 - valid)));
    return (w & keep) | (0x7F7F7F7Fu & ~keep);
}

// The epilogue of one decode work item, run by the four epilogue warps: accumulator
// columns acc + [0, h) (hi terms) and acc + [h, 2h) (lo terms) of this warp's TMEM lane
// quarter q -> the gate_up activation, written split as the next projection's B (block
// maxima shared with the partner warp of the 32-feature block through `xch` and the
// bounded barrier `xbar`), or the down rows of yp.  stg_bytes: this warp's 2 KB of
// staging; `chunk` counts the warp's 32-token chunks (the exchange buffers alternate).
// Returns false when a wait timed out.
template <bool kGateUp>
__device__ __forceinline__ bool epilogue_item(const Params &p, const Tile &t, uint32_t acc, uint8_t *stg_bytes,
                                              float *xch, uint32_t xbar, uint32_t &chunk, int q, int lane) {
    const int r = q * 32 + lane;             // weight row within the tile
    bool ok = true;
    const bool row_ok = r < t.mrows;
    const int n = t.m0 + r;
    const float bias = (p.bias && row_ok) ? __ldg(p.bias + (int64_t)t.e * p.N + n) : 0.0f;
        for (int c0 = 0; c0 < t.ntok; c0 += 32, ++chunk) {
        // hi-term columns, then the lo-term columns added in two pieces of 16
        // (keeps the live registers at 48)
        uint32_t vh[32];
        ptx::tmem_ld_32x32b_x32(acc + c0, vh);
        ptx::tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(vh[i]);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            uint32_t vl[16];
            ptx::tmem_ld_32x32b_x16(acc + t.h + c0 + 16 * hf, vl);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[16 * hf + i] += __uint_as_float(vl[i]);
        }
        const int nvalid = min(32, t.ntok - c0);
        if (kGateUp) {
            // lanes 2i (gate row) and 2i+1 (up row) hold one output feature; the
            // even lane finishes tokens 0..15 of the chunk, the odd lane 16..31,
            // into a bf16 staging tile [token][16 features]
            const bool odd = lane & 1;
            const float pb = __shfl_xor_sync(0xFFFFFFFFu, bias, 1);
            const float bg = odd ? pb : bias, bu = odd ? bias : pb;
            uint16_t *stg = reinterpret_cast<uint16_t *>(stg_bytes);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float mine = odd ? v[16 + i] : v[i];
                const float other = __shfl_xor_sync(0xFFFFFFFFu, odd ? v[i] : v[16 + i], 1);
                const float gate = (odd ? other : mine) + bg;
                const float up = (odd ? mine : other) + bu;
                const float a = clamped_swiglu(gate, up, p.alpha, p.limit);
                stg[(odd ? 16 + i : i) * 16 + (lane >> 1)] = (uint16_t)(pack_bf16x2(a, 0.0f) & 0xFFFFu);
            }
            __syncwarp();
            // lane = token: its 16 features, the 32-feature block maximum shared
            // with the partner warp (lane quarters 0/1 and 2/3 hold one block)
            const uint4 s0 = *reinterpret_cast<const uint4 *>(stg + lane * 16);
            const uint4 s1 = *reinterpret_cast<const uint4 *>(stg + lane * 16 + 8);
            const uint32_t wv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                amax = fmaxf(amax, fmaxf(fabsf(bf16lo_to_f32(wv[i])), fabsf(bf16hi_to_f32(wv[i]))));
            // double-buffered by chunk parity: a warp rewrites a buffer only after
            // the handshake of the next chunk, which its partner joins after
            // reading this one
            float *xs = xch + (chunk & 1) * 128;
            xs[q * 32 + lane] = amax;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(xbar);
            ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(xbar, chunk & 1u)) && ok;
            amax = fmaxf(amax, xs[(q ^ 1) * 32 + lane]);
            const uint32_t bsc = split_scale_byte(amax);
            uint32_t hq[4], lq[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t h0, l0, h1, l1;
                split_pair(bf16lo_to_f32(wv[2 * i]), bf16hi_to_f32(wv[2 * i]), bsc, h0, l0);
                split_pair(bf16lo_to_f32(wv[2 * i + 1]), bf16hi_to_f32(wv[2 * i + 1]), bsc, h1, l1);
                hq[i] = h0 | (h1 << 16);
                lq[i] = l0 | (l1 << 16);
            }
            const int I = p.N / 2;
            const int64_t RS = split_row_bytes(I);
            const int f0 = (t.m0 >> 1) + 16 * q;     // first feature of this warp
            if (lane < nvalid && f0 < I && in_bounds(t.row0 + c0 + lane, p.P) &&
                range_in_bounds(f0, f0 + 16, I)) {
                const int64_t row = t.row0 + c0 + lane;
                uint8_t *hrow = p.actq + row * RS;
                uint8_t *lrow = p.actq + ((int64_t)p.P + row) * RS;
                *reinterpret_cast<uint4 *>(hrow + f0) = make_uint4(hq[0], hq[1], hq[2], hq[3]);
                *reinterpret_cast<uint4 *>(lrow + f0) = make_uint4(lq[0], lq[1], lq[2], lq[3]);
                if ((q & 1) == 0) {   // one warp of the pair writes the block's scale bytes
                    const int blk = f0 >> 5;
                    const int64_t slot = I + 16 * (blk >> 2);
                    hrow[slot + (blk & 3)] = (uint8_t)bsc;
                    lrow[slot + (blk & 3)] = (uint8_t)(bsc - 4u);
                    if ((blk & 3) == 0) {
                        // the writer of a step's first block completes the slot the
                        // way the token split does: scale 1 (127) for blocks past I,
                        // zeros after the scale word, so no byte of the slot is left
                        // from an earlier call
                        const int nblk = I / 32;
#pragma unroll
                        for (int j = 1; j < 4; ++j)
                            if (blk + j >= nblk) hrow[slot + j] = lrow[slot + j] = 127u;
                        uint32_t *hw = reinterpret_cast<uint32_t *>(hrow + slot);
                        uint32_t *lw = reinterpret_cast<uint32_t *>(lrow + slot);
                        hw[1] = hw[2] = hw[3] = 0u;
                        lw[1] = lw[2] = lw[3] = 0u;
                    }
                }
            }
            __syncwarp();
        } else {
            // w * (acc + bias) for 32 tokens x the warp's 32 features, staged
            // so that each pair's row segment leaves as 16-byte stores
            int pair_l = 0;
            float wt_l = 1.0f;
            if (lane < nvalid && in_bounds(t.row0 + c0 + lane, p.P)) {
                pair_l = __ldg(p.sorted_pairs + t.row0 + c0 + lane);
                if (!p.weight_on_input) wt_l = __ldg(p.weights + pair_l);
            }
            // two passes of 16 tokens through a 2 KB staging tile
            float *stg = reinterpret_cast<float *>(stg_bytes);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float wi = __shfl_sync(0xFFFFFFFFu, wt_l, 16 * hf + i);
                    stg[i * 32 + lane] = wi * (v[16 * hf + i] + bias);
                }
                __syncwarp();
                if (32 * q < t.mrows) {                  // warp-uniform
#pragma unroll
                    for (int rd = 0; rd < 4; ++rd) {
                        const int piece = rd * 32 + lane;    // 16 tokens x 8 pieces of 16 B
                        const int tok = 16 * hf + (piece >> 3), part = piece & 7;
                        const int pi = __shfl_sync(0xFFFFFFFFu, pair_l, tok);
                        if (tok < nvalid && in_bounds(pi, p.P) &&
                            range_in_bounds(t.m0 + 32 * q + part * 4, t.m0 + 32 * q + part * 4 + 4, p.N)) {
                            const float4 val = *reinterpret_cast<const float4 *>(stg + (piece >> 3) * 32 + part * 4);
                            *reinterpret_cast<float4 *>(p.yp + (int64_t)pi * p.N + t.m0 + 32 * q + part * 4) = val;
                        }
                    }
                }
                __syncwarp();
            }
        }
    }
    return ok;
}

template <class Cfg, bool kGateUp>
__global__ void __launch_bounds__(Cfg::kThreads, 1)
    grouped_mxfp4_mxf_kernel(const __grid_constant__ CUtensorMap tmap_b,
                             const __grid_constant__ CUtensorMap tmap_bs,
                             const __grid_constant__ CUtensorMap tmap_w, const Params p) {
    constexpr int TOK = Cfg::TOK, S = Cfg::S, PS = Cfg::PS, G = Cfg::G, NACC = Cfg::NACC;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const gbase = smem_raw + (base - raw);
    const int kblocks = p.K / 32;
    const uint32_t sc_slot = Cfg::sc_slot_bytes(kblocks);
    auto a_stage = [&](int s) { return base + Cfg::OFF_A + s * WA_BYTES; };
    auto x_stage = [&](int s) { return base + Cfg::OFF_X + s * Cfg::X_BYTES; };
    auto wp_stage = [&](int s) { return base + Cfg::OFF_WP + s * WP_BYTES; };
    auto sc_stage = [&](int b) { return base + Cfg::OFF_SC + b * sc_slot; };
    const uint32_t bars = base + Cfg::OFF_BAR;
    // b_full(s): the token rows and their scale slots landed (producer arrival + bytes)
    // ready(s):  the four stager warps of the step's group stored its codes and scales
    auto b_full = [&](int s) { return bars + 8u * s; };
    auto ready = [&](int s) { return bars + 8u * (S + s); };
    auto empty = [&](int s) { return bars + 8u * (2 * S + s); };   // MMA done with slot s
    constexpr int B0 = 3 * S;
    auto wp_full = [&](int s) { return bars + 8u * (B0 + s); };
    auto wp_empty = [&](int s) { return bars + 8u * (B0 + PS + s); };
    auto a_full = [&](int b) { return bars + 8u * (B0 + 2 * PS + b); };
    auto a_empty = [&](int b) { return bars + 8u * (B0 + 2 * PS + NACC + b); };
    auto sc_full = [&](int b) { return bars + 8u * (B0 + 2 * PS + 2 * NACC + b); };
    auto sc_empty = [&](int b) { return bars + 8u * (B0 + 2 * PS + 2 * NACC + 2 + b); };
    // xch_bar(pair): both epilogue warps of a lane-quarter pair published their
    // per-token block maxima of the current chunk
    auto xch_bar = [&](int pr) { return bars + 8u * (B0 + 2 * PS + 2 * NACC + 4 + pr); };
    const uint32_t tmem_holder = bars + 8u * (B0 + 2 * PS + 2 * NACC + 6);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(b_full(s), 1);
            ptx::mbar_init(ready(s), 4);
            ptx::mbar_init(empty(s), 1);
        }
        for (int s = 0; s < PS; ++s) {
            ptx::mbar_init(wp_full(s), 1);
            ptx::mbar_init(wp_empty(s), 4 * WP_STEPS);   // four warps per K step of the load
        }
        for (int b = 0; b < NACC; ++b) {
            ptx::mbar_init(a_full(b), 1);
            ptx::mbar_init(a_empty(b), kEpiWarps);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(sc_full(b), 1);
            ptx::mbar_init(sc_empty(b), Cfg::kStageWarps);
            ptx::mbar_init(xch_bar(b), 2);
        }
        ptx::fence_mbarrier_init();
        ptx::prefetch_tmap(&tmap_b);
        ptx::prefetch_tmap(&tmap_bs);
        ptx::prefetch_tmap(&tmap_w);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, Cfg::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    // barriers and TMEM are set up; wait for the producer of this kernel's inputs, then
    // stage the schedule it wrote
    pdl_wait();
    pdl_trigger();
    int *const s_sched = reinterpret_cast<int *>(gbase + Cfg::OFF_SCHED);
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
        s_sched[i] = i < p.E ? __ldg(p.counts + i) : 0;
        s_sched[257 + i] = __ldg(p.offsets + i);
        s_sched[514 + i] = __ldg(p.tile_offsets + i);
    }
    __syncthreads();
    const Sched sc{s_sched, s_sched + 257, s_sched + 514};
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(gbase + (tmem_holder - base));

    const int w_tiles = (p.N + BM - 1) / BM;
    const int total = sc.tile_offsets[p.E] * w_tiles;
    // K steps per tile, rounded up to KALIGN: the extra steps read only the TMA's zero
    // fill (codes and token rows past K) with scale 1 and add nothing
    const int k_iters = ((p.K + BK - 1) / BK + Cfg::KALIGN - 1) / Cfg::KALIGN * Cfg::KALIGN;
    const int wp_loads = k_iters / WP_STEPS;   // packed loads per tile

    if (warp == 0) {
        // ------------------------------------------------------------ token TMA
        uint32_t it = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const Tile t = decode_tile<TOK>(p, sc, item, w_tiles);
            const int nbox = t.h / XBOX_ROWS;
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int s = it % S;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(empty(s), ((it / S) & 1u) ^ 1u)))) break;
                if (ptx::elect_one()) {
                    const uint32_t bar = b_full(s), xs = x_stage(s);
                    ptx::mbar_arrive_expect_tx(bar, 2 * nbox * (XBOX_BYTES + XBOX_ROWS * 16));
                    for (int b = 0; b < nbox; ++b) {
                        const int y = t.row0 + b * XBOX_ROWS;
                        ptx::tma_load_3d(xs + b * XBOX_BYTES, &tmap_b, kb * BK, y, 0, bar);
                        ptx::tma_load_3d(xs + (nbox + b) * XBOX_BYTES, &tmap_b, kb * BK, y, 1, bar);
                        ptx::tma_load_3d(xs + Cfg::X_DATA + b * XBOX_ROWS * 16, &tmap_bs, kb * 16, y, 0, bar);
                        ptx::tma_load_3d(xs + Cfg::X_DATA + (nbox + b) * XBOX_ROWS * 16, &tmap_bs, kb * 16, y, 1, bar);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == Cfg::kWpWarp) {
        // ------------------------------------------------------------ packed-weight TMA
        uint32_t it = 0, local = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++local) {
            const Tile t = decode_tile<TOK>(p, sc, item, w_tiles);
            const int sb = local & 1;
            if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(sc_empty(sb), ((local >> 1) & 1u) ^ 1u)))) break;
            if (ptx::elect_one()) {
                // the tile's scale rows, contiguous in [E, N, K/32]
                const uint32_t bytes = (uint32_t)(t.mrows * kblocks);
                ptx::mbar_arrive_expect_tx(sc_full(sb), bytes);
                ptx::bulk_load(sc_stage(sb), p.wscales + ((int64_t)t.e * p.N + t.m0) * kblocks, bytes, sc_full(sb));
            }
            __syncwarp();
            for (int j = 0; j < wp_loads; ++j, ++it) {
                const int s = it % PS;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(wp_empty(s), ((it / PS) & 1u) ^ 1u)))) break;
                if (ptx::elect_one()) {
                    ptx::mbar_arrive_expect_tx(wp_full(s), WP_BYTES);
                    ptx::tma_load_3d(wp_stage(s), &tmap_w, j * (int)WP_ROW, t.m0, t.e, wp_full(s));
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        uint32_t it = 0, local = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++local) {
            const Tile t = decode_tile<TOK>(p, sc, item, w_tiles);
            const uint32_t idesc = idesc_e2m1_e4m3(BM, 2 * t.h);
            const int b = local % NACC;
            if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(a_empty(b), ((local / NACC) & 1u) ^ 1u)))) break;
            ptx::tc_fence_after();
            const uint32_t d_tmem = tmem_base + b * Cfg::ACC_COLS;
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int s = it % S;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(b_full(s), (it / S) & 1u) &&
                                                        ptx::mbar_wait(ready(s), (it / S) & 1u))))
                    break;
                ptx::tc_fence_after();
                const uint64_t ad = ptx::sw128_kmajor_desc(a_stage(s));
                const uint64_t bd = ptx::sw128_kmajor_desc(x_stage(s));
                const uint32_t sfa = tmem_base + Cfg::SF_COL0 + s * Cfg::SF_STRIDE;
                if (ptx::elect_one()) {
#pragma unroll
                    for (int j = 0; j < KBS; ++j)   // +32 B per 32-element K block (start address >> 4)
                        ptx::mma_mxf8f6f4(d_tmem, ad + 2u * j, bd + 2u * j,
                                          idesc | ((uint32_t)j << 29) | ((uint32_t)j << 4), sfa, sfa + 4,
                                          (kb > 0 || j > 0) ? 1u : 0u);
                    ptx::mma_commit(empty(s));
                }
                __syncwarp();
            }
            if (ok && ptx::elect_one()) ptx::mma_commit(a_full(b));
            __syncwarp();
        }
    } else if (warp < kFirstStageWarp) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        float *const xch = reinterpret_cast<float *>(gbase + Cfg::OFF_XCH);
        uint32_t local = 0, chunk = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++local) {
            const Tile t = decode_tile<TOK>(p, sc, item, w_tiles);
            const int b = local % NACC;
            if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(a_full(b), (local / NACC) & 1u))) break;
            ptx::tc_fence_after();
            ok = epilogue_item<kGateUp>(p, t, tmem_base + b * Cfg::ACC_COLS + lane_off,
                                        gbase + Cfg::OFF_EPI + kEpiStage * q, xch, xch_bar(q >> 1), chunk, q,
                                        lane);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(a_empty(b));
        }
    } else if (warp < Cfg::kWpWarp) {
        // ------------------------------------------------------------ stagers
        // Thread = weight row 32 * (warp % 4) + lane (its TMEM lane): the row's 64
        // packed bytes of the step go to eight unpacked 16-byte chunks (8 code bytes,
        // 8 zero bytes) in the 128-byte swizzled K-major layout; the weight scale
        // words of rows lane, lane + 32, lane + 64, lane + 96 (columns 0..3) and the
        // token scale words of B rows lane + 32 c (columns 4 + c) go to this warp's
        // lane quarter of the step's scale-factor slot.
        const int grp = (warp - kFirstStageWarp) >> 2;
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        uint32_t it = 0, local = 0, pit = 0;   // step and packed-load counters of this CTA
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++local, pit += wp_loads) {
            const Tile t = decode_tile<TOK>(p, sc, item, w_tiles);
            const int sb = local & 1;
            // every stager warp takes part in every tile's scale slot (even with no step
            // of its own in the tile), so that the slot's arrival count never mixes tiles
            if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(sc_full(sb), (local >> 1) & 1u)))) break;
            const uint32_t scb = sc_stage(sb);
            for (int kb = (int)((grp - (int)(it % G) + G) % G); kb < k_iters; kb += G) {
                const uint32_t gi = it + (uint32_t)kb;
                const uint32_t pj = pit + (uint32_t)(kb / WP_STEPS);   // packed load of this step
                const int s = gi % S, ps = pj % PS;
                const int kb0 = kb * KBS;
                // weight scale words of rows lane + 32 c
                uint32_t sfa[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int rw = lane + 32 * c;
                    uint32_t w = 0x7F7F7F7Fu;
                    if (rw < t.mrows && kb0 < kblocks) {
                        const uint32_t a = scb + (uint32_t)(rw * kblocks + kb0);
                        const uint32_t lo16 = ptx::ld_shared_u16(a);
                        const uint32_t hi16 = (kb0 + 2 < kblocks) ? ptx::ld_shared_u16(a + 2) : 0x7F7Fu;
                        w = lo16 | (hi16 << 16);
                    }
                    w = mask_pad_blocks(w, kb0, kblocks);
                    if (__vcmpeq4(w, 0xFFFFFFFFu)) raise_device_error(MOE_DEVERR_BAD_SCALE);
                    sfa[c] = w;
                }
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(wp_full(ps), (pj / PS) & 1u)))) break;
                // this step's 64 bytes: 16-byte chunks 4 (kb % 2) .. + 3 of the row's
                // swizzled 128-byte line
                // the step's 64 bytes are 16-byte chunks c0 .. c0 + 3 of the row's line; load i
                // fetches logical chunk lc[i] (128-byte rows: swizzled positions; 256-byte rows:
                // chunks taken in a lane-rotated order so a warp's loads spread over banks)
                uint4 pk[4];
                uint32_t lc[4];
                const uint32_t src = wp_stage(ps) + row * WP_ROW;
                const uint32_t c0 = 4u * (uint32_t)(kb % WP_STEPS), sw = (uint32_t)(row & 7);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    lc[i] = WP_SWIZZLED ? (uint32_t)i : (uint32_t)((i + row) & 3);
                    const uint32_t phys = WP_SWIZZLED ? ((c0 + lc[i]) ^ sw) : (c0 + lc[i]);
                    pk[i] = ptx::ld_volatile_shared_v4(src + (phys << 4));
                }
                // hand the packed slot back to the TMA at once, after every lane's four
                // loads have landed (volatile loads are never repeated after this)
                ptx::sink_shared(base + Cfg::OFF_SINK + 4u * (uint32_t)(warp & 31),
                                 pk[0].x ^ pk[1].x ^ pk[2].x ^ pk[3].x);
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(wp_empty(ps));
                // the slot is free (MMA done) and the token rows with their scale slots landed
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(empty(s), ((gi / S) & 1u) ^ 1u) &&
                                                        ptx::mbar_wait(b_full(s), (gi / S) & 1u))))
                    break;
                ptx::tc_fence_after();
                // token scale words of B rows lane + 32 c (rows past 2h and token rows past
                // the tile are not used by the MMA; they get scale 1)
                uint32_t sfb[Cfg::NCB];
#pragma unroll
                for (int c = 0; c < Cfg::NCB; ++c) {
                    const int rb = lane + 32 * c;
                    const int j = rb >= t.h ? rb - t.h : rb;
                    uint32_t w = 0x7F7F7F7Fu;
                    if (rb < 2 * t.h && j < t.ntok) w = ptx::ld_shared_u32(x_stage(s) + Cfg::X_DATA + rb * 16);
                    sfb[c] = mask_pad_blocks(w, kb0, kblocks);
                }
                const uint32_t dst = a_stage(s) + row * 128;
                const uint32_t sw128 = (uint32_t)(row & 7);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    ptx::st_shared_v4(dst + (((2u * lc[i]) ^ sw128) << 4), pk[i].x, pk[i].y, 0u, 0u);
                    ptx::st_shared_v4(dst + (((2u * lc[i] + 1u) ^ sw128) << 4), pk[i].z, pk[i].w, 0u, 0u);
                }
                const uint32_t sf = tmem_base + lane_off + Cfg::SF_COL0 + s * Cfg::SF_STRIDE;
                ptx::tmem_st_32x32b_x4(sf, sfa);
                if constexpr (Cfg::NCB == 2) {
                    ptx::tmem_st_32x32b_x2(sf + 4, sfb[0], sfb[1]);
                } else if constexpr (Cfg::NCB == 4) {
                    ptx::tmem_st_32x32b_x4(sf + 4, sfb);
                } else {
                    static_assert(Cfg::NCB == 8, "token scale columns");
                    ptx::tmem_st_32x32b_x8(sf + 4, sfb);
                }
                ptx::tmem_st_wait();
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ready(s));
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(sc_empty(sb));
            it += (uint32_t)k_iters;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

#ifndef MOE_MXF_DECODE_S
#define MOE_MXF_DECODE_S 4
#endif
#ifndef MOE_MXF_DECODE_PS
#define MOE_MXF_DECODE_PS 4
#endif
#ifndef MOE_MXF_DECODE_G
#define MOE_MXF_DECODE_G 4
#endif
using DecodeCfg = Config<32, MOE_MXF_DECODE_S, MOE_MXF_DECODE_PS * 2 / WP_STEPS, 2, MOE_MXF_DECODE_G>;
#ifndef MOE_MXF_PREFILL_S
#define MOE_MXF_PREFILL_S 3
#endif
#ifndef MOE_MXF_PREFILL_G
#define MOE_MXF_PREFILL_G 1
#endif
using PrefillCfg = Config<128, MOE_MXF_PREFILL_S, 2, 1, MOE_MXF_PREFILL_G>;

}  // namespace mxf
}  // namespace moe
