// gemm_dec.cuh -- grouped MXFP4 expert GEMM for decode tiles (few token rows per
// expert) on the sm_100a block-scaled tensor-core path (tcgen05.mma kind::mxf8f6f4):
// the tensor core reads the E2M1 weight codes and their E8M0 block scales directly,
// against activations split exactly into two E4M3 terms (split.cuh).  Bound by the
// weight stream, so the whole design serves one goal: keep enough weight bytes in
// flight per SM that HBM stays busy.
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
// (MoE-Infinity PR #152, Changes: dequant-on-copy of fetched packed experts, [N, K//2]
// layout, E8M0 scales per 32 elements, bias, gate/up split, clamped SwiGLU, fp32
// accumulate; FreeToken PR #838: gate_up bias before the gated activation, down bias
// before the routing weight, sum w*(y + b).)
//
// Weight operand.  The MXF8F6F4 MMA wants 4-bit codes "unpacked" in shared memory
// (each 16-byte chunk of a K-major row holds 16 codes in its first 8 bytes).  The TMA
// engine writes that layout itself (tensor map element type 16 x U4 aligned to 16 B,
// 128-byte swizzle): one load per 128-element K step moves 8 KB of packed codes into
// a 16 KB slot, and the MMA reads the slot as it lands -- no thread touches the codes.
// When K is not a multiple of 128 the last 64 elements of each row are fetched as
// packed bytes and unpacked by the scale warp.
//
// Scale factors.  Per K step the MMA takes one E8M0 byte per (row, 32-element block)
// for the weights and for the token rows from tensor memory: four 32-bit columns per
// operand, lane l of column c holding row l + 32c (replicated in all lane quarters).
// The scale warp assembles both 512-byte shared-memory images per step (weight scales
// from the tile's scale rows, bulk-loaded once per tile; token scales from the split
// rows' per-step scale slots) and the MMA warp moves them into tensor memory with
// tcgen05.cp ahead of its MMAs.
//
// One persistent CTA per SM, 8 warps:
//   warp 0    token TMA: hi and lo rows of the token tile (16-row boxes) and their
//             16-byte scale slots, per K step, into the B ring
//   warp 1    TMEM owner and MMA issuer: 2 x tcgen05.cp + 4 MMAs 128 x 2h x 32 per step
//   warps 2-5 epilogue (TMEM lane quarter = warp % 4)
//   warp 6    weight TMA: the tile's scale rows (one bulk copy per tile), then per K
//             step the unpacked weight slot (or the packed tail box)
//   warp 7    scale images per step (and the tail unpack)
// The tile schedule (per-expert counts, row offsets, tile offsets) sits in shared
// memory; every wait is a bounded mbarrier wait.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "split.cuh"

namespace moe {
namespace dec {

constexpr int BM = 128;                          // weight rows per tile (TMEM lanes)
constexpr int BK = 128;                          // K elements per step
constexpr int KBS = BK / 32;                     // scale blocks per step
constexpr int TOK = 32;                          // token rows per tile
constexpr int NB = 2 * TOK;                      // B rows at most (hi + lo terms)
constexpr int XBOX_ROWS = 16;                    // token rows per TMA box
constexpr uint32_t XBOX_BYTES = XBOX_ROWS * BK;  // one E4M3 term of 16 rows
constexpr uint32_t A_BYTES = BM * BK;            // unpacked codes of a step (16 KB)
constexpr uint32_t A_TX = A_BYTES / 2;           // transaction bytes of an unpacking load:
                                                 // the packed bytes it reads, not the
                                                 // 16 KB it writes
constexpr uint32_t X_DATA = NB * BK;             // code bytes of B
constexpr uint32_t X_BYTES = X_DATA + NB * 16;   // + one 16-byte scale slot per B row
constexpr uint32_t TAIL_ROW = 32;                // packed bytes of the 64-element tail
constexpr uint32_t TAIL_BYTES = BM * TAIL_ROW;
constexpr uint32_t SF_IMAGE = 512;               // 32 lanes x 16 B
constexpr int kMaxE = 256;
constexpr int kEpiWarps = 4;
constexpr uint32_t kEpiStage = 2048;             // staging bytes per epilogue warp
constexpr uint32_t kXchBytes = 2 * 4 * 32 * 4;   // per-token block maxima of warp pairs

#ifndef MOE_DEC_SA
#define MOE_DEC_SA 8
#endif
#ifndef MOE_DEC_SB
#define MOE_DEC_SB 4
#endif
constexpr int SA = MOE_DEC_SA;   // weight slots (8 KB of HBM each in flight)
constexpr int SB = MOE_DEC_SB;   // token slots
constexpr int SF = 4;            // scale images (and tensor-memory scale slots)
constexpr int NACC = 2;          // accumulators

constexpr int kTokWarp = 0, kMmaWarp = 1, kFirstEpiWarp = 2, kWeightWarp = 6, kSfWarp = 7;
constexpr int kThreads = 256;

constexpr uint32_t ACC_COLS = NB;
constexpr uint32_t SF_COL0 = NACC * ACC_COLS;
constexpr uint32_t TMEM_COLS = 256;
static_assert(SF_COL0 + SF * 8 <= TMEM_COLS, "tensor memory columns");

constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_X = OFF_A + SA * A_BYTES;
constexpr uint32_t OFF_SF = OFF_X + SB * X_BYTES;
constexpr uint32_t OFF_TAIL = OFF_SF + SF * 2 * SF_IMAGE;
constexpr uint32_t OFF_EPI = OFF_TAIL + 2 * TAIL_BYTES;
constexpr uint32_t OFF_XCH = OFF_EPI + kEpiStage * kEpiWarps;
constexpr uint32_t OFF_SCHED = OFF_XCH + kXchBytes;
constexpr uint32_t SCHED_BYTES = 3 * 4 * (kMaxE + 1);
constexpr uint32_t OFF_BAR = (OFF_SCHED + SCHED_BYTES + 7u) & ~7u;
constexpr int NBARS = 2 * SA + 2 * SB + 2 * SF + 2 * NACC + 4 + 4 + 2;
constexpr uint32_t OFF_SC = (OFF_BAR + 8 * NBARS + 16 + 127u) & ~127u;
static_assert(X_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "1 KB aligned stages");

__host__ __device__ constexpr uint32_t sc_slot_bytes(int kblocks) { return ((uint32_t)(BM * kblocks) + 127u) & ~127u; }
__host__ __device__ constexpr uint32_t smem_bytes(int kblocks) { return OFF_SC + 2 * sc_slot_bytes(kblocks) + 1024; }

struct Params {
    const int32_t *counts;        // [E]
    const int32_t *offsets;       // [E + 1]
    const int32_t *tile_offsets;  // [E + 1] in TOK-row token tiles
    const uint8_t *wscales;       // [E, N, K/32] E8M0
    const float *bias;            // [E, N] or null
    int E, N, K, P;
    int K_full;                   // K rounded down to a multiple of 128 (unpacking loads)
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

struct Tile {
    int e;       // expert
    int row0;    // first expert-ordered row of the token tile
    int ntok;    // token rows in the tile (1..TOK)
    int h;       // ntok rounded up to 16: first B row of the lo terms
    int m0;      // first weight row
    int mrows;   // weight rows in range
};

// Work item -> tile from the schedule in shared memory; the weight tile index runs
// fastest, so the CTAs running at one time share token tiles through L2.
__device__ __forceinline__ Tile decode_tile(const int *s_counts, const int *s_off, const int *s_toff,
                                           const Params &p, int item, int w_tiles) {
    Tile t;
    const int g = item / w_tiles;
    const int wt = item - g * w_tiles;
    int lo = 0, hi = p.E - 1;   // largest e with tile_offsets[e] <= g
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_toff[mid] <= g)
            lo = mid;
        else
            hi = mid - 1;
    }
    t.e = lo;
    const int tt = g - s_toff[t.e];
    t.row0 = s_off[t.e] + tt * TOK;
    t.ntok = min(TOK, s_counts[t.e] - tt * TOK);
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
// become 127 (scale 1 for the zero codes past K).
__device__ __forceinline__ uint32_t mask_pad_blocks(uint32_t w, int kb0, int kblocks) {
    const int valid = kblocks - kb0;
    if (valid >= 4) return w;
    const uint32_t keep = valid <= 0 ? 0u : (0xFFFFFFFFu >> (8 * (4 - valid)));
    return (w & keep) | (0x7F7F7F7Fu & ~keep);
}

template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_mxfp4_dec_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_tail,
                             const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_bs,
                             const Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const gbase = smem_raw + (base - raw);
    const int kblocks = p.K / 32;
    const uint32_t sc_slot = sc_slot_bytes(kblocks);
    auto a_stage = [&](int s) { return base + OFF_A + (uint32_t)s * A_BYTES; };
    auto x_stage = [&](int s) { return base + OFF_X + (uint32_t)s * X_BYTES; };
    auto sfa_image = [&](int s) { return base + OFF_SF + (uint32_t)s * 2 * SF_IMAGE; };
    auto sfb_image = [&](int s) { return base + OFF_SF + (uint32_t)s * 2 * SF_IMAGE + SF_IMAGE; };
    auto tail_stage = [&](int b) { return base + OFF_TAIL + (uint32_t)b * TAIL_BYTES; };
    auto sc_stage = [&](int b) { return base + OFF_SC + (uint32_t)b * sc_slot; };
    int *const s_counts = reinterpret_cast<int *>(gbase + OFF_SCHED);
    int *const s_off = s_counts + (kMaxE + 1);
    int *const s_toff = s_off + (kMaxE + 1);
    const uint32_t bars = base + OFF_BAR;
    auto a_full = [&](int s) { return bars + 8u * s; };
    auto a_empty = [&](int s) { return bars + 8u * (SA + s); };
    auto b_full = [&](int s) { return bars + 8u * (2 * SA + s); };
    auto b_empty = [&](int s) { return bars + 8u * (2 * SA + SB + s); };
    constexpr int B1 = 2 * SA + 2 * SB;
    auto sf_full = [&](int s) { return bars + 8u * (B1 + s); };
    auto sf_empty = [&](int s) { return bars + 8u * (B1 + SF + s); };
    constexpr int B2 = B1 + 2 * SF;
    auto acc_full = [&](int b) { return bars + 8u * (B2 + b); };
    auto acc_empty = [&](int b) { return bars + 8u * (B2 + NACC + b); };
    constexpr int B3 = B2 + 2 * NACC;
    auto sc_full = [&](int b) { return bars + 8u * (B3 + b); };
    auto sc_empty = [&](int b) { return bars + 8u * (B3 + 2 + b); };
    auto tail_full = [&](int b) { return bars + 8u * (B3 + 4 + b); };
    auto tail_empty = [&](int b) { return bars + 8u * (B3 + 6 + b); };
    // xch_bar(pair): both epilogue warps of a lane-quarter pair published their
    // per-token block maxima of the current chunk
    auto xch_bar = [&](int pr) { return bars + 8u * (B3 + 8 + pr); };
    const uint32_t tmem_holder = bars + 8u * NBARS;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            ptx::mbar_init(a_full(s), 1);
            ptx::mbar_init(a_empty(s), 1);
        }
        for (int s = 0; s < SB; ++s) {
            ptx::mbar_init(b_full(s), 1);
            ptx::mbar_init(b_empty(s), 1);
        }
        for (int s = 0; s < SF; ++s) {
            ptx::mbar_init(sf_full(s), 1);
            ptx::mbar_init(sf_empty(s), 1);
        }
        for (int b = 0; b < NACC; ++b) {
            ptx::mbar_init(acc_full(b), 1);
            ptx::mbar_init(acc_empty(b), kEpiWarps);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(sc_full(b), 1);
            ptx::mbar_init(sc_empty(b), 1);
            ptx::mbar_init(tail_full(b), 1);
            ptx::mbar_init(tail_empty(b), 1);
            ptx::mbar_init(xch_bar(b), 2);
        }
        ptx::fence_mbarrier_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_tail);
        ptx::prefetch_tmap(&tmap_b);
        ptx::prefetch_tmap(&tmap_bs);
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(tmem_holder, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    // barriers and TMEM are set up; wait for the producer of this kernel's inputs, then
    // stage the schedule it wrote
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
        s_counts[i] = i < p.E ? __ldg(p.counts + i) : 0;
        s_off[i] = __ldg(p.offsets + i);
        s_toff[i] = __ldg(p.tile_offsets + i);
    }
    __syncthreads();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(gbase + (tmem_holder - base));

    const int w_tiles = (p.N + BM - 1) / BM;
    const int total = s_toff[p.E] * w_tiles;
    const int k_iters = (p.K + BK - 1) / BK;

    if (warp == kTokWarp) {
        // ------------------------------------------------------------ token TMA
        uint32_t it = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const Tile t = decode_tile(s_counts, s_off, s_toff, p, item, w_tiles);
            const int nbox = t.h / XBOX_ROWS;
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int s = it % SB;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(b_empty(s), ((it / SB) & 1u) ^ 1u)))) break;
                if (ptx::elect_one()) {
                    const uint32_t bar = b_full(s), xs = x_stage(s);
                    ptx::mbar_arrive_expect_tx(bar, 2 * nbox * (XBOX_BYTES + XBOX_ROWS * 16));
                    for (int b = 0; b < nbox; ++b) {
                        const int y = t.row0 + b * XBOX_ROWS;
                        ptx::tma_load_3d(xs + b * XBOX_BYTES, &tmap_b, kb * BK, y, 0, bar);
                        ptx::tma_load_3d(xs + (nbox + b) * XBOX_BYTES, &tmap_b, kb * BK, y, 1, bar);
                        ptx::tma_load_3d(xs + X_DATA + b * XBOX_ROWS * 16, &tmap_bs, kb * 16, y, 0, bar);
                        ptx::tma_load_3d(xs + X_DATA + (nbox + b) * XBOX_ROWS * 16, &tmap_bs, kb * 16, y, 1, bar);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == kWeightWarp) {
        // ------------------------------------------------------------ weight TMA
        uint32_t it = 0, local = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++local) {
            const Tile t = decode_tile(s_counts, s_off, s_toff, p, item, w_tiles);
            const int sb = local & 1;
            if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(sc_empty(sb), ((local >> 1) & 1u) ^ 1u)))) break;
            if (ptx::elect_one()) {
                // the tile's scale rows, contiguous in [E, N, K/32]
                const uint32_t bytes = (uint32_t)(t.mrows * kblocks);
                ptx::mbar_arrive_expect_tx(sc_full(sb), bytes);
                ptx::bulk_load(sc_stage(sb), p.wscales + ((int64_t)t.e * p.N + t.m0) * kblocks, bytes, sc_full(sb));
            }
            __syncwarp();
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int s = it % SA;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(a_empty(s), ((it / SA) & 1u) ^ 1u)))) break;
                if (kb * BK < p.K_full) {
                    if (ptx::elect_one()) {
                        ptx::mbar_arrive_expect_tx(a_full(s), A_TX);
                        ptx::tma_load_3d(a_stage(s), &tmap_a, kb * BK, t.m0, t.e, a_full(s));
                    }
                } else {
                    // the packed 64-element tail of the rows; the scale warp unpacks it into
                    // slot s (free now) and arrives on a_full(s) itself
                    if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(tail_empty(sb), ((local >> 1) & 1u) ^ 1u))))
                        break;
                    if (ptx::elect_one()) {
                        ptx::mbar_arrive_expect_tx(tail_full(sb), TAIL_BYTES);
                        ptx::tma_load_3d(tail_stage(sb), &tmap_tail, p.K_full / 2, t.m0, t.e, tail_full(sb));
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == kSfWarp) {
        // ------------------------------------------------------------ scale images (+ tail)
        // lane l writes row l of both 32 x 16 B images: weight rows l + 32 c, B rows
        // l + 32 c (c < 2; columns 2 and 3 of the token image are not read)
        uint32_t it = 0, local = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++local) {
            const Tile t = decode_tile(s_counts, s_off, s_toff, p, item, w_tiles);
            const int sbuf = local & 1;
            if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(sc_full(sbuf), (local >> 1) & 1u)))) break;
            const uint32_t scb = sc_stage(sbuf);
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int sf = it % SF, sx = it % SB;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(sf_empty(sf), ((it / SF) & 1u) ^ 1u) &&
                                                        ptx::mbar_wait(b_full(sx), (it / SB) & 1u))))
                    break;
                const int kb0 = kb * KBS;
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
                ptx::st_shared_v4(sfa_image(sf) + lane * 16, sfa[0], sfa[1], sfa[2], sfa[3]);
                // token scale words of B rows lane + 32 c (rows past 2h and token rows past
                // the tile are not used by the MMA; they get scale 1)
                uint32_t sfb[2];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int rb = lane + 32 * c;
                    const int j = rb >= t.h ? rb - t.h : rb;
                    uint32_t w = 0x7F7F7F7Fu;
                    if (rb < 2 * t.h && j < t.ntok) w = ptx::ld_shared_u32(x_stage(sx) + X_DATA + rb * 16);
                    sfb[c] = mask_pad_blocks(w, kb0, kblocks);
                }
                ptx::st_shared_v4(sfb_image(sf) + lane * 16, sfb[0], sfb[1], 0x7F7F7F7Fu, 0x7F7F7F7Fu);
                if (kb * BK >= p.K_full) {
                    // tail step: rows lane + 32 r, 32 packed bytes each -> chunks 0..3 of the
                    // row's unpacked line (8 code bytes, 8 zero bytes), chunks 4..7 zero
                    const int s = it % SA;
                    if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(tail_full(sbuf), (local >> 1) & 1u)))) break;
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int row = lane + 32 * r;
                        const uint32_t src = tail_stage(sbuf) + (uint32_t)row * TAIL_ROW;
                        const uint4 q0 = ptx::ld_shared_v4(src), q1 = ptx::ld_shared_v4(src + 16);
                        const uint32_t dst = a_stage(s) + (uint32_t)row * 128, sw = (uint32_t)(row & 7);
                        ptx::st_shared_v4(dst + ((0u ^ sw) << 4), q0.x, q0.y, 0u, 0u);
                        ptx::st_shared_v4(dst + ((1u ^ sw) << 4), q0.z, q0.w, 0u, 0u);
                        ptx::st_shared_v4(dst + ((2u ^ sw) << 4), q1.x, q1.y, 0u, 0u);
                        ptx::st_shared_v4(dst + ((3u ^ sw) << 4), q1.z, q1.w, 0u, 0u);
#pragma unroll
                        for (uint32_t j = 4; j < 8; ++j) ptx::st_shared_v4(dst + ((j ^ sw) << 4), 0u, 0u, 0u, 0u);
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        ptx::mbar_arrive(a_full(s));
                        ptx::mbar_arrive(tail_empty(sbuf));
                    }
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(sf_full(sf));
            }
            __syncwarp();
            if (ok && lane == 0) ptx::mbar_arrive(sc_empty(sbuf));
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        uint32_t it = 0, local = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++local) {
            const Tile t = decode_tile(s_counts, s_off, s_toff, p, item, w_tiles);
            const uint32_t idesc = idesc_e2m1_e4m3(BM, 2 * t.h);
            const int b = local % NACC;
            if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(acc_empty(b), ((local / NACC) & 1u) ^ 1u)))) break;
            ptx::tc_fence_after();
            const uint32_t d_tmem = tmem_base + b * ACC_COLS;
            for (int kb = 0; kb < k_iters; ++kb, ++it) {
                const int sa = it % SA, sx = it % SB, sf = it % SF;
                if (!(ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(a_full(sa), (it / SA) & 1u) &&
                                                        ptx::mbar_wait(b_full(sx), (it / SB) & 1u) &&
                                                        ptx::mbar_wait(sf_full(sf), (it / SF) & 1u))))
                    break;
                ptx::tc_fence_after();
                if (ptx::elect_one()) {
                    const uint32_t sft = tmem_base + SF_COL0 + (uint32_t)sf * 8u;
                    ptx::tmem_cp_32x128b_warpx4(sft, ptx::plain_kmajor_desc(sfa_image(sf)));
                    ptx::tmem_cp_32x128b_warpx4(sft + 4u, ptx::plain_kmajor_desc(sfb_image(sf)));
                    const uint64_t ad = ptx::sw128_kmajor_desc(a_stage(sa));
                    const uint64_t bd = ptx::sw128_kmajor_desc(x_stage(sx));
#pragma unroll
                    for (int j = 0; j < KBS; ++j)   // +32 B per 32-element K block (start address >> 4)
                        ptx::mma_mxf8f6f4(d_tmem, ad + 2u * j, bd + 2u * j,
                                          idesc | ((uint32_t)j << 29) | ((uint32_t)j << 4), sft, sft + 4u,
                                          (kb > 0 || j > 0) ? 1u : 0u);
                    ptx::mma_commit(a_empty(sa));
                    ptx::mma_commit(b_empty(sx));
                    ptx::mma_commit(sf_empty(sf));
                }
                __syncwarp();
            }
            if (ok && ptx::elect_one()) ptx::mma_commit(acc_full(b));
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int r = q * 32 + lane;             // weight row within the tile
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        float *const xch = reinterpret_cast<float *>(gbase + OFF_XCH);
        uint32_t local = 0, chunk = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++local) {
            const Tile t = decode_tile(s_counts, s_off, s_toff, p, item, w_tiles);
            const int b = local % NACC;
            if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(acc_full(b), (local / NACC) & 1u))) break;
            ptx::tc_fence_after();
            const bool row_ok = r < t.mrows;
            const int n = t.m0 + r;
            const float bias = (p.bias && row_ok) ? __ldg(p.bias + (int64_t)t.e * p.N + n) : 0.0f;
            const uint32_t acc = tmem_base + b * ACC_COLS + lane_off;
            for (int c0 = 0; c0 < t.ntok; c0 += 32, ++chunk) {
                // hi-term columns, then the lo-term columns added in two pieces of 16
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
                    uint16_t *stg = reinterpret_cast<uint16_t *>(gbase + OFF_EPI + kEpiStage * q);
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
                    if (lane == 0) ptx::mbar_arrive(xch_bar(q >> 1));
                    ok = __all_sync(0xFFFFFFFFu, ptx::mbar_wait(xch_bar(q >> 1), chunk & 1u));
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
                            const int64_t at = I + 16 * (blk >> 2) + (blk & 3);
                            hrow[at] = (uint8_t)bsc;
                            lrow[at] = (uint8_t)(bsc - 4u);
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
                    float *stg = reinterpret_cast<float *>(gbase + OFF_EPI + kEpiStage * q);
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
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(acc_empty(b));
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace dec
}  // namespace moe
