// permute.cuh -- group (token, slot) pairs by expert, then gather the expert inputs.
//
// Pair p = t*k + j routed to expert ids[p].  The grouped expert GEMMs want the
// pairs of each expert contiguous ("expert-ordered prefill views", FreeToken PR
// #838 "What it does"; the "[T, k, 2I] gathers on prefill" of its review), so:
//   counts[e]        pairs routed to expert e
//   offsets[e]       first row of expert e in expert order (exclusive scan), offsets[E] = rows
//   tile_offsets[e]  first M-tile of expert e for an M-tile of bm rows
//   sorted_pairs[r]  the pair p placed at row r; within an expert rows follow
//                    ascending p (a stable, deterministic order)
//   pair_rows[p]     (optional) the inverse: the row of pair p, -1 for a dropped pair
// Ids outside [0, E) raise MOE_DEVERR_BAD_EXPERT_ID and their pairs are dropped.
//
// C CTAs of 32 warps, with no communication between them.  The pairs are cut into
// 32*C sub-chunks of sc consecutive pairs; CTA c places the 32 sub-chunks of its range
// [c*32*sc, (c+1)*32*sc), warp w the w-th of them.  Every CTA reads all the ids and
// counts, per expert, the pairs before its range, in each of its sub-chunks and after
// its range (warp-private rows, so shared atomics only collide inside a warp); from
// these it has the totals (CTA 0 writes counts, offsets and tile_offsets), the expert
// starts (one warp's shuffle scan) and the first row of each of its sub-chunks in each
// expert.  Each warp then places its sub-chunk 32 pairs at a time, ranking equal
// experts with __match_any_sync.  The ranking is the costly step (match.any issues at
// about one per 32 clocks on an SM), which is why the pairs are spread over ~P/2048
// CTAs instead of one.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kPermuteThreads = 1024;
constexpr int kPermutePairsPerCta = 2048;

// Sub-chunk length for C CTAs.
__host__ __device__ constexpr int64_t permute_subchunk(int64_t P, int C) { return (P + 32 * (int64_t)C - 1) / (32 * (int64_t)C); }
// Dynamic shared memory of permute_pairs_kernel: three [32][E] count tables, the E + 1
// expert starts, and the CTA's sub-chunk ids (int16).
__host__ __device__ constexpr size_t permute_smem_bytes(int E, int64_t sc) {
    return sizeof(int) * (size_t)(3 * 32 * E + E + 1) + 2 * (size_t)(32 * sc);
}
constexpr size_t kPermuteSmemCap = 227 * 1024;

__device__ __forceinline__ int relative_expert(int32_t id, int expert_base, int E) {
    const int64_t e = (int64_t)id - expert_base;
    return (e >= 0 && e < E) ? (int)e : -1;
}

// ids are taken relative to expert_base: pair p belongs to expert ids[p] - expert_base
// of the E experts handled here (a rank's slice of the experts under expert parallelism;
// 0 for the whole layer).
__global__ void __launch_bounds__(kPermuteThreads) permute_pairs_kernel(
    const int32_t *__restrict__ ids, int expert_base, int64_t P, int E, int bm, int32_t *__restrict__ counts,
    int32_t *__restrict__ offsets, int32_t *__restrict__ tile_offsets,
    int32_t *__restrict__ sorted_pairs, int32_t *__restrict__ pair_rows) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) int sm_perm[];
    int *pre = sm_perm;                 // [32][E]: per-warp counts before the range
    int *post = pre + 32 * E;           // [32][E]: per-warp counts after the range
    int *cnt = post + 32 * E;           // [32][E]: per-sub-chunk counts, then first rows
    int *off = cnt + 32 * E;            // [E + 1]: expert start rows
    int16_t *ids_s = reinterpret_cast<int16_t *>(off + E + 1);   // [32 * sc]: the range's experts
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t sc = permute_subchunk(P, gridDim.x);
    const int64_t own_beg = min(P, (int64_t)blockIdx.x * 32 * sc);
    const int64_t own_end = min(P, own_beg + 32 * sc);
    // one CTA: every pair is in its range, the before/after tables stay unused
    const bool single = gridDim.x == 1;
    for (int i = threadIdx.x + (single ? 2 * 32 * E : 0); i < 3 * 32 * E; i += blockDim.x) sm_perm[i] = 0;
    __syncthreads();

    auto count_pair = [&](int64_t i, int32_t id) {
        const int e = relative_expert(id, expert_base, E);
        if (i < own_beg) {
            if (e >= 0) atomicAdd(&pre[warp * E + e], 1);
        } else if (i < own_end) {
            ids_s[i - own_beg] = (int16_t)e;
            if (e >= 0)
                atomicAdd(&cnt[(int)((i - own_beg) / sc) * E + e], 1);
            else
                raise_device_error(MOE_DEVERR_BAD_EXPERT_ID);
        } else if (e >= 0) {
            atomicAdd(&post[warp * E + e], 1);
        }
    };
    // all ids: 16-byte loads, four per thread in flight before their counts
    const int64_t nv = ((reinterpret_cast<uintptr_t>(ids) & 15u) == 0) ? P / 4 : 0;
    const int4 *ids4 = reinterpret_cast<const int4 *>(ids);
    for (int64_t i0 = threadIdx.x; i0 < nv; i0 += 4 * (int64_t)blockDim.x) {
        int4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i0 + u * (int64_t)blockDim.x < nv) v[u] = __ldg(ids4 + i0 + u * (int64_t)blockDim.x);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t i = i0 + u * (int64_t)blockDim.x;
            if (i >= nv) continue;
            count_pair(4 * i, v[u].x);
            count_pair(4 * i + 1, v[u].y);
            count_pair(4 * i + 2, v[u].z);
            count_pair(4 * i + 3, v[u].w);
        }
    }
    for (int64_t i = 4 * nv + threadIdx.x; i < P; i += blockDim.x) count_pair(i, __ldg(ids + i));
    __syncthreads();
    // per expert: the totals, then (after the scan) the first row of each sub-chunk
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int before = 0, total = 0;
        if (single) {
            for (int w = 0; w < 32; ++w) total += cnt[w * E + e];
        } else {
            for (int w = 0; w < 32; ++w) {
                before += pre[w * E + e];
                total += cnt[w * E + e] + post[w * E + e];
            }
        }
        off[e] = before + total;
        pre[e] = before;              // row 0 of pre is only read again as the "before" count
    }
    __syncthreads();
    if (warp == 0) {
        // lane l takes experts [l*per, l*per + per): its totals, an exclusive scan of
        // those over the lanes, then its experts' starts in order
        const int per = (E + 31) / 32;
        const int e0 = lane * per, e1 = min(e0 + per, E);
        int sum = 0, tsum = 0;
        for (int e = e0; e < e1; ++e) {
            sum += off[e];
            tsum += (off[e] + bm - 1) / bm;
        }
        int incl = sum, tincl = tsum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int a = __shfl_up_sync(0xFFFFFFFFu, incl, d), b = __shfl_up_sync(0xFFFFFFFFu, tincl, d);
            if (lane >= d) {
                incl += a;
                tincl += b;
            }
        }
        int run = incl - sum, trun = tincl - tsum;
        for (int e = e0; e < e1; ++e) {
            const int c = off[e];
            if (blockIdx.x == 0) {
                counts[e] = c;
                offsets[e] = run;
                tile_offsets[e] = trun;
            }
            off[e] = run;
            run += c;
            trun += (c + bm - 1) / bm;
        }
        if (lane == 31) {
            if (blockIdx.x == 0) {
                offsets[E] = incl;
                tile_offsets[E] = tincl;
            }
            off[E] = incl;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = off[e] + pre[e];
        for (int w = 0; w < 32; ++w) {
            const int c = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    const int64_t beg = min(own_end, own_beg + warp * sc);
    const int64_t end = min(own_end, beg + sc);
    for (int64_t base = beg; base < end; base += 32) {
        const int64_t p = base + lane;
        const int e = (p < end) ? (int)ids_s[p - own_beg] : -1;
        const bool valid = (p < end) && e >= 0;
        const int key = valid ? e : -1 - lane;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int row = valid ? cnt[warp * E + e] + rank : -1;
        __syncwarp();
        if (valid && in_bounds(row, P)) {
            sorted_pairs[row] = (int32_t)p;
            if (rank == 0) cnt[warp * E + e] += __popc(peers);
        }
        if (pair_rows && p < end) pair_rows[p] = row;
        __syncwarp();
    }
}

// x_perm[r] = x[t] (router weight on the output) or bf16(w[p] * x[t]) (router
// weight on the input), t = sorted_pairs[r] / k.  One warp per row, 16-byte chunks.
// Optionally (row_ids / row_weights non-null) also row_ids[r] = ids[p] and
// row_weights[r] = weights[p]: the rows as a self-contained batch, e.g. to ship to the
// rank that owns their experts.
__global__ void __launch_bounds__(256) gather_rows_kernel(
    const uint16_t *__restrict__ x, const float *__restrict__ weights,
    const int32_t *__restrict__ sorted_pairs, const int32_t *__restrict__ offsets, int E, int k,
    int64_t H, int weight_on_input, uint16_t *__restrict__ x_perm, const int32_t *__restrict__ ids,
    int32_t *__restrict__ row_ids, float *__restrict__ row_weights, int64_t P) {
    pdl_wait();
    pdl_trigger();
    const int rows = offsets[E];
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    const int64_t chunks = H / 8;
    for (int64_t r = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); r < rows;
         r += (int64_t)gridDim.x * wpb) {
        const int p = sorted_pairs[r];
        if (!in_bounds(r, P) || !in_bounds(p, P)) continue;   // warp-uniform (one row per warp)
        const int64_t t = p / k;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + t * H);
        uint4 *dst = reinterpret_cast<uint4 *>(x_perm + r * H);
        const float w = weight_on_input ? weights[p] : 1.0f;
        if (lane == 0 && row_ids) row_ids[r] = ids[p];
        if (lane == 0 && row_weights) row_weights[r] = weights[p];
        // four 16-byte loads in flight per lane before their stores
        for (int64_t c0 = lane; c0 < chunks; c0 += 4 * 32) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (c0 + 32 * u < chunks) v[u] = __ldg(src + c0 + 32 * u);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (c0 + 32 * u >= chunks) continue;
                if (weight_on_input) {
                    v[u].x = pack_bf16x2(bf16lo_to_f32(v[u].x) * w, bf16hi_to_f32(v[u].x) * w);
                    v[u].y = pack_bf16x2(bf16lo_to_f32(v[u].y) * w, bf16hi_to_f32(v[u].y) * w);
                    v[u].z = pack_bf16x2(bf16lo_to_f32(v[u].z) * w, bf16hi_to_f32(v[u].z) * w);
                    v[u].w = pack_bf16x2(bf16lo_to_f32(v[u].w) * w, bf16hi_to_f32(v[u].w) * w);
                }
                dst[c0 + 32 * u] = v[u];
            }
        }
    }
}

}  // namespace moe
