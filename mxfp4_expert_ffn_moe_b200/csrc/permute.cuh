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
// One CTA of 32 warps: warp w owns a contiguous chunk of pairs, counts its experts
// in a private shared-memory row, the chunk bases come from an exclusive scan over
// warps, and each warp then scatters its chunk in order using __match_any_sync to
// rank equal experts inside a 32-pair step.  When the ids fit (staged != 0) they are
// first copied into shared memory with independent, coalesced loads, so neither
// pass over them waits on a global load per step.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kPermuteThreads = 1024;

// Dynamic shared memory of permute_pairs_kernel: the count rows and expert starts,
// plus P staged ids when `staged`.
__host__ __device__ constexpr size_t permute_smem_bytes(int E, int64_t P, bool staged) {
    return sizeof(int) * (size_t)(32 * E + E + 1) + (staged ? sizeof(int) * (size_t)P : 0);
}
constexpr size_t kPermuteSmemCap = 200 * 1024;

__device__ __forceinline__ int relative_expert(int32_t id, int expert_base, int E) {
    const int64_t e = (int64_t)id - expert_base;
    return (e >= 0 && e < E) ? (int)e : -1;
}

// ids are taken relative to expert_base: pair p belongs to expert ids[p] - expert_base
// of the E experts handled here (a rank's slice of the experts under expert parallelism;
// 0 for the whole layer).
__global__ void __launch_bounds__(kPermuteThreads) permute_pairs_kernel(
    const int32_t *__restrict__ ids, int expert_base, int64_t P, int E, int bm, int staged, int32_t *__restrict__ counts,
    int32_t *__restrict__ offsets, int32_t *__restrict__ tile_offsets,
    int32_t *__restrict__ sorted_pairs, int32_t *__restrict__ pair_rows) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ int sm_perm[];
    int *cnt = sm_perm;             // [32][E]: per-warp counts, then per-warp running bases
    int *off = sm_perm + 32 * E;    // [E + 1]: expert start rows
    int *ids_s = off + E + 1;       // [P] when staged
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) cnt[i] = 0;
    if (staged)
        for (int64_t i = threadIdx.x; i < P; i += blockDim.x) ids_s[i] = relative_expert(__ldg(ids + i), expert_base, E);
    __syncthreads();
    // expert of pair p relative to expert_base, -1 when outside [0, E)
    auto expert_of = [&](int64_t p) { return staged ? ids_s[p] : relative_expert(__ldg(ids + p), expert_base, E); };

    const int64_t chunk = (P + 31) / 32;
    const int64_t beg = (int64_t)warp * chunk;
    const int64_t end = (beg + chunk < P) ? beg + chunk : P;
    for (int64_t p = beg + lane; p < end; p += 32) {
        const int e = expert_of(p);
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&cnt[warp * E + e], 1);
        else
            raise_device_error(MOE_DEVERR_BAD_EXPERT_ID);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < 32; ++w) {
            const int c = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += c;
        }
        off[e] = run;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0, trun = 0;
        for (int e = 0; e < E; ++e) {
            const int c = off[e];
            counts[e] = c;
            offsets[e] = run;
            tile_offsets[e] = trun;
            off[e] = run;
            run += c;
            trun += (c + bm - 1) / bm;
        }
        offsets[E] = run;
        tile_offsets[E] = trun;
        off[E] = run;
    }
    __syncthreads();
    for (int64_t base = beg; base < end; base += 32) {
        const int64_t p = base + lane;
        const int e = (p < end) ? expert_of(p) : -1;
        const bool valid = (p < end) && (unsigned)e < (unsigned)E;
        const int key = valid ? e : -1 - lane;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int wbase = valid ? cnt[warp * E + e] : 0;
        __syncwarp();
        if (valid && in_bounds(off[e] + wbase + rank, P)) {
            sorted_pairs[off[e] + wbase + rank] = (int32_t)p;
            if (rank == 0) cnt[warp * E + e] = wbase + __popc(peers);
        }
        if (pair_rows && p < end) pair_rows[p] = valid ? off[e] + wbase + rank : -1;
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
