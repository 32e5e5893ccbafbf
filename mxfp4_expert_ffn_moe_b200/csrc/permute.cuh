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
// warps (the expert starts from one warp's shuffle scan), and each warp then places
// its chunk in order using __match_any_sync to rank equal experts inside a 32-pair
// step.  When they fit (staged != 0, up to ~35K pairs), the ids are first copied
// into shared memory as 16-bit expert numbers with coalesced 16-byte loads, the pairs
// are placed into a shared-memory copy of sorted_pairs, and that copy leaves with
// coalesced 16-byte stores: one SM alone would otherwise issue one L2 transaction per
// pair for the scattered stores.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kPermuteThreads = 1024;

// Dynamic shared memory of permute_pairs_kernel: the count rows and expert starts;
// when staged, also the P ids (int16) and the P placed pairs (int32, 16-byte aligned).
__host__ __device__ constexpr size_t permute_ids_offset(int E) { return sizeof(int) * (size_t)(33 * E + 1); }
__host__ __device__ constexpr size_t permute_sorted_offset(int E, int64_t P) {
    return (permute_ids_offset(E) + 2 * (size_t)P + 15) & ~(size_t)15;
}
__host__ __device__ constexpr size_t permute_smem_bytes(int E, int64_t P, bool staged) {
    return staged ? permute_sorted_offset(E, P) + 4 * (size_t)P : permute_ids_offset(E);
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
    const int32_t *__restrict__ ids, int expert_base, int64_t P, int E, int bm, int staged, int32_t *__restrict__ counts,
    int32_t *__restrict__ offsets, int32_t *__restrict__ tile_offsets,
    int32_t *__restrict__ sorted_pairs, int32_t *__restrict__ pair_rows) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) unsigned char sm_perm_raw[];
    int *cnt = reinterpret_cast<int *>(sm_perm_raw);     // [32][E]: per-warp counts, then running bases
    int *off = cnt + 32 * E;                              // [E + 1]: expert start rows
    int16_t *ids_s = reinterpret_cast<int16_t *>(sm_perm_raw + permute_ids_offset(E));          // [P]
    int32_t *sorted_s = reinterpret_cast<int32_t *>(sm_perm_raw + permute_sorted_offset(E, P));  // [P]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) cnt[i] = 0;
    if (staged) {
        // 16-byte loads, eight per thread in flight before their stores
        const int64_t nv = ((reinterpret_cast<uintptr_t>(ids) & 15u) == 0) ? P / 4 : 0;
        const int4 *ids4 = reinterpret_cast<const int4 *>(ids);
        for (int64_t i0 = threadIdx.x; i0 < nv; i0 += 8 * (int64_t)blockDim.x) {
            int4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u * (int64_t)blockDim.x < nv) v[u] = __ldg(ids4 + i0 + u * (int64_t)blockDim.x);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t i = i0 + u * (int64_t)blockDim.x;
                if (i >= nv) continue;
                ids_s[4 * i] = (int16_t)relative_expert(v[u].x, expert_base, E);
                ids_s[4 * i + 1] = (int16_t)relative_expert(v[u].y, expert_base, E);
                ids_s[4 * i + 2] = (int16_t)relative_expert(v[u].z, expert_base, E);
                ids_s[4 * i + 3] = (int16_t)relative_expert(v[u].w, expert_base, E);
            }
        }
        for (int64_t i = 4 * nv + threadIdx.x; i < P; i += blockDim.x)
            ids_s[i] = (int16_t)relative_expert(__ldg(ids + i), expert_base, E);
    }
    __syncthreads();
    // expert of pair p relative to expert_base, -1 when outside [0, E)
    auto expert_of = [&](int64_t p) {
        return staged ? (int)ids_s[p] : relative_expert(__ldg(ids + p), expert_base, E);
    };

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
            counts[e] = c;
            offsets[e] = run;
            tile_offsets[e] = trun;
            off[e] = run;
            run += c;
            trun += (c + bm - 1) / bm;
        }
        if (lane == 31) {
            offsets[E] = incl;
            tile_offsets[E] = tincl;
            off[E] = incl;
        }
    }
    __syncthreads();
    int32_t *const place = staged ? sorted_s : sorted_pairs;
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
            place[off[e] + wbase + rank] = (int32_t)p;
            if (rank == 0) cnt[warp * E + e] = wbase + __popc(peers);
        }
        if (pair_rows && p < end) pair_rows[p] = valid ? off[e] + wbase + rank : -1;
        __syncwarp();
    }
    if (staged) {
        __syncthreads();
        const int rows = off[E];
        const int nv = ((reinterpret_cast<uintptr_t>(sorted_pairs) & 15u) == 0) ? rows / 4 : 0;
        for (int i = threadIdx.x; i < nv; i += blockDim.x)
            reinterpret_cast<int4 *>(sorted_pairs)[i] = reinterpret_cast<const int4 *>(sorted_s)[i];
        for (int i = 4 * nv + threadIdx.x; i < rows; i += blockDim.x) sorted_pairs[i] = sorted_s[i];
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
