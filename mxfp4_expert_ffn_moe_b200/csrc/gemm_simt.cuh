// gemm_simt.cuh -- grouped expert projections on CUDA cores (fp32 FMA).
//
// Expert e's rows [offsets[e], offsets[e+1]) of the expert-ordered input meet
// expert e's packed MXFP4 weight rows, decoded tile by tile into shared memory:
//   gate_up: h = x . W_gu[e]^T + b_gu[e]; gate = h[2i], up = h[2i+1];
//            act[r, i] = bf16(clamped_swiglu(gate, up))
//   down:    y = act . W_d[e]^T + b_d[e]; yp[p, :] = w[p] * y  (router weight on
//            the output) or y (router weight on the input), p = sorted_pairs[r]
// (MoE-Infinity PR #152, Changes: scales, bias, [N, K//2] layout, gate/up split,
// clamped SwiGLU, fp32 accumulate; FreeToken PR #838: bias before the activation
// and before the routing weight).
//
// Tile 64 rows x 64 weight rows, K step 32 (one scale block); 256 threads, each
// owning a 4 x 4 patch.  Blocks map to (expert, M-tile) through tile_offsets; the
// grid is sized by the host-side upper bound and surplus blocks return at once.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kSimtBM = 64, kSimtBN = 64, kSimtBK = 32;

__device__ __forceinline__ int find_tile_expert(const int32_t *__restrict__ tile_offsets, int E,
                                                int tix) {
    int lo = 0, hi = E - 1;  // largest e with tile_offsets[e] <= tix
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_offsets[mid] <= tix)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

template <bool kGateUp>
__global__ void __launch_bounds__(256) grouped_mxfp4_simt_kernel(
    const uint16_t *__restrict__ A,  // [rows, K] bf16, expert order
    const uint8_t *__restrict__ wblocks, const uint8_t *__restrict__ wscales,
    const float *__restrict__ bias,  // [E, N] or null
    const int32_t *__restrict__ counts, const int32_t *__restrict__ offsets,
    const int32_t *__restrict__ tile_offsets, int E, int N, int K,
    // gate_up epilogue
    uint16_t *__restrict__ act, float alpha, float limit,
    // down epilogue
    float *__restrict__ yp, const int32_t *__restrict__ sorted_pairs,
    const float *__restrict__ weights, int weight_on_input) {
    __shared__ float As[kSimtBK][kSimtBM + 4];
    __shared__ float Bs[kSimtBK][kSimtBN + 4];
    __shared__ float lut[16];

    const int tix = blockIdx.x;
    if (tix >= tile_offsets[E]) return;
    const int e = find_tile_expert(tile_offsets, E, tix);
    const int mt = tix - tile_offsets[e];
    const int row0 = offsets[e] + mt * kSimtBM;
    const int mrows = min(kSimtBM, counts[e] - mt * kSimtBM);
    const int n0 = blockIdx.y * kSimtBN;

    const int tid = threadIdx.x;
    if (tid < 16) {
        const uint32_t c = tid, ex = (c >> 1) & 3u, m = c & 1u;
        float mag = (ex == 0u) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, (int)ex - 1);
        lut[c] = (c & 8u) ? -mag : mag;
    }
    const int ty = tid >> 4, tx = tid & 15;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

    const int64_t kbytes = K / 2, kblocks = K / 32;
    for (int kb = 0; kb < K / kSimtBK; ++kb) {
        __syncthreads();
        {   // A tile: 64 rows x 32 bf16, 16 bytes per thread
            const int r = tid >> 2, ch = tid & 3;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r < mrows)
                v = *reinterpret_cast<const uint4 *>(A + (int64_t)(row0 + r) * K + kb * kSimtBK + ch * 8);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                As[ch * 8 + 2 * q][r] = bf16lo_to_f32(w4[q]);
                As[ch * 8 + 2 * q + 1][r] = bf16hi_to_f32(w4[q]);
            }
        }
        if (tid < kSimtBN) {  // B tile: one weight row per thread, one scale block
            const int n = n0 + tid;
            if (n < N) {
                const int64_t row = (int64_t)e * N + n;
                const uint4 q4 = *reinterpret_cast<const uint4 *>(wblocks + row * kbytes + kb * 16);
                const uint32_t s = wscales[row * kblocks + kb];
                if (s == 255u) raise_device_error(MOE_DEVERR_BAD_SCALE);
                const float sc = e8m0_to_f32(s);
                const uint32_t q[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                for (int w = 0; w < 4; ++w)
#pragma unroll
                    for (int nib = 0; nib < 8; ++nib)
                        Bs[w * 8 + nib][tid] = lut[(q[w] >> (4 * nib)) & 15u] * sc;
            } else {
#pragma unroll
                for (int kk = 0; kk < kSimtBK; ++kk) Bs[kk][tid] = 0.0f;
            }
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kSimtBK; ++kk) {
            const float4 a = *reinterpret_cast<const float4 *>(&As[kk][ty * 4]);
            const float4 b = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
    }

    const int c0 = n0 + tx * 4;
    if (c0 >= N) return;
    float bsum[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) bsum[j] = bias ? bias[(int64_t)e * N + c0 + j] : 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        if (r >= mrows) continue;
        const int64_t grow = row0 + r;
        if (kGateUp) {
            const float a0 = clamped_swiglu(acc[i][0] + bsum[0], acc[i][1] + bsum[1], alpha, limit);
            const float a1 = clamped_swiglu(acc[i][2] + bsum[2], acc[i][3] + bsum[3], alpha, limit);
            *reinterpret_cast<uint32_t *>(act + grow * (N / 2) + c0 / 2) = pack_bf16x2(a0, a1);
        } else {
            const int p = sorted_pairs[grow];
            const float w = weight_on_input ? 1.0f : weights[p];
            float4 o;
            o.x = w * (acc[i][0] + bsum[0]);
            o.y = w * (acc[i][1] + bsum[1]);
            o.z = w * (acc[i][2] + bsum[2]);
            o.w = w * (acc[i][3] + bsum[3]);
            *reinterpret_cast<float4 *>(yp + (int64_t)p * N + c0) = o;
        }
    }
}

}  // namespace moe
