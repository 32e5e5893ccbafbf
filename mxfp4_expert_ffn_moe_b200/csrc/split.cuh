// split.cuh -- exact two-term E4M3 split of bf16 activations for the block-scaled
// tensor-core path.
//
// A bf16 value v (8 significant bits) in a 32-element block whose largest magnitude
// has binary exponent e is written as
//     v = hi * S + lo * S / 16,   S = 2^(e - 7),   hi, lo in E4M3,
// hi = E4M3_rn(v / S) and lo = E4M3_rn((v - hi * S) * 16 / S).  |v| / S < 256, so hi
// never saturates; v - hi * S is exact in fp32 and has at most 4 significant bits, so
// lo holds it exactly unless it falls below the E4M3 subnormal range, i.e. for
// elements about 2^-14 of the block maximum and smaller (their residual error is at
// most 2^-14 S).  The E8M0 byte of the block stores S (bias 127); the lo term uses
// the byte minus 4.  With hi and lo both fed to the MXF8F6F4 MMA against E2M1
// weights, the products equal bf16(weights) x bf16(activations) of the plain
// formulation up to that residual (MoE-Infinity PR #152, Changes: bf16 activations
// times dequantized weights with fp32 accumulation).
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// E8M0 byte of the hi term for a block with largest magnitude amax: e + 120,
// clamped to [4, 254] (amax = 0 or below 2^-116 takes 4; the lo byte is then 0).
__device__ __forceinline__ uint32_t split_scale_byte(float amax) {
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
    return (uint32_t)min(max(e + 120, 4), 254);
}

// 2^(127 - b) for b in [4, 253] (the reciprocal of the hi scale).
__device__ __forceinline__ float split_inv_scale(uint32_t b) { return __uint_as_float((254u - b) << 23); }

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)byte, __NV_E4M3);
    __half_raw lo;
    lo.x = h.x;
    return __half2float(__half(lo));
}

// Two values of one block -> (hi bytes, lo bytes), each packed 2 x 8 bits (first value
// in the low byte).
__device__ __forceinline__ void split_pair(float v0, float v1, uint32_t b, uint32_t &hi2, uint32_t &lo2) {
    const float inv = split_inv_scale(b);
    const float s = __uint_as_float(b << 23);                 // 2^(b - 127)
    const __nv_fp8x2_storage_t h = __nv_cvt_float2_to_fp8x2(make_float2(v0 * inv, v1 * inv), __NV_SATFINITE, __NV_E4M3);
    const float r0 = v0 - e4m3_to_f32(h & 0xFFu) * s;
    const float r1 = v1 - e4m3_to_f32(h >> 8) * s;
    const float inv_lo = inv * 16.0f;
    const __nv_fp8x2_storage_t l = __nv_cvt_float2_to_fp8x2(make_float2(r0 * inv_lo, r1 * inv_lo), __NV_SATFINITE, __NV_E4M3);
    hi2 = h;
    lo2 = l;
}

// Row stride of a split plane: K code bytes, then one 16-byte slot per 128-element
// K step whose first 4 bytes are the step's four block scales (block j in byte j).
__host__ __device__ __forceinline__ int64_t split_row_bytes(int64_t K) { return K + 16 * ((K + 127) / 128); }

// Gather rows into expert order and split them (the first projection's B operand):
//   row r (expert order) = x[sorted_pairs[r] / k] (times the pair's router weight,
//   rounded to bf16, when the weight goes on the input)
//   xq[0][r][c], xq[1][r][c] (c < K): hi and lo terms (E4M3), planes of P rows of
//   split_row_bytes(K) bytes; xq[z][r][K + 16 st + j]: E8M0 byte of block j of step
//   st for that term (blocks past K hold 127).
// One warp per (row, step); lane i holds elements 4i .. 4i + 3 of the step.
__global__ void __launch_bounds__(256) split_rows_kernel(
    const uint16_t *__restrict__ x, const float *__restrict__ weights,
    const int32_t *__restrict__ sorted_pairs, const int32_t *__restrict__ offsets, int E, int k,
    int64_t K, int64_t P, int weight_on_input, uint8_t *__restrict__ xq) {
    pdl_wait();
    pdl_trigger();
    const int rows = offsets[E];
    const int lane = threadIdx.x & 31;
    const int64_t steps = (K + 127) / 128;
    const int64_t RS = split_row_bytes(K);
    const int64_t items = (int64_t)rows * steps;
    const int wpb = blockDim.x >> 5;
    for (int64_t it = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); it < items; it += (int64_t)gridDim.x * wpb) {
        const int64_t r = it / steps;
        const int64_t st = it - r * steps;
        const int p = __ldg(sorted_pairs + r);
        if (!in_bounds(r, P) || !in_bounds(p, P)) continue;   // warp-uniform (one item per warp)
        const int64_t c = st * 128 + 4 * lane;
        const bool in = c < K;                               // K is a multiple of 32
        uint2 raw = make_uint2(0u, 0u);
        if (in) raw = __ldg(reinterpret_cast<const uint2 *>(x + (int64_t)(p / k) * K + c));
        if (weight_on_input && in) {
            const float w = __ldg(weights + p);
            raw.x = pack_bf16x2(bf16lo_to_f32(raw.x) * w, bf16hi_to_f32(raw.x) * w);
            raw.y = pack_bf16x2(bf16lo_to_f32(raw.y) * w, bf16hi_to_f32(raw.y) * w);
        }
        const float v0 = bf16lo_to_f32(raw.x), v1 = bf16hi_to_f32(raw.x);
        const float v2 = bf16lo_to_f32(raw.y), v3 = bf16hi_to_f32(raw.y);
        float amax = fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3)));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 4));
        const uint32_t b = split_scale_byte(amax);
        uint32_t h01, l01, h23, l23;
        split_pair(v0, v1, b, h01, l01);
        split_pair(v2, v3, b, h23, l23);
        uint8_t *hi_row = xq + r * RS;
        uint8_t *lo_row = xq + (P + r) * RS;
        if (in) {
            *reinterpret_cast<uint32_t *>(hi_row + c) = h01 | (h23 << 16);
            *reinterpret_cast<uint32_t *>(lo_row + c) = l01 | (l23 << 16);
        }
        // lanes 0, 8, 16, 24 hold the four blocks' bytes
        const uint32_t mine = in ? b : 127u;
        const uint32_t b1 = __shfl_sync(0xFFFFFFFFu, mine, 8);
        const uint32_t b2 = __shfl_sync(0xFFFFFFFFu, mine, 16);
        const uint32_t b3 = __shfl_sync(0xFFFFFFFFu, mine, 24);
        if (lane == 0) {
            const uint32_t word = mine | (b1 << 8) | (b2 << 16) | (b3 << 24);
            *reinterpret_cast<uint4 *>(hi_row + K + 16 * st) = make_uint4(word, 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(lo_row + K + 16 * st) = make_uint4(__vsubus4(word, 0x04040404u), 0u, 0u, 0u);
        }
    }
}

}  // namespace moe
