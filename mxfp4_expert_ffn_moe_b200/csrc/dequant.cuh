// dequant.cuh -- standalone dequant-on-copy: packed MXFP4 bank -> bf16.
//
// MoE-Infinity PR #152 "expert offloading Phase 2 -- MXFP4 dequant-on-copy
// execution", Changes: mxfp4_dequantize turns fetched packed experts into bf16
// (golden rel-err 0.0, i.e. exact).  Element kk of a row sits in byte kk/2 (even
// element in the low nibble) and is scaled by the E8M0 byte kk/32 of that row.
//
// HBM-bound streaming kernel.  Each thread turns one 32-bit packed word (eight
// codes, a quarter of a 32-element scale block) into one 16-byte bf16 chunk, so a
// warp reads 128 contiguous bytes and writes 512 contiguous bytes per step.  The
// E2M1 magnitudes come from a 16-entry fp32 table in shared memory (16 distinct
// banks: no conflicts); values are scaled by an exact fp32 power of two and
// rounded to bf16, which never rounds for scale bytes <= 252 and gives the bf16
// subnormals / infinities of the exact product for the extreme bytes.
#pragma once
#include "common.cuh"

namespace moe {

__global__ void __launch_bounds__(256) mxfp4_dequant_kernel(const uint32_t *__restrict__ packed,
                                                            const uint8_t *__restrict__ scales,
                                                            uint4 *__restrict__ out,
                                                            int64_t n_words) {
    __shared__ float lut[16];
    if (threadIdx.x < 16) {
        // E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
        const uint32_t c = threadIdx.x, e = (c >> 1) & 3u, m = c & 1u;
        float mag = (e == 0u) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, (int)e - 1);
        lut[c] = (c & 8u) ? -mag : mag;
    }
    __syncthreads();

    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    constexpr int U = 4;
    for (; w + (U - 1) * stride < n_words; w += U * stride) {
        uint32_t word[U], s[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            word[u] = __ldg(packed + w + u * stride);
            s[u] = __ldg(scales + ((w + u * stride) >> 2));  // 4 words per 32-element block
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            uint4 v;
            if (s[u] == 255u) {
                raise_device_error(MOE_DEVERR_BAD_SCALE);
                v = make_uint4(0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u);
            } else {
                const float sc = e8m0_to_f32(s[u]);
                const uint32_t q = word[u];
                v.x = pack_bf16x2(lut[q & 15u] * sc, lut[(q >> 4) & 15u] * sc);
                v.y = pack_bf16x2(lut[(q >> 8) & 15u] * sc, lut[(q >> 12) & 15u] * sc);
                v.z = pack_bf16x2(lut[(q >> 16) & 15u] * sc, lut[(q >> 20) & 15u] * sc);
                v.w = pack_bf16x2(lut[(q >> 24) & 15u] * sc, lut[q >> 28] * sc);
            }
            __stcs(out + w + u * stride, v);
        }
    }
    for (; w < n_words; w += stride) {
        const uint32_t q = __ldg(packed + w);
        const uint32_t sb = __ldg(scales + (w >> 2));
        uint4 v;
        if (sb == 255u) {
            raise_device_error(MOE_DEVERR_BAD_SCALE);
            v = make_uint4(0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u);
        } else {
            const float sc = e8m0_to_f32(sb);
            v.x = pack_bf16x2(lut[q & 15u] * sc, lut[(q >> 4) & 15u] * sc);
            v.y = pack_bf16x2(lut[(q >> 8) & 15u] * sc, lut[(q >> 12) & 15u] * sc);
            v.z = pack_bf16x2(lut[(q >> 16) & 15u] * sc, lut[(q >> 20) & 15u] * sc);
            v.w = pack_bf16x2(lut[(q >> 24) & 15u] * sc, lut[q >> 28] * sc);
        }
        __stcs(out + w, v);
    }
}

}  // namespace moe
