// dequant.cuh -- standalone dequant-on-copy: packed MXFP4 bank -> bf16.
//
// MoE-Infinity PR #152 "expert offloading Phase 2 -- MXFP4 dequant-on-copy
// execution", Changes: mxfp4_dequantize turns fetched packed experts into bf16
// (golden rel-err 0.0, i.e. exact).  Element kk of a row sits in byte kk/2 (even
// element in the low nibble) and is scaled by the E8M0 byte kk/32 of that row.
//
// HBM-bound streaming kernel with a write-heavy mix (4.25 bits read per 16 written).
// Each thread decodes one 32-bit packed word (eight codes, a quarter of a 32-element
// scale block) with integer operations and packed bf16 multiplies, no table: the
// codes become the bf16 bit patterns of E2M1 * 2^-126 (sign to bit 15, exponent bits
// and mantissa msb to bits 8..6; code 1 = 0.5 is the subnormal 2^-127), then one bf16
// multiply by 2^(s-1) (two, by 2^126 and 2^(s-127), when s > 128) gives
// E2M1 * 2^(s-127), rounded to nearest even only where that is a bf16 subnormal or
// overflows -- the exact product otherwise.  A block of 256 threads decodes 1024
// consecutive words into 16 KB of shared memory and one bulk asynchronous copy writes
// it out (double-buffered); reads are coalesced 4-byte loads.  Measured on the
// gpt-oss-20b bank: bulk stores of 16 KB runs beat direct 16-byte stores by ~7 %, and
// one 16-byte load plus four strided 16-byte stores per thread lose ~30 %.
//
// Both decode kernels also serve dequant-on-copy from host memory (kHostSrc): the
// packed bank stays in page-locked host memory, the kernel reads it through its
// device mapping with plain coherent loads, so only the packed codes cross the host
// link and the bf16 weights land directly in device memory.
#pragma once
#include "common.cuh"

namespace moe {

// Packed-bank reads: the read-only path for device memory, plain global loads for
// mapped host memory.
template <bool kHostSrc>
__device__ __forceinline__ uint32_t load_word(const uint32_t *p) {
    if constexpr (kHostSrc) {
        uint32_t v;
        asm volatile("ld.global.u32 %0, [%1];" : "=r"(v) : "l"(p));
        return v;
    } else {
        return __ldg(p);
    }
}

template <bool kHostSrc>
__device__ __forceinline__ uint32_t load_byte(const uint8_t *p) {
    if constexpr (kHostSrc) {
        uint32_t v;
        asm volatile("ld.global.u8 %0, [%1];" : "=r"(v) : "l"(p));
        return v;
    } else {
        return __ldg(p);
    }
}

// Eight E2M1 codes (element 2j in the low nibble of byte j) -> four bf16x2 words of
// E2M1 * 2^(s - 127) for the multipliers of scale_multipliers.
__device__ __forceinline__ uint4 e2m1x8_scaled(uint32_t q, uint32_t m1, uint32_t m2) {
    const uint32_t lo = q & 0x0F0F0F0Fu, hi = (q >> 4) & 0x0F0F0F0Fu;
    uint32_t r[4];
    asm("prmt.b32 %0, %1, %2, 0x8480;" : "=r"(r[0]) : "r"(lo), "r"(hi));
    asm("prmt.b32 %0, %1, %2, 0x8581;" : "=r"(r[1]) : "r"(lo), "r"(hi));
    asm("prmt.b32 %0, %1, %2, 0x8682;" : "=r"(r[2]) : "r"(lo), "r"(hi));
    asm("prmt.b32 %0, %1, %2, 0x8783;" : "=r"(r[3]) : "r"(lo), "r"(hi));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        r[i] = (r[i] * 0x1040u) & 0x81C081C0u;   // sign, exponent bits, mantissa msb
        asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r[i]) : "r"(r[i]), "r"(m1));
        if (m2) asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r[i]) : "r"(r[i]), "r"(m2));
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// bf16x2 multipliers taking E2M1 * 2^-126 to E2M1 * 2^(s - 127): one (2^(s - 1)) when
// that is a normal bf16, else 2^126 then 2^(s - 127).
__device__ __forceinline__ void scale_multipliers(uint32_t s, uint32_t &m1, uint32_t &m2) {
    if (s <= 128u) {
        m1 = ((s + 126u) << 7) * 0x10001u;
        m2 = 0u;
    } else {
        m1 = 0x7E807E80u;
        m2 = (s << 7) * 0x10001u;
    }
}

template <bool kHostSrc>
__device__ __forceinline__ uint4 dequant_word(uint32_t q, uint32_t s) {
    if (s == 255u) {   // invalid scale byte: NaN and the device error word
        raise_device_error(MOE_DEVERR_BAD_SCALE);
        return make_uint4(0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u);
    }
    uint32_t m1, m2;
    scale_multipliers(s, m1, m2);
    return e2m1x8_scaled(q, m1, m2);
}

constexpr int kDequantThreads = 256;
constexpr int kDequantWords = 4 * kDequantThreads;   // words per round (16 KB of bf16)

// Block b decodes words [b * words_per_block, (b + 1) * words_per_block) of the bank
// (words_per_block a multiple of kDequantWords); each round's 16 KB leaves with one
// bulk copy from shared memory.
template <bool kHostSrc>
__global__ void __launch_bounds__(kDequantThreads) mxfp4_dequant_kernel(const uint32_t *__restrict__ packed,
                                                                        const uint8_t *__restrict__ scales,
                                                                        uint4 *__restrict__ out, int64_t n_words,
                                                                        int64_t words_per_block) {
    __shared__ __align__(128) uint4 stage[2][kDequantWords];
    const int64_t w0 = (int64_t)blockIdx.x * words_per_block;
    const int64_t w1 = min(n_words, w0 + words_per_block);
    int round = 0;
    for (int64_t base = w0; base < w1; base += kDequantWords, ++round) {
        const int b = round & 1;
        if (round >= 2) {
            // the copy that read this buffer two rounds ago has finished reading it
            if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            __syncthreads();
        }
        const int64_t n = min((int64_t)kDequantWords, w1 - base);
        uint32_t q[4], sb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t i = base + threadIdx.x + kDequantThreads * u;
            q[u] = i < w1 ? load_word<kHostSrc>(packed + i) : 0u;
            sb[u] = i < w1 ? load_byte<kHostSrc>(scales + (i >> 2)) : 127u;   // 4 words per scale block
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) stage[b][threadIdx.x + kDequantThreads * u] = dequant_word<kHostSrc>(q[u], sb[u]);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (threadIdx.x == 0) {
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(out + base),
                         "r"((uint32_t)__cvta_generic_to_shared(&stage[b][0])), "r"((uint32_t)(n * 16))
                         : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
    }
    // the copies must have read shared memory before the block exits
    if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ---- NVFP4 ------------------------------------------------------------------
// NVFP4 expert banks: the same packed E2M1 codes, one E4M3 scale byte per 16
// elements ([E, N, K/16]; OCP OFP8 v1.0: bias 7, 3 mantissa bits, subnormals
// m/8 * 2^-6, S.1111.111 = NaN) and one fp32 weight_scale_2 per expert (FreeToken
// PR #838, review item "NVFP4 down scale vs. down bias").

// fp32 value of an E4M3 byte (exact); NaN for S.1111.111.
__device__ __forceinline__ float e4m3_byte_value(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u, sign = (b & 0x80u) << 24;
    if (e == 15u && m == 7u) return __uint_as_float(0x7FC00000u);
    const float mag = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0x1p-9f;
    return __uint_as_float(__float_as_uint(mag) | sign);
}

// Sticky bit for a truncated product p = RZ(v * s) that sits exactly on a bf16 tie:
// set the last bit when v * s was inexact, so that the bf16 rounding goes up (in
// magnitude) as the exact product does.  v has at most 6 significant bits, so the
// exact product has at most 30: the fma residual is exact while |p| >= 2^-118; below
// that the product is formed in double, where it is exact.
__device__ __noinline__ uint32_t tie_sticky(float v, float s, uint32_t b) {
    const float p = __uint_as_float(b);
    bool inexact;
    if (fabsf(p) >= 0x1p-118f) {
        inexact = __fmaf_rn(v, s, -p) != 0.0f;
    } else {
        const double d = (double)v * (double)s;
        inexact = (double)p != d;
    }
    return inexact ? (b | 1u) : b;
}

// v * s (v with at most 6 significant bits, both finite) as an fp32 whose
// round-to-nearest-even conversion to bf16 equals rounding the exact product once.
// Truncating to fp32 keeps the product on the same side of every bf16 rounding
// boundary unless the truncated value lands exactly on a tie (low 16 bits 0x8000),
// where the sticky bit decides; this is round-to-odd (Boldo and Melquiond,
// "Emulation of FMA and correctly rounded sums: proved algorithms using rounding to
// odd", IEEE Trans. Computers 57(4), 2008) applied only where it can matter.
__device__ __forceinline__ float mul_for_bf16(float v, float s) {
    const uint32_t b = __float_as_uint(__fmul_rz(v, s));
    return __uint_as_float((b & 0xFFFFu) == 0x8000u ? tie_sticky(v, s, b) : b);
}

// Two fp32 values -> bf16x2; NaN as 0x7fc0 (the slow path for non-finite scale2).
__device__ __forceinline__ uint32_t pack_bf16x2_canon(float lo, float hi) {
    uint32_t r = pack_bf16x2(lo, hi);
    if (lo != lo) r = (r & 0xFFFF0000u) | 0x7FC0u;
    if (hi != hi) r = (r & 0x0000FFFFu) | 0x7FC00000u;
    return r;
}

// out[e, n, kk] = bf16(E2M1(code) * E4M3(scale[e, n, kk/16]) * scale2[e]), rounded
// once from the exact product; scale2 == nullptr means 1.  Grid: x strides over the
// words of one expert, y over experts, so weight_scale_2 is one load per block.
// Each thread turns one 32-bit word (eight codes, half a 16-element block) into one
// 16-byte bf16 chunk.  Paths: scale2 == 1 (products exact, plain conversion),
// finite scale2 (mul_for_bf16), non-finite scale2 (canonical NaNs); a NaN scale
// byte makes its whole word NaN and flags the device error word.
__device__ __forceinline__ uint4 nvfp4_word(uint32_t q, uint32_t sb, const float *lut, float s2, int mode) {
    if ((sb & 0x7Fu) == 0x7Fu) {
        raise_device_error(MOE_DEVERR_BAD_SCALE);
        return make_uint4(0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u);
    }
    const float sc = e4m3_byte_value(sb);
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float a = lut[(q >> (8 * j)) & 15u] * sc;          // exact: <= 6 significant bits
        float b = lut[(q >> (8 * j + 4)) & 15u] * sc;
        if (mode == 0) {
            o[j] = pack_bf16x2(a, b);
        } else if (mode == 1) {
            o[j] = pack_bf16x2(mul_for_bf16(a, s2), mul_for_bf16(b, s2));
        } else {
            o[j] = pack_bf16x2_canon(a * s2, b * s2);      // inf / NaN scale2: no rounding left
        }
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <bool kHostSrc>
__global__ void __launch_bounds__(256) nvfp4_dequant_kernel(const uint32_t *__restrict__ packed,
                                                            const uint8_t *__restrict__ scales,
                                                            const float *__restrict__ scale2,
                                                            uint4 *__restrict__ out,
                                                            int64_t words_per_expert, int64_t E) {
    __shared__ float lut[16];
    if (threadIdx.x < 16) {
        const uint32_t c = threadIdx.x, e = (c >> 1) & 3u, m = c & 1u;
        float mag = (e == 0u) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, (int)e - 1);
        lut[c] = (c & 8u) ? -mag : mag;
    }
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = blockIdx.y; e < E; e += gridDim.y) {
        const float s2 = scale2 ? __ldg(scale2 + e) : 1.0f;
        const int mode = s2 == 1.0f ? 0 : (isfinite(s2) ? 1 : 2);   // uniform over the block
        const uint32_t *src = packed + e * words_per_expert;
        const uint8_t *sc_e = scales + e * (words_per_expert >> 1);   // 2 words per 16-element block
        uint4 *dst = out + e * words_per_expert;
        constexpr int U = 4;
        int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        for (; w + (U - 1) * stride < words_per_expert; w += U * stride) {
            uint32_t word[U], sb[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                word[u] = load_word<kHostSrc>(src + w + u * stride);
                sb[u] = load_byte<kHostSrc>(sc_e + ((w + u * stride) >> 1));
            }
#pragma unroll
            for (int u = 0; u < U; ++u) __stcs(dst + w + u * stride, nvfp4_word(word[u], sb[u], lut, s2, mode));
        }
        for (; w < words_per_expert; w += stride)
            __stcs(dst + w, nvfp4_word(load_word<kHostSrc>(src + w), load_byte<kHostSrc>(sc_e + (w >> 1)), lut,
                                       s2, mode));
    }
}

}  // namespace moe
