// common.cuh -- small device helpers shared by the layer's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define MOE_DEVERR_BAD_EXPERT_ID 0x1
#define MOE_DEVERR_BAD_SCALE 0x2
#define MOE_DEVERR_TIMEOUT 0x4
#define MOE_DEVERR_BAD_LOGIT 0x8
#define MOE_DEVERR_OUT_OF_BOUNDS 0x10

namespace moe {

// Sticky per-device error word (one per loaded module, i.e. per device).
__device__ int g_device_error;

__device__ __forceinline__ void raise_device_error(int bits) { atomicOr(&g_device_error, bits); }

// Bounds-checked builds (MOE_CHECKED=1, a debugging variant of the library): every
// data-dependent global index is tested against its buffer's extent before the
// access; an index outside [0, n) raises MOE_DEVERR_OUT_OF_BOUNDS and the access is
// skipped (never a trap).  In the normal build the test is compiled away.
#ifndef MOE_CHECKED
#define MOE_CHECKED 0
#endif
__device__ __forceinline__ bool in_bounds(int64_t idx, int64_t n) {
    if constexpr (MOE_CHECKED) {
        if (idx < 0 || idx >= n) {
            raise_device_error(MOE_DEVERR_OUT_OF_BOUNDS);
            return false;
        }
    }
    return true;
}
// [lo, hi) within [0, n)
__device__ __forceinline__ bool range_in_bounds(int64_t lo, int64_t hi, int64_t n) {
    if constexpr (MOE_CHECKED) {
        if (lo < 0 || hi > n || lo > hi) {
            raise_device_error(MOE_DEVERR_OUT_OF_BOUNDS);
            return false;
        }
    }
    return true;
}

// fp32 value of an E8M0 scale byte: 2^(s - 127).  s = 0 is the fp32 subnormal
// 2^-127; s = 0xff is not a number (invalid per the MXFP4 validation rules).
__device__ __forceinline__ float e8m0_to_f32(uint32_t s) {
    if (s == 0u) return __uint_as_float(0x00400000u);
    if (s == 255u) return __uint_as_float(0x7FC00000u);
    return __uint_as_float(s << 23);
}

// Two fp32 values -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Clamped SwiGLU of the gpt-oss expert MLP:
//   g = min(gate, limit), u = clamp(up, -limit, limit), a = (u + 1) * g * sigmoid(alpha g).
// The sigmoid uses the hardware exponential and reciprocal intrinsics; their
// relative error (~1e-6) is far below the bf16 rounding the result receives.
// For very negative g, exp overflows to +inf and the quotient is 0, so a -> -0.
__device__ __forceinline__ float clamped_swiglu(float gate, float up, float alpha, float limit) {
    const float g = fminf(gate, limit);
    const float u = fminf(fmaxf(up, -limit), limit);
    const float sig = __fdividef(1.0f, 1.0f + __expf(-alpha * g));
    return (u + 1.0f) * (g * sig);
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Programmatic dependent launch.  pdl_wait(): block until the preceding kernel of
// the stream has completed and its writes are visible (returns at once when this
// kernel was launched without the programmatic-serialisation attribute); every
// kernel of the layer calls it before its first read of data a predecessor writes
// and before its first global write.  pdl_trigger(): let the next kernel of the
// stream be scheduled now (its blocks start as resources free up and then wait in
// their own pdl_wait), hiding launch latency and prologues.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace moe
