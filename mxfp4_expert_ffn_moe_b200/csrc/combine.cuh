// combine.cuh -- per-token sum of the k expert rows, in slot order.
//
// out[t] = sum_{j < k} yp[t*k + j], where yp already carries the routing weight
// applied to the biased expert output (sum w*(y + b), FreeToken PR #838 review
// "NVFP4 down scale vs. down bias"; with the router weight on the input the rows
// are unweighted).  Fixed j order in fp32, one bf16 rounding at the end, so the
// result is reproducible run to run.  Slots whose expert id is outside [0, E)
// were dropped by the permutation and contribute nothing.
#pragma once
#include "common.cuh"

namespace moe {

__global__ void __launch_bounds__(256) combine_rows_kernel(const float *__restrict__ yp,
                                                           const int32_t *__restrict__ ids,
                                                           int64_t T, int k, int E, int64_t H,
                                                           uint16_t *__restrict__ out) {
    pdl_wait();
    pdl_trigger();
    const int64_t q = H / 4;
    const int64_t n = T * q;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / q, c = i - t * q;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int e = __ldg(ids + t * k + j);
            if ((unsigned)e >= (unsigned)E) continue;
            const float4 v = __ldcs(reinterpret_cast<const float4 *>(yp + (t * k + j) * H) + c);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        uint2 o;
        o.x = pack_bf16x2(s.x, s.y);
        o.y = pack_bf16x2(s.z, s.w);
        reinterpret_cast<uint2 *>(out + t * H)[c] = o;
    }
}

// out[t] = sum_{j < k} y_rows[pair_rows[t*k + j]] in slot order (fp32, one bf16
// rounding), skipping pairs whose row is -1 (dropped): the combine of rows that come
// back in expert order, e.g. from the ranks that own their experts.
__global__ void __launch_bounds__(256) combine_pair_rows_kernel(const float *__restrict__ y_rows,
                                                                const int32_t *__restrict__ pair_rows,
                                                                int64_t T, int k, int64_t H,
                                                                uint16_t *__restrict__ out) {
    pdl_wait();
    pdl_trigger();
    const int64_t q = H / 4;
    const int64_t n = T * q;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / q, c = i - t * q;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int r = __ldg(pair_rows + t * k + j);
            if (r < 0 || !in_bounds(r, T * k)) continue;
            const float4 v = __ldcs(reinterpret_cast<const float4 *>(y_rows + (int64_t)r * H) + c);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        uint2 o;
        o.x = pack_bf16x2(s.x, s.y);
        o.y = pack_bf16x2(s.z, s.w);
        reinterpret_cast<uint2 *>(out + t * H)[c] = o;
    }
}

}  // namespace moe
