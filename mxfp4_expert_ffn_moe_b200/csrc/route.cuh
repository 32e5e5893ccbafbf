// route.cuh -- top-k routing: k largest router logits, then softmax over those k.
//
// The MXFP4 experts take routing data -- expert ids plus routing weights -- rather
// than a dispatch of expert ids (transformers PR #49431 "Restore GPT-OSS's
// router-masked expert-parallel plan").  Selection order: value descending, ties
// to the lower expert index.  Weights: exp(l_j - l_max) / sum_i exp(l_i - l_max)
// over the k chosen logits, in fp32.
//
// One warp per token; each lane holds VPL logits (expert lane + 32 v) in
// registers, k rounds of a warp-wide arg-max with the (value desc, index asc) rule.
// NaN logits are never chosen; a token with fewer than k other logits gets id -1
// and weight 0 in its remaining slots and raises MOE_DEVERR_BAD_LOGIT.
#pragma once
#include "common.cuh"

namespace moe {

template <int VPL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ logits,
                                                         int64_t T, int E, int k,
                                                         int32_t *__restrict__ ids,
                                                         float *__restrict__ weights) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *row = logits + t * E;
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? __ldg(row + e) : -INFINITY;
    }
    uint32_t taken = 0;  // bit i: slot i of this lane already chosen (or absent)
#pragma unroll
    for (int i = 0; i < VPL; ++i)
        if (lane + 32 * i >= E) taken |= 1u << i;

    float sel_v[8];
    int sel_i[8];
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = lane + 32 * i;
            const bool ok = !((taken >> i) & 1u);
            if (ok && (v[i] > bv || (v[i] == bv && e < bi))) {
                bv = v[i];
                bi = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        // bi == E-or-more only when every remaining logit is NaN (a NaN never wins a
        // comparison): the slot stays empty
        if (bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
        sel_v[j] = bv;
        sel_i[j] = bi;
    }
    if (lane == 0) {
        // empty slots (fewer than k non-NaN logits) get id -1 and weight 0 and flag
        // the device error word; the softmax runs over the chosen logits only
        const float m = sel_v[0];
        float ex[8], sum = 0.0f;
        for (int j = 0; j < k; ++j) {
            ex[j] = sel_i[j] < E ? expf(sel_v[j] - m) : 0.0f;
            sum += ex[j];
        }
        const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
        for (int j = 0; j < k; ++j) {
            const bool valid = sel_i[j] < E;
            if (!valid) raise_device_error(MOE_DEVERR_BAD_LOGIT);
            ids[t * k + j] = valid ? sel_i[j] : -1;
            weights[t * k + j] = ex[j] * inv;
        }
    }
}

}  // namespace moe
