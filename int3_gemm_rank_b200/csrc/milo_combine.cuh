// milo_combine.cuh -- the weighted un-permute of the MoE layer's expert
// outputs back to token order (or, for the grouped linear, the copy of each
// routed slot's row), four output columns at a time (the combine kernel).
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators", "Background": an MoE layer sends each token to a subset of
// its experts and mixes their outputs with the router's weights.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "milo_device.cuh"
#include "milo_kernels.h"

namespace milo {

// Sum over the split-K partials of one row, columns n..n+3, in split order
// (L2 loads: the partials come from the previous kernel), four loads in
// flight at a time.
__device__ __forceinline__ float4 split_sum4(const float* part, int splits, size_t split_stride, size_t off) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < splits; s0 += 4) {
        float4 v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (s0 + q < splits) v[q] = __ldcg(reinterpret_cast<const float4*>(part + (s0 + q) * split_stride + off));
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (s0 + q < splits) {
                if (s0 + q == 0) {
                    a = v[0];
                } else {
                    a.x += v[q].x; a.y += v[q].y; a.z += v[q].z; a.w += v[q].w;
                }
            }
    }
    return a;
}

// Output row o, columns n..n+3: per slot (grouped linear) the slot's row, or
// per token the router-weighted sum over its slots in slot order, then the
// shared experts in order.
__device__ __forceinline__ float4 combine4(const CombineParams& p, int o, int n) {
    const size_t sstride = static_cast<size_t>(p.R) * p.H;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.per_slot) {
        const int r = p.inv_perm[o];
        if (r >= 0 && in_range(p.dev_status, r < p.R))
            acc = split_sum4(p.y_part, p.splits, sstride, static_cast<size_t>(r) * p.H + n);
        return acc;
    }
    if (p.splits == 1) {
        // one partial per slot: eight slots at a time, their rows and weights
        // first, then all their partial rows in flight at once, added in slot
        // order
        for (int j0 = 0; j0 < p.k; j0 += 8) {
            int rows[8];
            float wts[8];
            float4 v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j0 + j < p.k) {
                    const int f = o * p.k + j0 + j;
                    rows[j] = p.inv_perm[f];
                    wts[j] = p.w[f];
                }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j0 + j < p.k && rows[j] >= 0 && rows[j] < p.R_routed)
                    v[j] = __ldcg(reinterpret_cast<const float4*>(p.y_part + static_cast<size_t>(rows[j]) * p.H + n));
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j0 + j < p.k && rows[j] >= 0 && rows[j] < p.R_routed) {
                    acc.x = fmaf(wts[j], v[j].x, acc.x);
                    acc.y = fmaf(wts[j], v[j].y, acc.y);
                    acc.z = fmaf(wts[j], v[j].z, acc.z);
                    acc.w = fmaf(wts[j], v[j].w, acc.w);
                }
        }
    } else {
        for (int j = 0; j < p.k; ++j) {
            const int f = o * p.k + j;
            const int r = p.inv_perm[f];
            if (r < 0 || r >= p.R_routed) continue;
            const float wj = p.w[f];
            const float4 v = split_sum4(p.y_part, p.splits, sstride, static_cast<size_t>(r) * p.H + n);
            acc.x = fmaf(wj, v.x, acc.x);
            acc.y = fmaf(wj, v.y, acc.y);
            acc.z = fmaf(wj, v.z, acc.z);
            acc.w = fmaf(wj, v.w, acc.w);
        }
    }
    for (int s = 0; s < p.S; ++s) {
        if (!in_range(p.dev_status, p.R_routed + s * p.T + o < p.R)) break;
        const float4 v = split_sum4(p.y_part, p.splits, sstride, static_cast<size_t>(p.R_routed + s * p.T + o) * p.H + n);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    return acc;
}

// Store four output values in the output type (FP16_RANGE for an fp16 overflow).
__device__ __forceinline__ void store4(const CombineParams& p, size_t off, float4 acc, int32_t& st) {
    if (p.y_dt == MILO_F32) {
        *reinterpret_cast<float4*>(static_cast<float*>(p.y) + off) = acc;
    } else if (p.y_dt == MILO_F16) {
        const __half2 lo = __floats2half2_rn(acc.x, acc.y), hi = __floats2half2_rn(acc.z, acc.w);
        if (__hisinf(lo.x) || __hisinf(lo.y) || __hisinf(hi.x) || __hisinf(hi.y)) st |= MILO_DEV_FP16_RANGE;
        __half2* dst = reinterpret_cast<__half2*>(static_cast<__half*>(p.y) + off);
        dst[0] = lo;
        dst[1] = hi;
    } else {
        __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.y) + off);
        dst[0] = __floats2bfloat162_rn(acc.x, acc.y);
        dst[1] = __floats2bfloat162_rn(acc.z, acc.w);
    }
}

}  // namespace milo
