// aux.cu -- the kernels around the grouped int3 GEMM:
//   rows_kernel    routed/shared row bookkeeping from the router's offsets/perm
//   prep_kernel    activations -> fp16 MMA fragments (power-of-8 factors of the
//                  int3 field extraction folded in) and per-group sums
//   lorc_kernel    compensator down-projection t = x V^T per expert
//   combine_kernel weighted un-permute back to token order, split-K reduction
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators": the compensator is a rank-r product U V added to the
// quantised weight ("MiLo Algorithm"), so x (W_q + U V)^T splits into the int3
// GEMM and (x V^T) U^T; the MoE layer combines the routed experts' outputs.
#include <cuda_runtime.h>

#include "milo_device.cuh"
#include "milo_kernels.h"

namespace milo {

// ---------------------------------------------------------------------------
// rows: groups (first row, count) for routed + shared experts, row -> token
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) rows_kernel(const RowsParams p) {
    __shared__ int ok_off[MILO_MAX_EXPERTS + 1];
    const int F = p.T * p.k;
    int32_t st = 0;
    if (threadIdx.x == 0) {
        // Clamp the offsets into a non-decreasing sequence within [0, F].
        int prev = 0;
        for (int e = 0; e <= p.E; ++e) {
            int o = p.offsets[e];
            if (e == 0 && o != 0) st |= MILO_DEV_BAD_EXPERT_ID;
            if (o < prev || o > F) {
                st |= MILO_DEV_BAD_EXPERT_ID;
                o = o < prev ? prev : F;
            }
            ok_off[e] = e == 0 ? 0 : o;
            prev = ok_off[e];
        }
        for (int e = 0; e < p.E; ++e) {
            p.grp[2 * e] = ok_off[e];
            p.grp[2 * e + 1] = ok_off[e + 1] - ok_off[e];
        }
        for (int s = 0; s < p.S; ++s) {
            p.grp[2 * (p.E + s)] = p.R_routed + s * p.T;
            p.grp[2 * (p.E + s) + 1] = p.T;
        }
    }
    __syncthreads();
    const int used = ok_off[p.E];
    if (p.inv)
        for (int f = threadIdx.x; f < F; f += blockDim.x) p.inv[f] = -1;
    __syncthreads();
    for (int r = threadIdx.x; r < p.R_routed; r += blockDim.x) {
        int src = -1;
        if (r < used) {
            const int f = p.perm ? p.perm[r] : r;
            if (f >= 0 && f < F) {
                src = f / p.k;
                if (p.inv) p.inv[f] = r;
            } else {
                st |= MILO_DEV_BAD_EXPERT_ID;
            }
        }
        p.row_src[r] = src;
    }
    for (int r = threadIdx.x; r < p.S * p.T; r += blockDim.x) p.row_src[p.R_routed + r] = r % p.T;
    flag(p.dev_status, st);
}

cudaError_t launch_rows(const RowsParams& p, cudaStream_t s) {
    rows_kernel<<<1, 256, 0, s>>>(p);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// prep: fragment-ordered activations and group sums, one block per row
// ---------------------------------------------------------------------------
template <int S, int H>
__device__ __forceinline__ uint32_t frag_pair(const __half (&x)[32]) {
    constexpr int t = sched_word(S, H), f = sched_field(S, H);
    constexpr int m = reg_code(t, f);
    const __half sc = __float2half_rn(act_scale(t, f));
    const __half lo = __hmul(x[m], sc), hi = __hmul(x[m + 1], sc);
    return static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
}

template <int S>
__device__ __forceinline__ uint2 frag_step(const __half (&x)[32]) {
    return make_uint2(frag_pair<S, 0>(x), frag_pair<S, 1>(x));
}

__global__ void __launch_bounds__(128) prep_kernel(const PrepParams p) {
    const int row = blockIdx.x;
    const int SB = p.K / 128;
    const int src = p.row_src ? p.row_src[row] : row;
    int32_t st = 0;
    for (int base = 0; base < SB * 4; base += blockDim.x) {
        const int idx = base + threadIdx.x;
        const bool active = idx < SB * 4;
        const int sb = idx >> 2, c = idx & 3;
        __half x[32];
        float s0 = 0.0f, s1 = 0.0f;
        if (active && src >= 0) {
            const uint16_t* rowp = p.src + static_cast<size_t>(src) * p.K + 128 * sb;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const uint4* v = reinterpret_cast<const uint4*>(rowp + 64 * half + 16 * c);
                const uint4 u0 = v[0], u1 = v[1];
                const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    x[16 * half + 2 * i] = to_half(static_cast<uint16_t>(w[i] & 0xFFFFu), p.src_bf16, st);
                    x[16 * half + 2 * i + 1] = to_half(static_cast<uint16_t>(w[i] >> 16), p.src_bf16, st);
                }
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) s0 += __half2float(x[m]);
#pragma unroll
            for (int m = 16; m < 32; ++m) s1 += __half2float(x[m]);
        } else {
#pragma unroll
            for (int m = 0; m < 32; ++m) x[m] = __ushort_as_half(0);
        }
        // group sums over the four units of the super-block (lanes 4j..4j+3)
        s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
        s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 2);
        s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
        s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 2);
        if (!active) continue;
        if (c == 0) {
            p.gsum[static_cast<size_t>(row) * p.gpad + 2 * sb] = s0;
            p.gsum[static_cast<size_t>(row) * p.gpad + 2 * sb + 1] = s1;
        }
        uint2* out = reinterpret_cast<uint2*>(p.frag + (static_cast<size_t>(row) * SB + sb) * kFragHalvesPerSB) + c;
        out[0 * 4] = frag_step<0>(x);
        out[1 * 4] = frag_step<1>(x);
        out[2 * 4] = frag_step<2>(x);
        out[3 * 4] = frag_step<3>(x);
        out[4 * 4] = frag_step<4>(x);
        out[5 * 4] = frag_step<5>(x);
        out[6 * 4] = frag_step<6>(x);
        out[7 * 4] = frag_step<7>(x);
        out[8 * 4] = frag_step<8>(x);
    }
    for (int j = 2 * SB + threadIdx.x; j < p.gpad; j += blockDim.x)
        p.gsum[static_cast<size_t>(row) * p.gpad + j] = 0.0f;
    flag(p.dev_status, st);
}

cudaError_t launch_prep(const PrepParams& p, cudaStream_t s) {
    if (p.R <= 0) return cudaSuccess;
    prep_kernel<<<p.R, 128, 0, s>>>(p);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// lorc: t[p, col0 + j] = sum_k x[p, k] V[j, k] for the rows of each expert,
// one block per (expert, projection, 16-rank block); four warps split K and
// the partial tiles are added in a fixed order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t load_x_pair(const uint16_t* row, int k, bool bf16, int32_t& st) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(row + k);
    const __half lo = to_half(static_cast<uint16_t>(w & 0xFFFFu), bf16, st);
    const __half hi = to_half(static_cast<uint16_t>(w >> 16), bf16, st);
    return static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
}

__global__ void __launch_bounds__(128) lorc_kernel(const LorcParams p, int rank_blocks) {
    __shared__ float part[4][16][17];
    const int nproj = p.proj_b >= 0 ? 2 : 1;
    const int e = blockIdx.x / (nproj * rank_blocks);
    const int rem = blockIdx.x % (nproj * rank_blocks);
    const int which = rem / rank_blocks, rblk = rem % rank_blocks;
    const ProjDev* P = p.table + e * p.stride + (which == 0 ? p.proj_a : p.proj_b);
    const int r = P->rank;
    const int j0 = 16 * rblk;
    if (j0 >= r) return;
    const int row0 = p.grp[2 * e], m = p.grp[2 * e + 1];
    if (m <= 0 || row0 < 0 || row0 + m > p.R) return;
    const int col0 = which == 0 ? 0 : p.t_col_b;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int kq = p.K / 4;   // K is a multiple of 128
    const int kbeg = warp * kq;
    int32_t st = 0;
    for (int mt = 0; mt < m; mt += 16) {
        float acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
        const int ra = mt + g, rb = mt + g + 8;
        const int sa = ra < m ? (p.row_src ? p.row_src[row0 + ra] : row0 + ra) : -1;
        const int sb_ = rb < m ? (p.row_src ? p.row_src[row0 + rb] : row0 + rb) : -1;
        const uint16_t* xa = sa >= 0 ? p.src + static_cast<size_t>(sa) * p.K : nullptr;
        const uint16_t* xb = sb_ >= 0 ? p.src + static_cast<size_t>(sb_) * p.K : nullptr;
        const uint16_t* v0 = (j0 + g < r) ? P->V + static_cast<size_t>(j0 + g) * p.K : nullptr;
        const uint16_t* v1 = (j0 + 8 + g < r) ? P->V + static_cast<size_t>(j0 + 8 + g) * p.K : nullptr;
        for (int k = kbeg; k < kbeg + kq; k += 16) {
            const int kc = k + 2 * c;
            const uint32_t a0 = xa ? load_x_pair(xa, kc, p.src_bf16, st) : 0u;
            const uint32_t a1 = xb ? load_x_pair(xb, kc, p.src_bf16, st) : 0u;
            const uint32_t a2 = xa ? load_x_pair(xa, kc + 8, p.src_bf16, st) : 0u;
            const uint32_t a3 = xb ? load_x_pair(xb, kc + 8, p.src_bf16, st) : 0u;
            const uint32_t b00 = v0 ? *reinterpret_cast<const uint32_t*>(v0 + kc) : 0u;
            const uint32_t b01 = v0 ? *reinterpret_cast<const uint32_t*>(v0 + kc + 8) : 0u;
            const uint32_t b10 = v1 ? *reinterpret_cast<const uint32_t*>(v1 + kc) : 0u;
            const uint32_t b11 = v1 ? *reinterpret_cast<const uint32_t*>(v1 + kc + 8) : 0u;
            mma16816(acc[0], a0, a1, a2, a3, b00, b01);
            mma16816(acc[1], a0, a1, a2, a3, b10, b11);
        }
        // acc[h][i]: row g + 8*(i>>1), rank 8h + 2c + (i&1)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 4; ++i) part[warp][g + 8 * (i >> 1)][8 * h + 2 * c + (i & 1)] = acc[h][i];
        __syncthreads();
        for (int idx = threadIdx.x; idx < 256; idx += blockDim.x) {
            const int rr = idx / 16, jj = idx % 16;
            const float v = ((part[0][rr][jj] + part[1][rr][jj]) + part[2][rr][jj]) + part[3][rr][jj];
            if (mt + rr < m && j0 + jj < r)
                p.t[static_cast<size_t>(row0 + mt + rr) * p.tcols + col0 + j0 + jj] =
                    __half_as_ushort(__float2half_rn(v));
        }
        __syncthreads();
    }
    flag(p.dev_status, st);
}

cudaError_t launch_lorc(const LorcParams& p, cudaStream_t s) {
    const int rank_blocks = (MILO_MAX_RANK + 15) / 16;
    const int nproj = p.proj_b >= 0 ? 2 : 1;
    const int blocks = p.n_exp * nproj * rank_blocks;
    if (blocks <= 0) return cudaSuccess;
    lorc_kernel<<<blocks, 128, 0, s>>>(p, rank_blocks);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// combine: y[t] = sum_j w[t,j] * y_slot[inv[t*k+j]] + sum_s y_shared[s, t]
// (or, per slot, y[f] = y_slot[inv[f]]), split-K partials summed in order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float4 row_sum(const float* part, int splits, size_t split_stride,
                                          size_t off) {
    float4 a = *reinterpret_cast<const float4*>(part + off);
    for (int s = 1; s < splits; ++s) {
        const float4 b = *reinterpret_cast<const float4*>(part + s * split_stride + off);
        a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    return a;
}

__global__ void __launch_bounds__(256) combine_kernel(const CombineParams p) {
    const int H4 = p.H / 4;
    const int rows_out = p.per_slot ? p.T * p.k : p.T;
    const long long total = static_cast<long long>(rows_out) * H4;
    const size_t sstride = static_cast<size_t>(p.R) * p.H;
    int32_t st = 0;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int o = static_cast<int>(i / H4);
        const int n = static_cast<int>(i % H4) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p.per_slot) {
            const int r = p.inv_perm[o];
            if (r >= 0) acc = row_sum(p.y_part, p.splits, sstride, static_cast<size_t>(r) * p.H + n);
        } else {
            for (int j = 0; j < p.k; ++j) {
                const int f = o * p.k + j;
                const int r = p.inv_perm[f];
                if (r < 0 || r >= p.R_routed) continue;
                const float wj = p.w[f];
                const float4 v = row_sum(p.y_part, p.splits, sstride, static_cast<size_t>(r) * p.H + n);
                acc.x = fmaf(wj, v.x, acc.x);
                acc.y = fmaf(wj, v.y, acc.y);
                acc.z = fmaf(wj, v.z, acc.z);
                acc.w = fmaf(wj, v.w, acc.w);
            }
            for (int s = 0; s < p.S; ++s) {
                const float4 v = row_sum(p.y_part, p.splits, sstride,
                                         static_cast<size_t>(p.R_routed + s * p.T + o) * p.H + n);
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
        }
        const size_t off = static_cast<size_t>(o) * p.H + n;
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
    flag(p.dev_status, st);
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t s) {
    const long long rows_out = p.per_slot ? static_cast<long long>(p.T) * p.k : p.T;
    const long long total = rows_out * (p.H / 4);
    if (total <= 0) return cudaSuccess;
    long long blocks = (total + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    combine_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace milo
