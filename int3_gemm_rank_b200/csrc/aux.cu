// aux.cu -- the kernels around the grouped int3 GEMM:
//   prep_kernel    activations -> fp16 MMA fragments (the row's power-of-2
//                  scale and those of the int3 field extraction folded in)
//                  and per-group sums; the
//                  first one of a call also does the row bookkeeping (expert
//                  groups, row -> token) from the router's offsets and perm
//   lorc_*_kernel  compensator down-projection t = x V^T per expert
//   combine_kernel weighted un-permute back to token order, split-K reduction
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators": the compensator is a rank-r product U V added to the
// quantised weight ("MiLo Algorithm"), so x (W_q + U V)^T splits into the int3
// GEMM and (x V^T) U^T; the MoE layer combines the routed experts' outputs.
#include <cuda_runtime.h>

#include <climits>

#include "milo_combine.cuh"
#include "milo_device.cuh"
#include "milo_host.h"
#include "milo_kernels.h"

static_assert(milo::kBlockSB == milo::kBlobBlockBytes && milo::kQTileSBWords * 4 == milo::kBlobWordBytes &&
                  milo::kGroupBytes == milo::kBlobGroupBytes,
              "blob block layout");

namespace milo {

// ---------------------------------------------------------------------------
// prep: fragment-ordered activations and group sums, one block per row
// ---------------------------------------------------------------------------
// Activations of register (word t, field f) times 2^(6 - e): exact, the
// scaled row's values being below 2 (see act_scale).
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

// Expert groups (first row, count), clamped into a non-decreasing sequence
// within [0, T*k]; shared experts follow the routed rows.  Block (0, 0) only.
__device__ void build_groups(const PrepParams& p, int32_t& st) {
    // ok_off[e] = max(ok_off[e-1], min(offsets[e], F)), ok_off[0] = 0: a
    // running maximum, so warp 0 scans it 32 experts at a time after all
    // threads have loaded the offsets.
    __shared__ int ok_off[MILO_MAX_EXPERTS + 1];
    const int F = p.T * p.k;
    const int lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) ok_off[e] = p.offsets[e];
    __syncthreads();
    if (threadIdx.x < 32) {
        int run = 0;
        for (int base = 0; base <= p.E; base += 32) {
            const int e = base + lane;
            const int o = e <= p.E ? ok_off[e] : 0;
            int incl = e == 0 ? 0 : (e <= p.E ? min(o, F) : INT_MIN);
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
                if (lane >= d) incl = max(incl, y);
            }
            incl = max(incl, run);
            const int up = __shfl_up_sync(0xFFFFFFFFu, incl, 1);   // every lane takes part
            const int prev = lane == 0 ? run : up;
            if (e <= p.E) {
                if ((e == 0 && o != 0) || o > F || (e > 0 && o < prev)) st |= MILO_DEV_BAD_EXPERT_ID;
            }
            __syncwarp();
            if (e <= p.E) ok_off[e] = incl;
            run = __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        p.grp[2 * e] = ok_off[e];
        p.grp[2 * e + 1] = ok_off[e + 1] - ok_off[e];
    }
    for (int s = threadIdx.x; s < p.S; s += blockDim.x) {
        p.grp[2 * (p.E + s)] = p.R_routed + s * p.T;
        p.grp[2 * (p.E + s) + 1] = p.T;
    }
    if (p.inv) {
        for (int f = threadIdx.x; f < F; f += blockDim.x) p.inv[f] = -1;
        __syncthreads();
        const int used = ok_off[p.E];
        for (int r = threadIdx.x; r < used; r += blockDim.x) {
            const int f = p.perm ? p.perm[r] : r;
            if (f >= 0 && f < F) p.inv[f] = r;
        }
    }
}

// Source row (token) of row `row`, or -1.
__device__ __forceinline__ int row_source(const PrepParams& p, int row, int32_t& st) {
    if (row >= p.R_routed) return (row - p.R_routed) % p.T;
    const int F = p.T * p.k;
    int used = p.offsets[p.E];
    used = used < 0 ? 0 : (used > F ? F : used);
    if (row >= used) return -1;
    const int f = p.perm ? p.perm[row] : row;
    if (f < 0 || f >= F) {
        st |= MILO_DEV_BAD_EXPERT_ID;
        return -1;
    }
    return f / p.k;
}

// Largest magnitude of row `src` (K elements, fp16 or bf16), over the whole
// block; 0 for a zero row.  NaN counts as larger than everything (the caller's
// scale then falls back to 1 and the conversion flags it).
__device__ __forceinline__ uint32_t row_max_bits(const PrepParams& p, int src) {
    __shared__ uint32_t wmax[4];
    uint32_t mx = 0u;
    if (src >= 0) {
        const uint4* rowv = reinterpret_cast<const uint4*>(p.src + static_cast<size_t>(src) * p.K);
        for (int i = threadIdx.x; i < p.K / 8; i += blockDim.x) {
            const uint4 u = rowv[i];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                mx = max(mx, __float_as_uint(fabsf(act_f32(static_cast<uint16_t>(w[q] & 0xFFFFu), p.src_bf16))));
                mx = max(mx, __float_as_uint(fabsf(act_f32(static_cast<uint16_t>(w[q] >> 16), p.src_bf16))));
            }
        }
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
    __syncthreads();
    return max(max(wmax[0], wmax[1]), max(wmax[2], wmax[3]));
}

__global__ void __launch_bounds__(128) prep_kernel(const PrepParams p) {
    grid_dep_launch();
    grid_dep_wait();
    const int row = blockIdx.x;
    const int SB = p.K / 128;
    int32_t st = 0;
    if (p.zero) {
        const int nb = gridDim.x * gridDim.y, b = blockIdx.x * gridDim.y + blockIdx.y;
        for (int i = b * blockDim.x + threadIdx.x; i < p.nzero; i += nb * blockDim.x) p.zero[i] = 0;
    }
    int src;
    if (p.rows) {
        if (blockIdx.x == 0 && blockIdx.y == 0) build_groups(p, st);
        src = row_source(p, row, st);
        if (blockIdx.y == 0 && threadIdx.x == 0) p.row_src[row] = src;
    } else {
        src = p.row_src ? p.row_src[row] : row;
    }
    // the source has T rows (tokens) when rows come from the router, else R
    if (src >= 0 && !in_range(p.dev_status, src < (p.rows || p.row_src ? p.T : p.R))) src = -1;
    // the row's scale 2^a: every block of the row reads the whole row (the
    // blocks of one row are few, and only while rows are few)
    const float scale = row_scale_for(row_max_bits(p, src));
    if (blockIdx.y == 0 && threadIdx.x == 0) p.rscale[row] = scale;
    for (int base = blockIdx.y * blockDim.x; base < SB * 4; base += gridDim.y * blockDim.x) {
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
                    x[16 * half + 2 * i] = to_half_scaled(static_cast<uint16_t>(w[i] & 0xFFFFu), p.src_bf16, scale, st);
                    x[16 * half + 2 * i + 1] = to_half_scaled(static_cast<uint16_t>(w[i] >> 16), p.src_bf16, scale, st);
                }
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) s0 += __half2float(x[m]);
#pragma unroll
            for (int m = 16; m < 32; ++m) s1 += __half2float(x[m]);
            if (p.plain) {
                // the row's scaled values, plain: 16 at 128 sb + 16c, 16 at + 64
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = static_cast<uint32_t>(__half_as_ushort(x[2 * i])) |
                           (static_cast<uint32_t>(__half_as_ushort(x[2 * i + 1])) << 16);
                uint4* o = reinterpret_cast<uint4*>(p.plain + static_cast<size_t>(row) * p.K + 128 * sb + 16 * c);
                o[0] = make_uint4(w[0], w[1], w[2], w[3]);
                o[1] = make_uint4(w[4], w[5], w[6], w[7]);
                uint4* o2 = reinterpret_cast<uint4*>(p.plain + static_cast<size_t>(row) * p.K + 128 * sb + 64 + 16 * c);
                o2[0] = make_uint4(w[8], w[9], w[10], w[11]);
                o2[1] = make_uint4(w[12], w[13], w[14], w[15]);
            }
        } else {
#pragma unroll
            for (int m = 0; m < 32; ++m) x[m] = __ushort_as_half(0);
            if (active && p.plain) {
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                uint4* o = reinterpret_cast<uint4*>(p.plain + static_cast<size_t>(row) * p.K + 128 * sb + 16 * c);
                uint4* o2 = reinterpret_cast<uint4*>(p.plain + static_cast<size_t>(row) * p.K + 128 * sb + 64 + 16 * c);
                o[0] = o[1] = o2[0] = o2[1] = z;
            }
        }
        // group sums over the four units of the super-block (lanes 4j..4j+3)
        s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
        s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 2);
        s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
        s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 2);
        if (!active) continue;
        if (p.layout == 1) {
            // tcgen05 GEMM: [R][K] with the K slots of each super-block in the
            // order of the A columns (unit c's first-group registers at columns
            // 8c..8c+7, its second-group ones at 32+8c..), group sums [R][4*chunks]
            uint4* o1 = reinterpret_cast<uint4*>(p.frag + static_cast<size_t>(row) * p.K + 128 * sb + 16 * c);
            uint4* o2 = reinterpret_cast<uint4*>(p.frag + static_cast<size_t>(row) * p.K + 128 * sb + 64 + 16 * c);
            const uint2 f0 = frag_step<0>(x), f1 = frag_step<1>(x), f2 = frag_step<2>(x), f3 = frag_step<3>(x);
            const uint2 f4 = frag_step<4>(x), f5 = frag_step<5>(x), f6 = frag_step<6>(x), f7 = frag_step<7>(x);
            o1[0] = make_uint4(f0.x, f0.y, f1.x, f1.y);
            o1[1] = make_uint4(f2.x, f2.y, f3.x, f3.y);
            o2[0] = make_uint4(f4.x, f4.y, f5.x, f5.y);
            o2[1] = make_uint4(f6.x, f6.y, f7.x, f7.y);
            if (c == 0) {
                // the two group sums (|sum| <= 128) split exactly enough into
                // fp16 hi + lo (2^-22 relative), slots (hi, lo, hi, lo) per group; a
                // pair of super-blocks shares 16 slots, the odd tail's second half is 0
                uint32_t v[4];
                const float gs[2] = {s0, s1};
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    const __half hi = __float2half_rn(gs[g]);
                    const __half lo = __float2half_rn(gs[g] - __half2float(hi));
                    v[2 * g] = v[2 * g + 1] =
                        static_cast<uint32_t>(__half_as_ushort(hi)) | (static_cast<uint32_t>(__half_as_ushort(lo)) << 16);
                }
                uint4* zp = reinterpret_cast<uint4*>(p.gsum + (static_cast<size_t>(row) * ((SB + 1) / 2) + (sb >> 1)) * 16);
                zp[sb & 1] = make_uint4(v[0], v[1], v[2], v[3]);
                if (sb == SB - 1 && !(sb & 1)) zp[1] = make_uint4(0u, 0u, 0u, 0u);
            }
            continue;
        }
        // chunk-major layout: the 16-row tile of one K chunk is one contiguous
        // block; the chunk's four group sums sit in the row's padding
        const size_t crow = static_cast<size_t>(sb >> 1) * p.R + row;
        if (c == 0) {
            float* gs = reinterpret_cast<float*>(p.frag + crow * kFragRowHalves + kGsumHalf);
            gs[2 * (sb & 1)] = s0;
            gs[2 * (sb & 1) + 1] = s1;
            if (!(sb & 1)) gs[kInvSlot] = inv_pow2(scale);   // the GEMM epilogue's 2^-a
        }
        // per super-block: step-major, lane-in-quad c, 4 fp16 each
        uint2* out = reinterpret_cast<uint2*>(p.frag + crow * kFragRowHalves + (sb & 1) * kFragHalvesPerSB) + c;
        out[0 * 4] = frag_step<0>(x);
        out[1 * 4] = frag_step<1>(x);
        out[2 * 4] = frag_step<2>(x);
        out[3 * 4] = frag_step<3>(x);
        out[4 * 4] = frag_step<4>(x);
        out[5 * 4] = frag_step<5>(x);
        out[6 * 4] = frag_step<6>(x);
        out[7 * 4] = frag_step<7>(x);
    }
    flag(p.dev_status, st);
}

cudaError_t launch_prep(const PrepParams& p, cudaStream_t s) {
    if (p.R <= 0) return cudaSuccess;
    // 32 super-blocks per block; several blocks per row fill the GPU at decode
    // sizes, one block per row once rows are many (each block of a row reads
    // the whole row for its scale)
    const int chunks = p.R >= 256 ? 1 : (p.K / 128 * 4 + 127) / 128;
    return launch_pdl(prep_kernel, dim3(p.R, chunks), dim3(128), 0, s, p);
}

// ---------------------------------------------------------------------------
// lorc: t[p, col0 + j] = sum_k x'[p, k] V[j, k] for the rows of each expert,
// x' = fp16(x 2^a) with the row's scale (so t carries the row's 2^a too).
// One block per (expert, projection, 16-rank block, K slice, row-tile group);
// its four warps split the K slice and their 16x16 tiles are added in a fixed
// order into part[slice].  The block that finishes a (expert, projection,
// rank block, row group) last adds the slices in order and rounds to fp16
// (a counter per tile says which block that is).  Both orders are fixed, so
// the result does not depend on scheduling.
// ---------------------------------------------------------------------------
constexpr int kLorcRankBlocks = (MILO_MAX_RANK + 15) / 16;
constexpr int kLorcChunk = 256;             // K staged per step (per block)
constexpr int kLorcPitch = kLorcChunk + 8;  // fp16; rows fall on different banks

__global__ void __launch_bounds__(128) lorc_partial_kernel(const LorcParams p) {
    grid_dep_launch();
    grid_dep_wait();
    __shared__ __align__(16) uint16_t xs[16][kLorcPitch];
    __shared__ __align__(16) uint16_t vs[16][kLorcPitch];
    __shared__ float part[4][16][17];
    __shared__ int src_row[16];
    __shared__ float src_scale[16];
    const int nproj = p.proj_b >= 0 ? 2 : 1;
    int b = blockIdx.x;
    const int split = b % p.splits;
    b /= p.splits;
    const int rblk = b % kLorcRankBlocks;
    b /= kLorcRankBlocks;
    const int which = b % nproj;
    const int e = b / nproj;
    const ProjDev* P = p.table + e * p.stride + (which == 0 ? p.proj_a : p.proj_b);
    const int r = P->rank;
    const int j0 = 16 * rblk;
    // Columns [col0, col0 + span) of t belong to this projection.  Ranks past r
    // are written as zeros so that an MMA over the whole span sees finite values.
    const int span = p.proj_b >= 0 ? p.t_col_b : p.tcols;
    if (j0 >= span) return;
    const int row0 = p.grp[2 * e], m = p.grp[2 * e + 1];
    if (m <= 0 || row0 < 0 || row0 + m > p.R) return;
    const int col0 = which == 0 ? 0 : p.t_col_b;
    // t's columns, and (K split) the slice counter of this tile
    if (!in_range(p.dev_status, col0 + span <= p.tcols &&
                                    (p.splits == 1 || ((e * nproj + which) * kLorcRankBlocks + rblk) * p.row_groups +
                                                              static_cast<int>(blockIdx.y) < kLorcCounters)))
        return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    // K slice of this block: whole super-blocks, the last slice may be shorter
    const int slice_sb = (p.K / 128 + p.splits - 1) / p.splits;
    const int kbeg = min(p.K, split * slice_sb * 128);
    const int kend = min(p.K, kbeg + slice_sb * 128);
    float* out = p.part + static_cast<size_t>(split) * p.R * p.tcols;
    int32_t st = 0;
    if (j0 >= r) {   // ranks of this block are all past r: zeros only, from the first slice
        if (split == 0)
            for (int mt = 16 * blockIdx.y; mt < m; mt += 16 * p.row_groups)
                for (int idx = threadIdx.x; idx < 256; idx += blockDim.x) {
                    const int rr = idx / 16, jj = idx % 16;
                    if (mt + rr < m && j0 + jj < span)
                        p.t[static_cast<size_t>(row0 + mt + rr) * p.tcols + col0 + j0 + jj] = 0;
                }
        return;
    }
    const bool single = p.splits == 1;
    for (int mt = 16 * blockIdx.y; mt < m; mt += 16 * p.row_groups) {
        __syncthreads();
        if (threadIdx.x < 16) {
            const int i = threadIdx.x;
            src_row[i] = mt + i < m ? (p.row_src ? p.row_src[row0 + mt + i] : row0 + mt + i) : -1;
            src_scale[i] = mt + i < m ? p.rscale[row0 + mt + i] : 1.0f;
        }
        float acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
        for (int kc = kbeg; kc < kend; kc += kLorcChunk) {
            // this chunk: 256 or, at the end of a slice, 128 (slices are whole super-blocks)
            const int cs = min(kLorcChunk, kend - kc);
            const int kw = cs / 4;                    // K per warp: 32 or 64
            __syncthreads();
            // stage x rows and V rows [16][cs] with 16-byte loads
            const int per_row = cs / 8;
            for (int i = threadIdx.x; i < 32 * per_row; i += blockDim.x) {
                const int rr = (i / per_row) & 15, ch = i % per_row, isv = i / (16 * per_row);
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (isv) {
                    if (P->lorc3) continue;   // int3 rows: below, one unit per thread
                    if (j0 + rr < r)
                        v = *reinterpret_cast<const uint4*>(P->V + static_cast<size_t>(j0 + rr) * p.K + kc + 8 * ch);
                    *reinterpret_cast<uint4*>(&vs[rr][8 * ch]) = v;
                } else {
                    const int sr = src_row[rr];
                    if (sr >= 0)
                        v = scaled_pairs(*reinterpret_cast<const uint4*>(p.src + static_cast<size_t>(sr) * p.K + kc + 8 * ch),
                                        p.src_bf16, src_scale[rr], st);
                    *reinterpret_cast<uint4*>(&xs[rr][8 * ch]) = v;
                }
            }
            if (P->lorc3) {
                // int3 V: unit c of super-block sb of rank row j0 + rr, dequantised to
                // fp16: its first 16 codes at 16c.., its last 16 at 64 + 16c..
                const uint8_t* vb = reinterpret_cast<const uint8_t*>(P->V);
                for (int i = threadIdx.x; i < 16 * (cs / 32); i += blockDim.x) {
                    const int rr = i / (cs / 32), u = i % (cs / 32), sb = u >> 2, c = u & 3;
                    const int j = j0 + rr, b = (kc >> 7) + sb;
                    uint32_t h0[8], h1[8];
                    if (j < r) {
                        const uint32_t* wp = reinterpret_cast<const uint32_t*>(vb + lorc_words_off(j, b, c));
                        const uint32_t w3[3] = {wp[0], wp[1], wp[2]};
                        const uint32_t sz0 = *reinterpret_cast<const uint32_t*>(vb + lorc_sz_off(j, 2 * b));
                        const uint32_t sz1 = *reinterpret_cast<const uint32_t*>(vb + lorc_sz_off(j, 2 * b + 1));
                        unit_half_dequant(w3, 0, sz_scale(sz0), sz_zero(sz0), h0);
                        unit_half_dequant(w3, 1, sz_scale(sz1), sz_zero(sz1), h1);
                    } else {
#pragma unroll
                        for (int q = 0; q < 8; ++q) h0[q] = h1[q] = 0u;
                    }
                    uint16_t* row = &vs[rr][128 * sb + 16 * c];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        reinterpret_cast<uint4*>(row)[q] = make_uint4(h0[4 * q], h0[4 * q + 1], h0[4 * q + 2], h0[4 * q + 3]);
                        reinterpret_cast<uint4*>(row + 64)[q] =
                            make_uint4(h1[4 * q], h1[4 * q + 1], h1[4 * q + 2], h1[4 * q + 3]);
                    }
                }
            }
            __syncthreads();
            for (int k = warp * kw; k < warp * kw + kw; k += 16) {
                const int kk = k + 2 * c;
                const uint32_t a0 = *reinterpret_cast<const uint32_t*>(&xs[g][kk]);
                const uint32_t a1 = *reinterpret_cast<const uint32_t*>(&xs[g + 8][kk]);
                const uint32_t a2 = *reinterpret_cast<const uint32_t*>(&xs[g][kk + 8]);
                const uint32_t a3 = *reinterpret_cast<const uint32_t*>(&xs[g + 8][kk + 8]);
                const uint32_t b00 = *reinterpret_cast<const uint32_t*>(&vs[g][kk]);
                const uint32_t b01 = *reinterpret_cast<const uint32_t*>(&vs[g][kk + 8]);
                const uint32_t b10 = *reinterpret_cast<const uint32_t*>(&vs[g + 8][kk]);
                const uint32_t b11 = *reinterpret_cast<const uint32_t*>(&vs[g + 8][kk + 8]);
                mma16816(acc[0], a0, a1, a2, a3, b00, b01);
                mma16816(acc[1], a0, a1, a2, a3, b10, b11);
            }
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
            if (mt + rr < m && j0 + jj < span) {
                const size_t o = static_cast<size_t>(row0 + mt + rr) * p.tcols + col0 + j0 + jj;
                if (single) p.t[o] = t_half(j0 + jj < r ? v : 0.0f, st);
                else out[o] = j0 + jj < r ? v : 0.0f;
            }
        }
    }
    flag(p.dev_status, st);
    if (single) return;
    // the last block of this tile to finish adds the slices in order
    __shared__ int last;
    __threadfence();
    __syncthreads();
    int32_t* ctr = p.done + ((e * nproj + which) * kLorcRankBlocks + rblk) * p.row_groups + blockIdx.y;
    if (threadIdx.x == 0) last = atomicAdd(ctr, 1) == p.splits - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    const size_t slice = static_cast<size_t>(p.R) * p.tcols;
    for (int mt = 16 * blockIdx.y; mt < m; mt += 16 * p.row_groups)
        for (int idx = threadIdx.x; idx < 256; idx += blockDim.x) {
            const int rr = idx / 16, jj = idx % 16;
            if (mt + rr < m && j0 + jj < span) {
                const size_t o = static_cast<size_t>(row0 + mt + rr) * p.tcols + col0 + j0 + jj;
                float v = 0.0f;
                for (int sp = 0; sp < p.splits; ++sp) v += __ldcg(p.part + sp * slice + o);
                p.t[o] = t_half(v, st);
            }
        }
    if (threadIdx.x == 0) *ctr = 0;   // ready for the next launch
    flag(p.dev_status, st);
}

// Many rows per expert (no K split): one block per (expert, projection, 64-row
// tile) computes all 64 ranks over the whole K, so a V row is read once per 64
// rows instead of once per 16.  Four warps take 16 rows each; K advances 64 at
// a time through shared memory, the next chunk's loads in flight (registers)
// while the current one is multiplied.  One fixed order: deterministic.
constexpr int kLtRows = 64, kLtK = 64, kLtPitch = kLtK + 8;   // fp16 pitch: rows on different banks

__global__ void __launch_bounds__(128) lorc_tile_kernel(const LorcParams p) {
    grid_dep_launch();
    grid_dep_wait();
    __shared__ __align__(16) uint16_t xs[kLtRows][kLtPitch];
    __shared__ __align__(16) uint16_t vs[MILO_MAX_RANK][kLtPitch];
    __shared__ int src_row[kLtRows];
    __shared__ float src_scale[kLtRows];
    const int nproj = p.proj_b >= 0 ? 2 : 1;
    const int which = blockIdx.x % nproj, e = blockIdx.x / nproj;
    const ProjDev* P = p.table + e * p.stride + (which == 0 ? p.proj_a : p.proj_b);
    const int r = P->rank;
    const int span = p.proj_b >= 0 ? p.t_col_b : p.tcols;
    const int col0 = which == 0 ? 0 : p.t_col_b;
    const int row0 = p.grp[2 * e], m = p.grp[2 * e + 1];
    if (m <= 0 || row0 < 0 || row0 + m > p.R) return;
    if (!in_range(p.dev_status, col0 + span <= p.tcols)) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int nr8 = (r + 7) / 8;                      // n8 rank tiles that hold ranks < r
    int32_t st = 0;
    for (int mt = kLtRows * blockIdx.y; mt < m; mt += kLtRows * gridDim.y) {
        if (r == 0) {
            for (int idx = threadIdx.x; idx < kLtRows * span; idx += blockDim.x) {
                const int rr = idx / span, jj = idx % span;
                if (mt + rr < m) p.t[static_cast<size_t>(row0 + mt + rr) * p.tcols + col0 + jj] = 0;
            }
            continue;
        }
        __syncthreads();
        if (threadIdx.x < kLtRows) {
            const int i = threadIdx.x;
            src_row[i] = mt + i < m ? (p.row_src ? p.row_src[row0 + mt + i] : row0 + mt + i) : -1;
            src_scale[i] = mt + i < m ? p.rscale[row0 + mt + i] : 1.0f;
        }
        __syncthreads();
        // this thread's share of a chunk: x rows (4 x 16 B) and V rows (4 x 16 B)
        uint4 xr[4], vr[4];
        // int3 V: a chunk of 64 positions is one group, 16 codes in each of the
        // super-block's four units; this thread takes rank row tid / 2, units
        // 2 (tid & 1) and 2 (tid & 1) + 1 (positions 32 (tid & 1) .. + 31)
        const uint8_t* vb = reinterpret_cast<const uint8_t*>(P->V);
        const int urow = threadIdx.x >> 1, uu = threadIdx.x & 1;
        uint32_t vw[6] = {0u, 0u, 0u, 0u, 0u, 0u}, vsz = 0u;
        auto fetch = [&](int kc) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = threadIdx.x + 128 * q;       // 0..511: row i / 8, 16-byte piece i % 8
                const int rr = i >> 3, pc = i & 7;
                const int sr = src_row[rr];
                xr[q] = sr >= 0 ? *reinterpret_cast<const uint4*>(p.src + static_cast<size_t>(sr) * p.K + kc + 8 * pc)
                                : make_uint4(0u, 0u, 0u, 0u);
                if (!P->lorc3)
                    vr[q] = rr < r ? *reinterpret_cast<const uint4*>(P->V + static_cast<size_t>(rr) * p.K + kc + 8 * pc)
                                   : make_uint4(0u, 0u, 0u, 0u);
            }
            if (P->lorc3 && urow < r) {
                const uint32_t* wp = reinterpret_cast<const uint32_t*>(vb + lorc_words_off(urow, kc >> 7, 2 * uu));
#pragma unroll
                for (int q = 0; q < 6; ++q) vw[q] = wp[q];
                vsz = *reinterpret_cast<const uint32_t*>(vb + lorc_sz_off(urow, kc >> 6));
            }
        };
        float acc[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;
        fetch(0);
        for (int kc = 0; kc < p.K; kc += kLtK) {
            __syncthreads();     // the previous chunk's multiplies are done
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = threadIdx.x + 128 * q;
                const int rr = i >> 3, pc = i & 7;
                *reinterpret_cast<uint4*>(&xs[rr][8 * pc]) = scaled_pairs(xr[q], p.src_bf16, src_scale[rr], st);
                if (!P->lorc3) *reinterpret_cast<uint4*>(&vs[rr][8 * pc]) = vr[q];
            }
            if (P->lorc3) {
                uint32_t h[2][8];
                if (urow < r) {
                    const int half = (kc >> 6) & 1;
                    const uint32_t wa[3] = {vw[0], vw[1], vw[2]}, wb[3] = {vw[3], vw[4], vw[5]};
                    unit_half_dequant(wa, half, sz_scale(vsz), sz_zero(vsz), h[0]);
                    unit_half_dequant(wb, half, sz_scale(vsz), sz_zero(vsz), h[1]);
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) h[0][q] = h[1][q] = 0u;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(&vs[urow][32 * uu + 8 * q]) =
                        make_uint4(h[q >> 1][4 * (q & 1)], h[q >> 1][4 * (q & 1) + 1], h[q >> 1][4 * (q & 1) + 2],
                                   h[q >> 1][4 * (q & 1) + 3]);
            }
            __syncthreads();
            if (kc + kLtK < p.K) fetch(kc + kLtK);
#pragma unroll
            for (int k16 = 0; k16 < kLtK; k16 += 16) {
                const int kk = k16 + 2 * c;
                const int ra = 16 * warp + g;
                const uint32_t a0 = *reinterpret_cast<const uint32_t*>(&xs[ra][kk]);
                const uint32_t a1 = *reinterpret_cast<const uint32_t*>(&xs[ra + 8][kk]);
                const uint32_t a2 = *reinterpret_cast<const uint32_t*>(&xs[ra][kk + 8]);
                const uint32_t a3 = *reinterpret_cast<const uint32_t*>(&xs[ra + 8][kk + 8]);
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    if (n < nr8) {
                        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&vs[8 * n + g][kk]);
                        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&vs[8 * n + g][kk + 8]);
                        mma16816(acc[n], a0, a1, a2, a3, b0, b1);
                    }
                }
            }
        }
        // acc[n][i]: row 16 * warp + g + 8 * (i >> 1), rank 8n + 2c + (i & 1)
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int rr = 16 * warp + g + 8 * (i >> 1), j = 8 * n + 2 * c + (i & 1);
                if (mt + rr < m && j < span)
                    p.t[static_cast<size_t>(row0 + mt + rr) * p.tcols + col0 + j] = t_half(j < r ? acc[n][i] : 0.0f, st);
            }
    }
    flag(p.dev_status, st);
}

cudaError_t launch_lorc(const LorcParams& p, cudaStream_t s) {
    const int nproj = p.proj_b >= 0 ? 2 : 1;
    if (p.n_exp <= 0 || p.R <= 0) return cudaSuccess;
    if (p.splits == 1 && p.row_groups >= 8) {
        // many rows: 64-row tiles, each block striding over its expert's tiles
        const int tiles = (p.R + kLtRows - 1) / kLtRows;
        return launch_pdl(lorc_tile_kernel, dim3(static_cast<unsigned>(p.n_exp * nproj), std::min(tiles, 64)),
                          dim3(128), 0, s, p);
    }
    const long long blocks = static_cast<long long>(p.n_exp) * nproj * kLorcRankBlocks * p.splits;
    return launch_pdl(lorc_partial_kernel, dim3(static_cast<unsigned>(blocks), p.row_groups), dim3(128), 0, s, p);
}

// ---------------------------------------------------------------------------
// combine: y[t] = sum_j w[t,j] * y_slot[inv[t*k+j]] + sum_s y_shared[s, t]
// (or, per slot, y[f] = y_slot[inv[f]]), split-K partials summed in order.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(64) combine_kernel(const CombineParams p) {
    grid_dep_launch();
    grid_dep_wait();
    const int H4 = p.H / 4;
    const int rows_out = p.per_slot ? p.T * p.k : p.T;
    const long long total = static_cast<long long>(rows_out) * H4;
    int32_t st = 0;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int o = static_cast<int>(i / H4);
        const int n = static_cast<int>(i % H4) * 4;
        store4(p, static_cast<size_t>(o) * p.H + n, combine4(p, o, n), st);
    }
    flag(p.dev_status, st);
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t s) {
    const long long rows_out = p.per_slot ? static_cast<long long>(p.T) * p.k : p.T;
    const long long total = rows_out * (p.H / 4);
    if (total <= 0) return cudaSuccess;
    // small blocks: at decode sizes the outputs are few, and spreading them
    // over more SMs hides the dependent loads (inv_perm, then the partials)
    long long blocks = (total + 63) / 64;
    if (blocks > 8192) blocks = 8192;
    return launch_pdl(combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(64), 0, s, p);
}

}  // namespace milo
