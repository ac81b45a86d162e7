// quant.cu -- the offline MiLo quantiser on the GPU: HQQ quantise-and-pack,
// the rank-r compensator of the residual by randomized subspace iteration,
// and the refinement rounds (sm_100a).
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators", section "MiLo Algorithm: Mixture of Low-Rank Compensators":
// the weights are first quantised with HQQ; the SVD of the residual
// W - W_quant gives the top-r compensator U V; quantisation and compensation
// are then refined in turn.
//
// Design: this runs once per weight, offline, so the kernels favour a fixed
// arithmetic order (deterministic results, codes that are a fixed function of
// the inputs) over speed:
//   - hqq_pack_kernel: one thread per (row, 128-code super-block), like the
//     round-to-nearest packer; the target W - U V, the HQQ iterations and the
//     residual use explicitly rounded fp32 operations (no contraction).
//   - sgemm_kernel: fp32 C = A B with arbitrary strides (64 x 64 tiles, 4 x 4
//     per thread, the reduction never split): the sketch products R omega,
//     R^T Y, Y^T R and the small basis changes.
//   - gram_kernel + gram_sum_kernel: X^T X in fp64, partial sums per row chunk
//     added in a fixed order.
//   - chol_kernel (one block): Cholesky factor of a Gram matrix and the inverse
//     of the factor in fp64: the basis change of Cholesky QR.
//   - jacobi_kernel (one block): cyclic Jacobi eigenpairs of B B^T in fp64,
//     l/2 disjoint rotations per step (round-robin ordering).
//   - apply_kernel + err_sum_kernel: ||R - U V||_F in fp64 and the next
//     round's target W - U V in one coalesced pass, the best-round
//     bookkeeping; copy_best_kernel keeps the best round's blob, U and V.
#include <cuda_runtime.h>

#include "milo_blob.cuh"
#include "milo_device.cuh"
#include "milo_host.h"

namespace milo {

namespace {

__device__ __forceinline__ float f16v(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// ---------------------------------------------------------------------------
// HQQ quantise and pack
// ---------------------------------------------------------------------------

struct HqqArgs {
    const uint16_t* W;      // [N, K] fp16
    const uint16_t* U;      // [N, r] fp16 or null
    const uint16_t* V;      // [r, K] fp16 or null
    const float* T;         // [N, K] fp32 target W - U V formed beforehand, or null
    uint8_t* blob;
    float* resid;           // [N, K] or null
    int32_t* dev_status;
    int N, K, r, iters;
    float beta, kappa;
};

// One group of 64 targets t: HQQ's zero-point fit with p = 1/2 shrinkage,
// keeping the zero point of lowest L1 error; returns the fp16 scale and zero.
__device__ __forceinline__ int32_t hqq_group(const float (&t)[64], int iters, float beta0, float kappa,
                                             __half& sh, __half& zh) {
    int32_t st = 0;
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        if (!isfinite(t[i])) st |= MILO_DEV_NONFINITE;
        mn = t[i] < mn ? t[i] : mn;
        mx = t[i] > mx ? t[i] : mx;
    }
    sh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 7.0f));
    if ((__half_as_ushort(sh) & 0x7FFF) == 0) sh = __ushort_as_half(0x3C00);   // s := 1
    const float s = __half2float(sh);
    float z = __fdiv_rn(-mn, s);
    const float inv = __fdiv_rn(1.0f, s);   // HQQ quantises with the inverse scale
    float beta = beta0, best_err = INFINITY, best_z = z;
    for (int it = 0; it < iters; ++it) {
        float err = 0.0f, acc = 0.0f;
        const float beta2 = __fmul_rn(beta, beta);
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            float r = rintf(__fadd_rn(__fmul_rn(t[i], inv), z));
            if (!(r >= 0.0f)) r = 0.0f;
            if (r > 7.0f) r = 7.0f;
            const float e = __fsub_rn(t[i], __fmul_rn(__fsub_rn(r, z), s));
            const float a = fabsf(e);
            err = __fadd_rn(err, a);
            float w_e = 0.0f;
            // a^3 beta^2 < 1/2 means 1 / (sqrt(a) beta) > 1.41 a, so the shrinkage
            // is zero whatever the rounding; only larger errors need the formula
            const float a3b2 = __fmul_rn(__fmul_rn(__fmul_rn(a, a), a), beta2);
            if (a > 0.0f && !(a3b2 < 0.5f)) {
                const float m = __fsub_rn(a, __fdiv_rn(1.0f, __fmul_rn(__fsqrt_rn(a), beta)));
                if (m > 0.0f) w_e = e < 0.0f ? -m : m;
            }
            acc = __fadd_rn(acc, __fsub_rn(r, __fmul_rn(__fsub_rn(t[i], w_e), inv)));
        }
        if (err < best_err) {
            best_err = err;
            best_z = z;
        }
        z = __fmul_rn(acc, 0.015625f);
        beta = __fmul_rn(beta, kappa);
    }
    zh = __float2half_rn(best_z);
    if (!isfinite(s) || !isfinite(__half2float(zh))) st |= MILO_DEV_FP16_RANGE;
    return st;
}

__global__ void __launch_bounds__(128, 4) hqq_pack_kernel(const HqqArgs a) {
    const int SB = a.K / 128;
    const int Npad = (a.N + 63) / 64 * 64;
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid >= static_cast<long long>(Npad) * SB) return;
    const int n = static_cast<int>(gid / SB);
    const int b = static_cast<int>(gid % SB);
    if (n >= a.N) {
        blob_zero_row(a.blob, n, b, SB);
        return;
    }
    int32_t st = 0;
    uint32_t words[12];
#pragma unroll
    for (int i = 0; i < 12; ++i) words[i] = 0u;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const size_t k0 = static_cast<size_t>(n) * a.K + 128 * b + 64 * g;
        float t[64];
        if (a.T) {
            const float4* tp = reinterpret_cast<const float4*>(a.T + k0);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float4 v = tp[i];
                t[4 * i] = v.x; t[4 * i + 1] = v.y; t[4 * i + 2] = v.z; t[4 * i + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) t[i] = f16v(a.W[k0 + i]);
        }
        // t = W - U V, one rank term at a time (when not formed beforehand)
#pragma unroll 1
        for (int p = 0; p < (a.T ? 0 : a.r); ++p) {
            const float u = f16v(a.U[static_cast<size_t>(n) * a.r + p]);
            const uint16_t* vr = a.V + static_cast<size_t>(p) * a.K + 128 * b + 64 * g;
#pragma unroll
            for (int i = 0; i < 64; ++i) t[i] = __fsub_rn(t[i], __fmul_rn(u, f16v(vr[i])));
        }
        __half sh, zh;
        st |= hqq_group(t, a.iters, a.beta, a.kappa, sh, zh);
        blob_store_sz(a.blob, n, 2 * b + g, SB, __half_as_ushort(sh), __half_as_ushort(zh));
        const float s = __half2float(sh), z = __half2float(zh);
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            float r = rintf(__fadd_rn(__fdiv_rn(t[i], s), z));
            if (!(r >= 0.0f)) r = 0.0f;
            if (r > 7.0f) r = 7.0f;
            place_code(words, 64 * g + i, static_cast<uint32_t>(r));
            if (a.resid) a.resid[k0 + i] = __fsub_rn(f16v(a.W[k0 + i]), __fmul_rn(__fsub_rn(r, z), s));
        }
    }
    blob_store_words(a.blob, n, b, SB, words);
    flag(a.dev_status, st);
}

// ---------------------------------------------------------------------------
// fp32 GEMM with arbitrary strides
// ---------------------------------------------------------------------------

struct GemmArgs {
    int M, Nn, Kd;
    const float* A;          // A(m, k) = A[m * sam + k * sak]
    long long sam, sak;
    const float* B;          // B(k, n) = B[k * sbk + n * sbn]
    long long sbk, sbn;
    float* C;                // C(m, n) = C[m * ldc + n] (fp32), or
    uint16_t* C16;           // the same in fp16 (round to nearest)
    long long ldc;
    int32_t* dev_status;
    float* Cpart;            // split reduction: slice z writes Cpart[z][m][n], else null
    int kslice;              // reduction length per slice (multiple of kGK)
};

constexpr int kGT = 64;      // output tile width (and the height of the small tile)
constexpr int kGK = 16;      // reduction slice per shared-memory stage

// C = A B over the reduction in index order per 16-wide slice, TM x 64 output
// tiles (TM = 128: 8 x 4 outputs per thread; 64: 4 x 4).  Tile loads walk the
// operand's contiguous dimension across threads.
template <int TM>
__global__ void __launch_bounds__(256) sgemm_kernel(const GemmArgs a) {
    constexpr int RM = TM / 16;          // output rows per thread
    __shared__ __align__(16) float As[kGK][TM + 4];
    __shared__ __align__(16) float Bs[kGK][kGT + 4];
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * kGT;
    const int tm = (tid / 16) * RM, tn = (tid % 16) * 4;
    float acc[RM][4];
#pragma unroll
    for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
    const int kbeg = blockIdx.z * a.kslice;
    const int kend = min(a.Kd, kbeg + a.kslice);
    for (int k0 = kbeg; k0 < kend; k0 += kGK) {
#pragma unroll
        for (int i = 0; i < RM; ++i) {               // A: TM x 16 values, RM per thread
            const int idx = tid + 256 * i;
            int mm, kk;
            if (a.sak == 1) { kk = idx % kGK; mm = idx / kGK; }
            else { mm = idx % TM; kk = idx / TM; }
            const int m = m0 + mm, k = k0 + kk;
            As[kk][mm] = (m < a.M && k < kend) ? a.A[m * a.sam + k * a.sak] : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {                // B: 16 x 64 values, 4 per thread
            const int idx = tid + 256 * i;
            int kk, nn;
            if (a.sbn == 1) { nn = idx % kGT; kk = idx / kGT; }
            else { kk = idx % kGK; nn = idx / kGK; }
            const int n = n0 + nn, kb = k0 + kk;
            Bs[kk][nn] = (n < a.Nn && kb < kend) ? a.B[kb * a.sbk + n * a.sbn] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kGK; ++kk) {
            float ar[RM];
#pragma unroll
            for (int h = 0; h < RM / 4; ++h) {
                const float4 av = *reinterpret_cast<const float4*>(&As[kk][tm + 4 * h]);
                ar[4 * h] = av.x; ar[4 * h + 1] = av.y; ar[4 * h + 2] = av.z; ar[4 * h + 3] = av.w;
            }
            const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][tn]);
            const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < RM; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
        }
        __syncthreads();
    }
    int32_t st = 0;
#pragma unroll
    for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = m0 + tm + i, n = n0 + tn + j;
            if (m >= a.M || n >= a.Nn) continue;
            if (a.Cpart) {
                a.Cpart[(static_cast<size_t>(blockIdx.z) * a.M + m) * a.Nn + n] = acc[i][j];
            } else if (a.C16) {
                const __half h = __float2half_rn(acc[i][j]);
                if (!isfinite(__half2float(h))) st |= MILO_DEV_FP16_RANGE;
                a.C16[m * a.ldc + n] = __half_as_ushort(h);
            } else {
                a.C[m * a.ldc + n] = acc[i][j];
            }
        }
    flag(a.dev_status, st);
}

// C(m, n) = sum over slices z, in order, of Cpart[z][m][n] (fp32 or fp16 out).
__global__ void split_sum_kernel(const float* Cpart, int S, int M, int Nn, float* C, uint16_t* C16, long long ldc,
                                 int32_t* dev_status) {
    const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= static_cast<long long>(M) * Nn) return;
    float v = 0.0f;
    for (int z = 0; z < S; ++z) v += Cpart[static_cast<size_t>(z) * M * Nn + e];
    const int m = static_cast<int>(e / Nn), n = static_cast<int>(e % Nn);
    if (C16) {
        const __half h = __float2half_rn(v);
        if (!isfinite(__half2float(h))) flag(dev_status, MILO_DEV_FP16_RANGE);
        C16[m * ldc + n] = __half_as_ushort(h);
    } else {
        C[m * ldc + n] = v;
    }
}

// ---------------------------------------------------------------------------
// Gram matrices in fp64
// ---------------------------------------------------------------------------

struct GramArgs {
    const float* X;          // X(i, c) = X[i * sxi + c * sxc], i < M, c < l
    long long sxi, sxc;
    double* part;            // [chunks][l][l]
    int M, l, rows_per_chunk;
};

constexpr int kGramRows = 32;   // rows staged in shared memory at a time
constexpr int kMaxSketch = 128;

// Block c adds X(i, a) X(i, b) over its rows in index order; thread
// (tid / 16, tid % 16) owns an (l/16 x l/16) tile of (a, b).
__global__ void __launch_bounds__(256) gram_kernel(const GramArgs g) {
    __shared__ float xs[kGramRows][kMaxSketch + 1];
    const int tid = threadIdx.x;
    const int ts = g.l / 16;
    const int ta = (tid / 16) * ts, tb = (tid % 16) * ts;
    double acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
    const int r0 = blockIdx.x * g.rows_per_chunk;
    const int r1 = min(g.M, r0 + g.rows_per_chunk);
    for (int base = r0; base < r1; base += kGramRows) {
        const int nr = min(kGramRows, r1 - base);
        for (int idx = tid; idx < kGramRows * g.l; idx += 256) {
            int i, c;
            if (g.sxc == 1) { c = idx % g.l; i = idx / g.l; }
            else { i = idx % kGramRows; c = idx / kGramRows; }
            xs[i][c] = i < nr ? g.X[(base + i) * g.sxi + c * g.sxc] : 0.0f;
        }
        __syncthreads();
        for (int i = 0; i < nr; ++i) {
#pragma unroll
            for (int aa = 0; aa < 8; ++aa) {
                if (aa >= ts) break;
                const double xa = xs[i][ta + aa];
#pragma unroll
                for (int bb = 0; bb < 8; ++bb) {
                    if (bb >= ts) break;
                    acc[aa][bb] = fma(xa, static_cast<double>(xs[i][tb + bb]), acc[aa][bb]);
                }
            }
        }
        __syncthreads();
    }
    double* out = g.part + static_cast<size_t>(blockIdx.x) * g.l * g.l;
#pragma unroll
    for (int aa = 0; aa < 8; ++aa)
#pragma unroll
        for (int bb = 0; bb < 8; ++bb)
            if (aa < ts && bb < ts) out[(ta + aa) * g.l + tb + bb] = acc[aa][bb];
}

// G[e] = sum over chunks of part[chunk][e], in chunk order.
__global__ void gram_sum_kernel(const double* part, int chunks, int ll, double* G) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= ll) return;
    double s = 0.0;
    for (int c = 0; c < chunks; ++c) s += part[static_cast<size_t>(c) * ll + e];
    G[e] = s;
}

// ---------------------------------------------------------------------------
// Cholesky QR basis change (one block)
// ---------------------------------------------------------------------------

// G [l, l] fp64 (symmetric positive semi-definite) -> M fp32 [l, l] with
// Y M = Y L^-T, L the Cholesky factor of G.  A pivot below 1e-10 of its
// diagonal entry marks a column that lies in the span of the earlier ones:
// its column of M is zero (the basis drops that direction).  L and X = L^-1
// are lower triangles packed in shared memory (entry (i, j), j <= i, at
// i (i + 1) / 2 + j), fp64.
__device__ __forceinline__ int tri(int i, int j) { return i * (i + 1) / 2 + j; }

__global__ void __launch_bounds__(256) chol_kernel(const double* G, int l, float* M) {
    extern __shared__ double sh[];
    double* L = sh;                               // [l (l + 1) / 2]
    double* X = sh + l * (l + 1) / 2;             // [l (l + 1) / 2]
    __shared__ int dead[kMaxSketch];
    const int tid = threadIdx.x;
    for (int i = 0; i < l; ++i)
        for (int j = tid; j <= i; j += blockDim.x) L[tri(i, j)] = G[i * l + j];
    __syncthreads();
    for (int j = 0; j < l; ++j) {
        if (tid == 0) {
            double d = L[tri(j, j)];
            for (int k = 0; k < j; ++k) d -= L[tri(j, k)] * L[tri(j, k)];
            const bool gone = !(d > 1e-10 * G[j * l + j]);
            dead[j] = gone;
            L[tri(j, j)] = gone ? 1.0 : sqrt(d);
        }
        __syncthreads();
        const double piv = L[tri(j, j)];
        for (int i = j + 1 + tid; i < l; i += blockDim.x) {
            double v = 0.0;
            if (!dead[j]) {
                v = L[tri(i, j)];
                for (int k = 0; k < j; ++k) v -= L[tri(i, k)] * L[tri(j, k)];
                v /= piv;
            }
            L[tri(i, j)] = v;
        }
        __syncthreads();
    }
    // X = L^-1 by forward substitution, one column per thread
    for (int c = tid; c < l; c += blockDim.x) {
        for (int i = c; i < l; ++i) {
            double v = i == c ? 1.0 : 0.0;
            for (int k = c; k < i; ++k) v -= L[tri(i, k)] * X[tri(k, c)];
            X[tri(i, c)] = v / L[tri(i, i)];
        }
    }
    __syncthreads();
    // M[k][i] = X[i][k] (zero above the diagonal of X); the row of X of a
    // dropped column is zero
    for (int idx = tid; idx < l * l; idx += blockDim.x) {
        const int k = idx / l, i = idx % l;
        M[idx] = (dead[i] || k > i) ? 0.0f : static_cast<float>(X[tri(i, k)]);
    }
}

// ---------------------------------------------------------------------------
// Symmetric eigenpairs by cyclic Jacobi (one block)
// ---------------------------------------------------------------------------

// C [l, l] fp64 symmetric (l even) -> the top r eigenpairs in descending
// order of eigenvalue, emitted as MU fp32 [l, r] = P_r sigma^(1/2) and MV fp32
// [r, l] = sigma^(-1/2) P_r^T with sigma = sqrt(max(lambda, 0)); directions
// with sigma <= 1e-12 sigma_0 get zeros.  The eigenvectors P accumulate in
// fp32 in shared memory next to the fp64 matrix.  Each sweep pairs every index with every other once
// (round-robin: index l-1 fixed, the rest rotating), l/2 disjoint rotations
// per step; at most kJacobiSweeps sweeps, fewer once the off-diagonal mass
// falls below 1e-24 of the total (off-diagonal entries near 1e-12 of the
// matrix: far below the fp32 and fp16 outputs).
constexpr int kJacobiSweeps = 40;

__global__ void __launch_bounds__(256) jacobi_kernel(const double* C, int l, int r, float* MU, float* MV) {
    extern __shared__ double As[];               // [l][l + 1], then P fp32 [l][l + 1]
    float* P = reinterpret_cast<float*>(As + l * (l + 1));
    __shared__ double cs[kMaxSketch / 2], sn[kMaxSketch / 2];
    __shared__ int pp[kMaxSketch / 2], qq[kMaxSketch / 2], order[kMaxSketch];
    __shared__ double red[256];
    __shared__ int stop;
    const int ld = l + 1, tid = threadIdx.x, half = l / 2, m = l - 1;
    for (int idx = tid; idx < l * l; idx += blockDim.x) {
        As[(idx / l) * ld + idx % l] = C[idx];
        P[(idx / l) * ld + idx % l] = (idx / l == idx % l) ? 1.0f : 0.0f;
    }
    __syncthreads();
    for (int sweep = 0; sweep < kJacobiSweeps; ++sweep) {
        double off = 0.0, tot = 0.0;
        for (int idx = tid; idx < l * l; idx += blockDim.x) {
            const double v = As[(idx / l) * ld + idx % l];
            tot += v * v;
            if (idx / l != idx % l) off += v * v;
        }
        red[tid] = off;
        __syncthreads();
        for (int s = 128; s > 0; s >>= 1) {
            if (tid < s) red[tid] += red[tid + s];
            __syncthreads();
        }
        const double off_all = red[0];
        __syncthreads();
        red[tid] = tot;
        __syncthreads();
        for (int s = 128; s > 0; s >>= 1) {
            if (tid < s) red[tid] += red[tid + s];
            __syncthreads();
        }
        if (tid == 0) stop = !(off_all > 1e-24 * red[0]);
        __syncthreads();
        if (stop) break;
        for (int step = 0; step < m; ++step) {
            if (tid < half) {
                int p, q;
                if (tid == 0) { p = step % m; q = m; }
                else { p = (step + tid) % m; q = (step - tid + m) % m; }
                const double app = As[p * ld + p], aqq = As[q * ld + q], apq = As[p * ld + q];
                double c = 1.0, s = 0.0;
                if (apq != 0.0) {
                    const double tau = (aqq - app) / (2.0 * apq);
                    const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
                    c = 1.0 / sqrt(1.0 + t * t);
                    s = t * c;
                }
                cs[tid] = c; sn[tid] = s; pp[tid] = p; qq[tid] = q;
            }
            __syncthreads();
            // rows: A <- J^T A
            for (int idx = tid; idx < half * l; idx += blockDim.x) {
                const int k = idx / l, j = idx % l, p = pp[k], q = qq[k];
                const double ap = As[p * ld + j], aq = As[q * ld + j];
                As[p * ld + j] = cs[k] * ap - sn[k] * aq;
                As[q * ld + j] = sn[k] * ap + cs[k] * aq;
            }
            __syncthreads();
            // columns: A <- A J, P <- P J
            for (int idx = tid; idx < half * l; idx += blockDim.x) {
                const int k = idx / l, i = idx % l, p = pp[k], q = qq[k];
                const double ap = As[i * ld + p], aq = As[i * ld + q];
                As[i * ld + p] = cs[k] * ap - sn[k] * aq;
                As[i * ld + q] = sn[k] * ap + cs[k] * aq;
                const double vp = P[i * ld + p], vq = P[i * ld + q];
                P[i * ld + p] = static_cast<float>(cs[k] * vp - sn[k] * vq);
                P[i * ld + q] = static_cast<float>(sn[k] * vp + cs[k] * vq);
            }
            __syncthreads();
        }
    }
    // descending eigenvalue order, the lower index first on ties (NaN last):
    // every index gets a distinct rank, so order[] is a permutation
    for (int i = tid; i < l; i += blockDim.x) {
        const double li = As[i * ld + i] == As[i * ld + i] ? As[i * ld + i] : -INFINITY;
        int rank = 0;
        for (int j = 0; j < l; ++j) {
            const double lj = As[j * ld + j] == As[j * ld + j] ? As[j * ld + j] : -INFINITY;
            rank += (lj > li || (lj == li && j < i)) ? 1 : 0;
        }
        order[rank] = i;
    }
    __syncthreads();
    const double sig0 = sqrt(fmax(As[order[0] * ld + order[0]], 0.0));
    for (int idx = tid; idx < l * r; idx += blockDim.x) {
        const int a = idx / r, i = idx % r;
        const double sig = sqrt(fmax(As[order[i] * ld + order[i]], 0.0));
        const bool live = sig0 > 0.0 && sig > 1e-12 * sig0;
        const double root = live ? sqrt(sig) : 0.0;
        const double v = P[a * ld + order[i]];
        MU[a * r + i] = static_cast<float>(v * root);
        MV[i * l + a] = live ? static_cast<float>(v / root) : 0.0f;
    }
}

// ---------------------------------------------------------------------------
// Error norm, best round, copies
// ---------------------------------------------------------------------------

// One thread per (row n, 4 consecutive columns), so a warp reads 128
// consecutive entries of each V row.  Per entry it forms the products
// U[n, p] V[p, k] (exact in fp32: fp16 times fp16) once and uses them twice:
//   - the error term (R - sum_p U V)^2, summed over p in fp64;
//   - when T is not null, the next round's target t = W, then t = t - U V for
//     p = 0..r-1 rounded to fp32 at every step (the order milo_hqq_pack uses).
// Block partials of the squared error go to part[] (fixed reduction tree).
constexpr int kApplyThreads = 256;

__global__ void __launch_bounds__(kApplyThreads) apply_kernel(const float* R, const uint16_t* W, const uint16_t* U,
                                                              const uint16_t* V, int N, int K, int r, float* T,
                                                              double* part) {
    __shared__ double ws[kApplyThreads / 32];
    const int K4 = K / 4;
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    double acc = 0.0;
    if (gid < static_cast<long long>(N) * K4) {
        const int n = static_cast<int>(gid / K4), k0 = static_cast<int>(gid % K4) * 4;
        const size_t o = static_cast<size_t>(n) * K + k0;
        const float4 rv = *reinterpret_cast<const float4*>(R + o);
        const uint2 wv = *reinterpret_cast<const uint2*>(W + o);
        float t[4] = {f16v(wv.x & 0xFFFFu), f16v(wv.x >> 16), f16v(wv.y & 0xFFFFu), f16v(wv.y >> 16)};
        double uv[4] = {0.0, 0.0, 0.0, 0.0};
        for (int p = 0; p < r; ++p) {
            const float u = f16v(U[static_cast<size_t>(n) * r + p]);
            const uint2 vv = *reinterpret_cast<const uint2*>(V + static_cast<size_t>(p) * K + k0);
            const float v[4] = {f16v(vv.x & 0xFFFFu), f16v(vv.x >> 16), f16v(vv.y & 0xFFFFu), f16v(vv.y >> 16)};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float prod = __fmul_rn(u, v[j]);
                t[j] = __fsub_rn(t[j], prod);
                uv[j] += static_cast<double>(prod);
            }
        }
        const float rr[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const double d = static_cast<double>(rr[j]) - uv[j];
            acc = fma(d, d, acc);
        }
        if (T) *reinterpret_cast<float4*>(T + o) = make_float4(t[0], t[1], t[2], t[3]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
    if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double sum = 0.0;
        for (int w = 0; w < kApplyThreads / 32; ++w) sum += ws[w];
        part[blockIdx.x] = sum;
    }
}

// err[round] = sqrt(sum of parts); best[0] keeps the lowest error so far
// (fp64), flag[0] = 1 when this round is the new best (the first round always).
__global__ void __launch_bounds__(256) err_sum_kernel(const double* part, int nparts, int round, float* err,
                                                      double* best, int* improved) {
    __shared__ double red[256];
    double s = 0.0;
    for (int i = threadIdx.x; i < nparts; i += 256) s += part[i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double e = sqrt(red[0]);
        if (err) err[round] = static_cast<float>(e);
        const bool better = round == 0 || e < best[0];
        if (better) best[0] = e;
        improved[0] = better ? 1 : 0;
    }
}

// dst = src (16-byte units) when improved[0] is set.
__global__ void copy_best_kernel(const int* improved, const uint4* src0, uint4* dst0, size_t n0, const uint4* src1,
                                 uint4* dst1, size_t n1, const uint4* src2, uint4* dst2, size_t n2) {
    if (!improved[0]) return;
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    const size_t i0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (size_t i = i0; i < n0; i += stride) dst0[i] = src0[i];
    for (size_t i = i0; i < n1; i += stride) dst1[i] = src1[i];
    for (size_t i = i0; i < n2; i += stride) dst2[i] = src2[i];
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

namespace {

constexpr int kGramChunk = 64;    // rows per Gram partial
// Split reductions: a product whose output tiles fill fewer than 148 blocks and
// whose reduction is long splits it into S slices (S x blocks <= 296) summed in
// slice order by split_sum_kernel, so the partials fit kSplitFloats.
constexpr int kSplitFloats = 296 * 2 * kGT * kGT;   // S x (blocks of up to 128 x 64) <= 296 x 8192

struct QuantWs {
    size_t R, T, Y, Y2, Z, Z2, B, part, gpart, G, M, MU, MV, U, V, blob, epart, best, flag, total;
    int l, chunks, eblocks;
};

QuantWs quant_layout(int N, int K, const milo_lorc_params& p) {
    QuantWs w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = round_up(off + bytes, 256);
        return o;
    };
    const int r = p.rank;
    const int l = r > 0 ? p.sketch : 0;
    w.l = l;
    w.R = take(static_cast<size_t>(N) * K * 4);
    if (r > 0) {
        w.Y = take(static_cast<size_t>(N) * l * 4);
        w.Y2 = take(static_cast<size_t>(N) * l * 4);
        w.Z = take(static_cast<size_t>(K) * l * 4);
        w.Z2 = take(static_cast<size_t>(K) * l * 4);
        w.B = take(static_cast<size_t>(l) * K * 4);
        w.gpart = take(static_cast<size_t>(kSplitFloats) * 4);
        if (p.rounds > 0) w.T = take(static_cast<size_t>(N) * K * 4);
        w.chunks = (std::max(N, K) + kGramChunk - 1) / kGramChunk;
        w.part = take(static_cast<size_t>(w.chunks) * l * l * 8);
        w.G = take(static_cast<size_t>(l) * l * 8);
        w.M = take(static_cast<size_t>(l) * l * 4);
        w.MU = take(static_cast<size_t>(l) * r * 4);
        w.MV = take(static_cast<size_t>(r) * l * 4);
        w.U = take(static_cast<size_t>(N) * r * 2);
        w.V = take(static_cast<size_t>(r) * K * 2);
    }
    w.blob = take(static_cast<size_t>((N + 63) / 64) * (K / 128) * kBlockSB);
    w.eblocks = static_cast<int>((static_cast<long long>(N) * (K / 4) + kApplyThreads - 1) / kApplyThreads);
    w.epart = take(static_cast<size_t>(w.eblocks) * 8);
    w.best = take(8);
    w.flag = take(4);
    w.total = off;
    return w;
}

milo_status check_hqq(int N, int K, int rank, int iters, float beta, float kappa, const char* who) {
    const std::string f = who;
    if (N <= 0 || K <= 0) return fail(MILO_ERR_INVALID_ARG, f + ": N and K must be positive");
    if (K % 128) return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": K must be a multiple of 128");
    if (N > (1 << 22) || K > (1 << 22) || static_cast<long long>(N) * K > (1LL << 34))
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": N and K at most 4194304 and N * K at most 2^34");
    if (rank < 0) return fail(MILO_ERR_INVALID_ARG, f + ": negative rank");
    if (rank > MILO_MAX_RANK) return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": rank above 64");
    if (iters < 0 || iters > 1000) return fail(MILO_ERR_INVALID_ARG, f + ": hqq_iters outside 0..1000");
    if (!(beta > 0.0f) || !isfinite(beta) || !(kappa > 0.0f) || !isfinite(kappa))
        return fail(MILO_ERR_INVALID_ARG, f + ": hqq_beta and hqq_kappa must be finite and positive");
    return MILO_OK;
}

milo_status launch_hqq(const HqqArgs& a, cudaStream_t st) {
    const long long threads = static_cast<long long>((a.N + 63) / 64 * 64) * (a.K / 128);
    hqq_pack_kernel<<<static_cast<unsigned>((threads + 127) / 128), 128, 0, st>>>(a);
    return check_launch("hqq_pack_kernel");
}

milo_status gemm(cudaStream_t st, int M, int Nn, int Kd, const float* A, long long sam, long long sak, const float* B,
                 long long sbk, long long sbn, float* C, uint16_t* C16, long long ldc, int32_t* dev_status,
                 float* gpart) {
    const bool tall = M >= 2 * kGT;                  // 128-row tiles when the output is tall
    const int TM = tall ? 2 * kGT : kGT;
    const int gx = (Nn + kGT - 1) / kGT, gy = (M + TM - 1) / TM;
    int S = 1;
    if (gpart && gx * gy < 148 && Kd >= 2048) S = std::min(8, std::max(1, 296 / (gx * gy)));
    const int kslice = static_cast<int>(round_up((Kd + S - 1) / S, kGK));
    S = (Kd + kslice - 1) / kslice;
    const GemmArgs a{M, Nn, Kd, A, sam, sak, B, sbk, sbn, C, C16, ldc, dev_status, S > 1 ? gpart : nullptr, kslice};
    if (tall) sgemm_kernel<2 * kGT><<<dim3(gx, gy, S), 256, 0, st>>>(a);
    else sgemm_kernel<kGT><<<dim3(gx, gy, S), 256, 0, st>>>(a);
    if (S > 1) {
        const long long e = static_cast<long long>(M) * Nn;
        split_sum_kernel<<<static_cast<unsigned>((e + 255) / 256), 256, 0, st>>>(gpart, S, M, Nn, C, C16, ldc,
                                                                                dev_status);
    }
    return check_launch("sgemm_kernel");
}

// G = X^T X for X(i, c) = X[i * sxi + c * sxc], i < M, c < l.
milo_status gram(cudaStream_t st, const float* X, long long sxi, long long sxc, int M, int l, double* part,
                 double* G) {
    const int chunks = (M + kGramChunk - 1) / kGramChunk;
    const GramArgs g{X, sxi, sxc, part, M, l, kGramChunk};
    gram_kernel<<<chunks, 256, 0, st>>>(g);
    gram_sum_kernel<<<(l * l + 255) / 256, 256, 0, st>>>(part, chunks, l * l, G);
    return check_launch("gram_kernel");
}

size_t chol_smem(int l) { return static_cast<size_t>(l) * (l + 1) * 8; }          // two packed triangles
size_t jacobi_smem(int l) { return static_cast<size_t>(l) * (l + 1) * (8 + 4); }  // fp64 matrix, fp32 P

// Y [M, l] <- a basis of its columns: Cholesky QR once (between power steps,
// where only the spanned subspace matters) or twice (orthonormal to fp32
// rounding, for the Rayleigh-Ritz step).  The result is in Y either way.
milo_status orth(cudaStream_t st, float* Y, float* Y2, int M, int l, uint8_t* base, const QuantWs& w,
                 int32_t* dev_status, int passes) {
    milo_status s;
    double* G = reinterpret_cast<double*>(base + w.G);
    float* Mm = reinterpret_cast<float*>(base + w.M);
    float* gpart = reinterpret_cast<float*>(base + w.gpart);
    for (int pass = 0; pass < passes; ++pass) {
        if ((s = gram(st, Y, l, 1, M, l, reinterpret_cast<double*>(base + w.part), G)) != MILO_OK) return s;
        chol_kernel<<<1, 256, chol_smem(l), st>>>(G, l, Mm);
        if ((s = check_launch("chol_kernel")) != MILO_OK) return s;
        // the product lands in the other buffer; after an odd pass copy it back
        if ((s = gemm(st, M, l, l, Y, l, 1, Mm, l, 1, Y2, nullptr, l, dev_status, gpart)) != MILO_OK) return s;
        std::swap(Y, Y2);
    }
    if (passes % 2)
        return check_cuda(cudaMemcpyAsync(Y2, Y, static_cast<size_t>(M) * l * 4, cudaMemcpyDeviceToDevice, st),
                          "orth copy");
    return MILO_OK;
}

// U fp16 [N, r], V fp16 [r, K] from R [N, K] (randomized subspace iteration).
milo_status compensator(cudaStream_t st, const float* R, const float* omega, int N, int K, int r, int q,
                        uint8_t* base, const QuantWs& w, uint16_t* U, uint16_t* V, int32_t* dev_status) {
    milo_status s;
    const int l = w.l;
    float* Y = reinterpret_cast<float*>(base + w.Y);
    float* Y2 = reinterpret_cast<float*>(base + w.Y2);
    float* Z = reinterpret_cast<float*>(base + w.Z);
    float* Z2 = reinterpret_cast<float*>(base + w.Z2);
    float* Bm = reinterpret_cast<float*>(base + w.B);
    double* G = reinterpret_cast<double*>(base + w.G);
    float* gpart = reinterpret_cast<float*>(base + w.gpart);
    if ((s = gemm(st, N, l, K, R, K, 1, omega, l, 1, Y, nullptr, l, dev_status, gpart)) != MILO_OK) return s;
    if ((s = orth(st, Y, Y2, N, l, base, w, dev_status, q > 0 ? 1 : 2)) != MILO_OK) return s;
    for (int it = 0; it < q; ++it) {
        if ((s = gemm(st, K, l, N, R, 1, K, Y, l, 1, Z, nullptr, l, dev_status, gpart)) != MILO_OK) return s;
        if ((s = orth(st, Z, Z2, K, l, base, w, dev_status, 1)) != MILO_OK) return s;
        if ((s = gemm(st, N, l, K, R, K, 1, Z, l, 1, Y, nullptr, l, dev_status, gpart)) != MILO_OK) return s;
        if ((s = orth(st, Y, Y2, N, l, base, w, dev_status, it + 1 < q ? 1 : 2)) != MILO_OK) return s;
    }
    if ((s = gemm(st, l, K, N, Y, 1, l, R, K, 1, Bm, nullptr, K, dev_status, gpart)) != MILO_OK) return s;
    if ((s = gram(st, Bm, 1, K, K, l, reinterpret_cast<double*>(base + w.part), G)) != MILO_OK) return s;
    float* MU = reinterpret_cast<float*>(base + w.MU);
    float* MV = reinterpret_cast<float*>(base + w.MV);
    jacobi_kernel<<<1, 256, jacobi_smem(l), st>>>(G, l, r, MU, MV);
    if ((s = check_launch("jacobi_kernel")) != MILO_OK) return s;
    if ((s = gemm(st, N, r, l, Y, l, 1, MU, r, 1, nullptr, U, r, dev_status, gpart)) != MILO_OK) return s;
    return gemm(st, r, K, l, MV, l, 1, Bm, K, 1, nullptr, V, K, dev_status, gpart);
}

}  // namespace

}  // namespace milo

using namespace milo;

extern "C" milo_status milo_hqq_pack(const uint16_t* W, const uint16_t* U, const uint16_t* V, int32_t rank,
                                     int32_t N, int32_t K, int32_t hqq_iters, float hqq_beta, float hqq_kappa,
                                     void* packed, float* residual, int32_t* dev_status, void* stream) {
    clear_error();
    milo_status s = check_hqq(N, K, rank, hqq_iters, hqq_beta, hqq_kappa, "milo_hqq_pack");
    if (s != MILO_OK) return s;
    if (!W || !packed) return fail(MILO_ERR_INVALID_ARG, "milo_hqq_pack: NULL W or packed");
    if (rank > 0 && (!U || !V)) return fail(MILO_ERR_INVALID_ARG, "milo_hqq_pack: NULL U or V with rank > 0");
    if (!aligned(packed, 16) || !aligned(W, 2) || (residual && !aligned(residual, 4)))
        return fail(MILO_ERR_INVALID_ARG, "milo_hqq_pack: misaligned buffer (packed needs 16 bytes)");
    const HqqArgs a{W, rank > 0 ? U : nullptr, rank > 0 ? V : nullptr, nullptr, static_cast<uint8_t*>(packed), residual,
                    dev_status, N, K, rank, hqq_iters, hqq_beta, hqq_kappa};
    return launch_hqq(a, static_cast<cudaStream_t>(stream));
}

static milo_status check_lorc(int32_t N, int32_t K, const milo_lorc_params* p, const char* who) {
    const std::string f = who;
    if (!p) return fail(MILO_ERR_INVALID_ARG, f + ": NULL params");
    milo_status s = check_hqq(N, K, p->rank, p->hqq_iters, p->hqq_beta, p->hqq_kappa, who);
    if (s != MILO_OK) return s;
    if (p->rank % 8) return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": rank must be a multiple of 8");
    if (p->rounds < 0 || p->rounds > 16) return fail(MILO_ERR_INVALID_ARG, f + ": rounds outside 0..16");
    if (p->rank > 0) {
        if (p->sketch < p->rank || p->sketch > kMaxSketch || p->sketch % 16)
            return fail(MILO_ERR_INVALID_ARG, f + ": sketch must be a multiple of 16 in rank..128");
        if (p->power_iters < 0 || p->power_iters > 8)
            return fail(MILO_ERR_INVALID_ARG, f + ": power_iters outside 0..8");
    }
    return MILO_OK;
}

extern "C" milo_status milo_quantize_lorc_workspace(int32_t N, int32_t K, const milo_lorc_params* params,
                                                    size_t* bytes) {
    clear_error();
    milo_status s = check_lorc(N, K, params, "milo_quantize_lorc_workspace");
    if (s != MILO_OK) return s;
    if (!bytes) return fail(MILO_ERR_INVALID_ARG, "milo_quantize_lorc_workspace: NULL bytes");
    *bytes = quant_layout(N, K, *params).total;
    return MILO_OK;
}

extern "C" milo_status milo_quantize_lorc(const uint16_t* W, int32_t N, int32_t K, const milo_lorc_params* params,
                                          const float* omega, void* packed, uint16_t* U, uint16_t* V, float* err,
                                          void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
    clear_error();
    milo_status s = check_lorc(N, K, params, "milo_quantize_lorc");
    if (s != MILO_OK) return s;
    const milo_lorc_params p = *params;
    const int r = p.rank;
    if (!W || !packed || !ws) return fail(MILO_ERR_INVALID_ARG, "milo_quantize_lorc: NULL W, packed or ws");
    if (r > 0 && (!omega || !U || !V))
        return fail(MILO_ERR_INVALID_ARG, "milo_quantize_lorc: NULL omega, U or V with rank > 0");
    if (!aligned(packed, 16) || !aligned(ws, 256) || !aligned(W, 8) || (r > 0 && (!aligned(U, 16) ||
        !aligned(V, 16) || !aligned(omega, 4))) || (err && !aligned(err, 4)))
        return fail(MILO_ERR_INVALID_ARG,
                    "milo_quantize_lorc: misaligned buffer (W needs 8 bytes, packed, U, V 16, ws 256)");
    const QuantWs w = quant_layout(N, K, p);
    if (ws_bytes < w.total) return fail(MILO_ERR_WORKSPACE, "milo_quantize_lorc: workspace too small");
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (r > 0) {
        if ((s = check_cuda(cudaFuncSetAttribute(chol_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(chol_smem(w.l))),
                            "chol_kernel attribute")) != MILO_OK)
            return s;
        if ((s = check_cuda(cudaFuncSetAttribute(jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(jacobi_smem(w.l))),
                            "jacobi_kernel attribute")) != MILO_OK)
            return s;
    }
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* R = reinterpret_cast<float*>(base + w.R);
    uint16_t* Uw = r > 0 ? reinterpret_cast<uint16_t*>(base + w.U) : nullptr;
    uint16_t* Vw = r > 0 ? reinterpret_cast<uint16_t*>(base + w.V) : nullptr;
    uint8_t* blob = base + w.blob;
    double* best = reinterpret_cast<double*>(base + w.best);
    int* improved = reinterpret_cast<int*>(base + w.flag);
    const size_t blob_bytes = static_cast<size_t>((N + 63) / 64) * (K / 128) * kBlockSB;
    const int rounds = r > 0 ? p.rounds : 0;
    float* T = p.rounds > 0 && r > 0 ? reinterpret_cast<float*>(base + w.T) : nullptr;
    for (int t = 0; t <= rounds; ++t) {
        // round t quantises W (t = 0) or the target W - U V formed by the last round
        const HqqArgs h{W, nullptr, nullptr, t > 0 ? T : nullptr, blob, R, dev_status, N, K, 0, p.hqq_iters,
                        p.hqq_beta, p.hqq_kappa};
        if ((s = launch_hqq(h, st)) != MILO_OK) return s;
        if (r > 0 && (s = compensator(st, R, omega, N, K, r, p.power_iters, base, w, Uw, Vw, dev_status)) != MILO_OK)
            return s;
        apply_kernel<<<w.eblocks, kApplyThreads, 0, st>>>(R, W, Uw, Vw, N, K, r, t < rounds ? T : nullptr,
                                                          reinterpret_cast<double*>(base + w.epart));
        err_sum_kernel<<<1, 256, 0, st>>>(reinterpret_cast<double*>(base + w.epart), w.eblocks, t, err, best,
                                          improved);
        copy_best_kernel<<<296, 256, 0, st>>>(improved, reinterpret_cast<const uint4*>(blob),
                                              static_cast<uint4*>(packed), blob_bytes / 16,
                                              reinterpret_cast<const uint4*>(Uw), reinterpret_cast<uint4*>(U),
                                              r > 0 ? static_cast<size_t>(N) * r * 2 / 16 : 0,
                                              reinterpret_cast<const uint4*>(Vw), reinterpret_cast<uint4*>(V),
                                              r > 0 ? static_cast<size_t>(r) * K * 2 / 16 : 0);
        if ((s = check_launch("milo_quantize_lorc round")) != MILO_OK) return s;
    }
    return MILO_OK;
}
