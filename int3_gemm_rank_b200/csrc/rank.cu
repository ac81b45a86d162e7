// rank.cu -- adaptive compensator ranks: the kurtosis of a weight matrix
// (sm_100a reduction) and the allocation of a rank budget by score (host).
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators", section "MiLo Algorithm: Mixture of Low-Rank Compensators",
// adaptive rank selection: weights with a higher kurtosis (heavier tails, more
// quantisation error) get a higher rank (strategy 3), and so do experts that
// are activated more often (strategy 2).  Both reduce to "more rank for a
// higher score"; milo_assign_ranks takes the scores.
//
// Kurtosis: one pass over the fp16 entries with fp64 power sums (w^2 and w^4 of
// an fp16 value are exact in fp64), a fixed grid so that the partial sums and
// their order do not depend on the device, and a one-block final step.
// HBM-bound: 2 bytes per entry.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "milo_device.cuh"
#include "milo_host.h"

namespace milo {

namespace {

constexpr int kKurtBlocks = 592;      // 4 blocks per SM on 148 SMs, fixed
constexpr int kKurtThreads = 256;

// Thread (b, t) sums w, w^2, w^3, w^4 over the 8-entry pieces i = 8 (b * 256 +
// t) + 8 * 592 * 256 * k, k = 0, 1, ... (16-byte loads, four issued before
// their arithmetic so that enough bytes are in flight), in increasing k; then
// the block adds its threads in a fixed tree.
constexpr int kKurtUnroll = 4;

__device__ __forceinline__ void kurt_piece(const uint16_t* __restrict__ W, long long i, long long count,
                                           uint16_t (&v)[8]) {
    if (i + 8 <= count) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(W + i));
        const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[2 * j] = static_cast<uint16_t>(w4[j] & 0xFFFFu);
            v[2 * j + 1] = static_cast<uint16_t>(w4[j] >> 16);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = i + j < count ? W[i + j] : 0;   // +0 adds nothing
    }
}

__global__ void __launch_bounds__(kKurtThreads) kurt_partial_kernel(const uint16_t* __restrict__ W, long long count,
                                                                    double* __restrict__ part,
                                                                    int32_t* __restrict__ dev_status) {
    __shared__ double red[4][kKurtThreads];
    double s1 = 0.0, s2 = 0.0, s3 = 0.0, s4 = 0.0;
    int32_t st = 0;
    const long long piece = static_cast<long long>(gridDim.x) * blockDim.x * 8;
    for (long long i0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i0 < count;
         i0 += kKurtUnroll * piece) {
        uint16_t v[kKurtUnroll][8];
#pragma unroll
        for (int u = 0; u < kKurtUnroll; ++u) {
            const long long i = i0 + u * piece;
            if (i < count) kurt_piece(W, i, count, v[u]);
            else
#pragma unroll
                for (int j = 0; j < 8; ++j) v[u][j] = 0;
        }
#pragma unroll
        for (int u = 0; u < kKurtUnroll; ++u)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const double x = static_cast<double>(__half2float(__ushort_as_half(v[u][j])));
                if (!isfinite(x)) st |= MILO_DEV_NONFINITE;
                const double x2 = x * x;
                s1 += x;
                s2 += x2;
                s3 += x2 * x;
                s4 += x2 * x2;
            }
    }
    red[0][threadIdx.x] = s1;
    red[1][threadIdx.x] = s2;
    red[2][threadIdx.x] = s3;
    red[3][threadIdx.x] = s4;
    __syncthreads();
    for (int o = kKurtThreads / 2; o > 0; o >>= 1) {
        if (threadIdx.x < o)
#pragma unroll
            for (int m = 0; m < 4; ++m) red[m][threadIdx.x] += red[m][threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x < 4) part[blockIdx.x * 4 + threadIdx.x] = red[threadIdx.x][0];
    flag(dev_status, st);
}

// out[0] = m4 / m2^2 from the block partials: thread t adds partials t,
// t + 256, ... in order, then a fixed tree over the threads.  m2 = 0 (a
// constant matrix) gives 0.
__global__ void __launch_bounds__(kKurtThreads) kurt_final_kernel(const double* __restrict__ part, int nparts,
                                                                  long long count, double* __restrict__ out) {
    __shared__ double red[4][kKurtThreads];
    double s[4] = {0.0, 0.0, 0.0, 0.0};
    for (int b = threadIdx.x; b < nparts; b += kKurtThreads)
#pragma unroll
        for (int m = 0; m < 4; ++m) s[m] += part[b * 4 + m];
#pragma unroll
    for (int m = 0; m < 4; ++m) red[m][threadIdx.x] = s[m];
    __syncthreads();
    for (int o = kKurtThreads / 2; o > 0; o >>= 1) {
        if (threadIdx.x < o)
#pragma unroll
            for (int m = 0; m < 4; ++m) red[m][threadIdx.x] += red[m][threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x != 0) return;
    const double n = static_cast<double>(count);
    const double mu = red[0][0] / n, e2 = red[1][0] / n, e3 = red[2][0] / n, e4 = red[3][0] / n;
    const double m2 = e2 - mu * mu;
    const double m4 = e4 - 4.0 * mu * e3 + 6.0 * mu * mu * e2 - 3.0 * mu * mu * mu * mu;
    out[0] = m2 > 0.0 ? m4 / (m2 * m2) : 0.0;
}

}  // namespace

}  // namespace milo

using namespace milo;

extern "C" milo_status milo_kurtosis_workspace(size_t* bytes) {
    clear_error();
    if (!bytes) return fail(MILO_ERR_INVALID_ARG, "milo_kurtosis_workspace: NULL bytes");
    *bytes = static_cast<size_t>(kKurtBlocks) * 4 * sizeof(double);
    return MILO_OK;
}

extern "C" milo_status milo_kurtosis(const uint16_t* W, int64_t count, double* out, void* ws, size_t ws_bytes,
                                     int32_t* dev_status, void* stream) {
    clear_error();
    if (count <= 0) return fail(MILO_ERR_INVALID_ARG, "milo_kurtosis: count must be positive");
    if (!W || !out || !ws) return fail(MILO_ERR_INVALID_ARG, "milo_kurtosis: NULL pointer");
    if (!aligned(W, 16) || !aligned(ws, 8) || !aligned(out, 8))
        return fail(MILO_ERR_INVALID_ARG, "milo_kurtosis: W must be 16-byte aligned, ws and out 8-byte");
    if (ws_bytes < static_cast<size_t>(kKurtBlocks) * 4 * sizeof(double))
        return fail(MILO_ERR_WORKSPACE, "milo_kurtosis: workspace too small");
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    double* part = static_cast<double*>(ws);
    kurt_partial_kernel<<<kKurtBlocks, kKurtThreads, 0, st>>>(W, count, part, dev_status);
    kurt_final_kernel<<<1, kKurtThreads, 0, st>>>(part, kKurtBlocks, count, out);
    return check_launch("milo_kurtosis");
}

// Rank budget by score (host).  Units of 8 ranks: the budget is
// floor(n * avg_rank / 8) units, each matrix at most max_rank / 8.  Shares
// proportional to the scores (negative scores count as 0; when no remaining
// score is positive the rest is shared equally), with water-filling at the
// cap: matrices whose share reaches the cap are fixed there and the rest is
// re-shared among the others.  Then each takes the floor of its share and the
// leftover units go one each in decreasing order of the fractional part (ties:
// higher score, then lower index), pass after pass until the budget is used
// or every matrix is at the cap.
extern "C" milo_status milo_assign_ranks(const double* score, int32_t n, int32_t avg_rank, int32_t max_rank,
                                         int32_t* ranks) {
    clear_error();
    if (n <= 0 || !score || !ranks) return fail(MILO_ERR_INVALID_ARG, "milo_assign_ranks: bad arguments");
    if (avg_rank < 0 || max_rank < 0 || max_rank > MILO_MAX_RANK || max_rank % 8)
        return fail(MILO_ERR_INVALID_ARG, "milo_assign_ranks: max_rank must be a multiple of 8 in 0..64");
    for (int i = 0; i < n; ++i)
        if (!std::isfinite(score[i])) return fail(MILO_ERR_INVALID_ARG, "milo_assign_ranks: non-finite score");
    const long long cap = max_rank / 8;
    long long units = std::min(static_cast<long long>(n) * avg_rank / 8, cap * n);
    std::vector<double> s(n), share(n, 0.0);
    double total = 0.0;
    for (int i = 0; i < n; ++i) total += (s[i] = std::max(score[i], 0.0));
    if (!(total > 0.0)) std::fill(s.begin(), s.end(), 1.0);
    std::vector<char> fixed(n, 0);
    double left = static_cast<double>(units);
    std::vector<double> eff(s);
    for (;;) {
        double active = 0.0;
        for (int i = 0; i < n; ++i)
            if (!fixed[i]) active += eff[i];
        if (!(active > 0.0)) {                 // only zero scores left: share the rest equally
            for (int i = 0; i < n; ++i)
                if (!fixed[i]) eff[i] = 1.0;
            for (int i = 0; i < n; ++i)
                if (!fixed[i]) active += eff[i];
        }
        bool changed = false;
        for (int i = 0; i < n; ++i) {
            if (fixed[i]) continue;
            share[i] = active > 0.0 ? left * eff[i] / active : 0.0;
            if (share[i] >= static_cast<double>(cap)) {
                share[i] = static_cast<double>(cap);
                fixed[i] = 1;
                left -= static_cast<double>(cap);
                changed = true;
            }
        }
        if (!changed) break;
    }
    std::vector<long long> u(n);
    long long used = 0;
    for (int i = 0; i < n; ++i) used += (u[i] = std::min(cap, static_cast<long long>(std::floor(share[i]))));
    std::vector<int> order(n);
    for (int i = 0; i < n; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
        const double fa = share[a] - std::floor(share[a]), fb = share[b] - std::floor(share[b]);
        if (fa != fb) return fa > fb;
        return s[a] > s[b];
    });
    while (used < units) {                     // passes over the order until the budget is used
        bool took = false;
        for (int k = 0; k < n && used < units; ++k) {
            const int i = order[k];
            if (u[i] < cap) {
                ++u[i];
                ++used;
                took = true;
            }
        }
        if (!took) break;
    }
    for (int i = 0; i < n; ++i) ranks[i] = static_cast<int32_t>(8 * u[i]);
    return MILO_OK;
}
