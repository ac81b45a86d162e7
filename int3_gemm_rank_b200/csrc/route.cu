// route.cu -- top-k softmax router and stable expert grouping.
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators", section "Background": an MoE layer activates a subset of its
// experts for each token.  Routing here is the Mixtral-style top-k over the
// router logits, and the grouping (per-expert histogram, exclusive scan,
// stable scatter) turns the top-k ids into per-expert row lists for the
// grouped GEMM.  The grouping is one thread block (a single block keeps the
// scatter stable without inter-block synchronisation); the top-k runs in
// that block for few tokens and on many blocks, one launch earlier, for many.
#include <cuda_runtime.h>

#include "milo_device.cuh"
#include "milo_host.h"

namespace milo {

constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kTopkThreads = 256;            // multi-block top-k: one warp per token
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kRouteSplitT = 512;            // from this many tokens the top-k runs on many blocks

// Top-k of token t, one warp: the lanes hold the token's logits (expert e at
// lane e % 32, slot e / 32) and k rounds of a warp arg-max pick the largest
// remaining logit, ties to the lower expert id.  A 32-bit key orders by value
// (the fp16 bits made order-preserving) in its high half and by descending id
// in its low half, so one warp max-reduction picks; 0 marks empty or picked.
// NaN counts as -inf (and is flagged).  Slot j = j-th pick.
__device__ __forceinline__ void topk_token(const uint16_t* __restrict__ logits, int t, int E, int k, uint32_t flags,
                                           int32_t* __restrict__ ids, float* __restrict__ wts, int lane,
                                           int32_t& st) {
    constexpr int kSlots = (MILO_MAX_EXPERTS + 31) / 32;
    const uint16_t* l = logits + static_cast<size_t>(t) * E;
    float v[kSlots];
    uint32_t key[kSlots];
#pragma unroll
    for (int i = 0; i < kSlots; ++i) {
        const int e = 32 * i + lane;
        v[i] = -INFINITY;
        key[i] = 0u;   // below every real key: empty or already picked
        if (e < E) {
            uint32_t b = l[e];
            float x = __half2float(__ushort_as_half(static_cast<uint16_t>(b)));
            if (!isfinite(x)) st |= MILO_DEV_NONFINITE;
            if (x != x) {
                x = -INFINITY;
                b = 0xFC00u;   // fp16 -inf
            }
            v[i] = x;
            const uint32_t ord = (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
            key[i] = (ord << 16) | (0xFFFFu - static_cast<uint32_t>(e));
        }
    }
    // lane j keeps pick j (k <= 16 < 32); the renormalising sum runs in slot order
    int my_e = 0;
    float my_v = 0.0f, m = 0.0f, den = 0.0f;
    for (int j = 0; j < k; ++j) {
        uint32_t best = 0u;
#pragma unroll
        for (int i = 0; i < kSlots; ++i) best = max(best, key[i]);
        best = __reduce_max_sync(0xFFFFFFFFu, best);
        const int e = static_cast<int>(0xFFFFu - (best & 0xFFFFu));
        const uint32_t ord = best >> 16;
        const float val = __half2float(__ushort_as_half(static_cast<uint16_t>((ord & 0x8000u) ? (ord & 0x7FFFu) : (~ord & 0xFFFFu))));
        if (j == 0) m = val;
        if (flags & MILO_ROUTE_RENORM) den += expf(val - m);
        if (lane == j) {
            my_e = e;
            my_v = val;
        }
#pragma unroll
        for (int i = 0; i < kSlots; ++i)
            if (32 * i + lane == e) key[i] = 0u;
    }
    if (!(flags & MILO_ROUTE_RENORM)) {
#pragma unroll
        for (int i = 0; i < kSlots; ++i)
            if (32 * i + lane < E) den += expf(v[i] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xFFFFFFFFu, den, o);
    }
    if (lane < k) {
        ids[static_cast<size_t>(t) * k + lane] = my_e;
        wts[static_cast<size_t>(t) * k + lane] = expf(my_v - m) / den;
    }
}

// Many tokens: the top-k alone, one warp per token over many blocks.
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const uint16_t* __restrict__ logits, int T, int E, int k,
                                                            uint32_t flags, int32_t* __restrict__ ids,
                                                            float* __restrict__ wts, int32_t* __restrict__ dev_status) {
    grid_dep_launch();
    grid_dep_wait();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * kTopkWarps + (threadIdx.x >> 5);
    int32_t st = 0;
    if (t < T) topk_token(logits, t, E, k, flags, ids, wts, lane, st);
    if (lane == 0) flag(dev_status, st);
}

// The grouping, one block: per-expert histogram (one atomic per expert per
// warp), exclusive scan, stable scatter of the flat slots f = t * k + j into
// expert order.  With `topk` set the block first runs the top-k of all tokens
// itself (few tokens: one launch instead of two).
__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel(const uint16_t* __restrict__ logits, int T, int E, int k, uint32_t flags, int topk,
             int32_t* __restrict__ ids, float* __restrict__ wts, int32_t* __restrict__ offsets,
             int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
             int32_t* __restrict__ dev_status) {
    __shared__ int count[MILO_MAX_EXPERTS + 1];
    __shared__ int cursor[MILO_MAX_EXPERTS];
    __shared__ int wcnt[kRouteWarps][MILO_MAX_EXPERTS];   // per chunk: slots of expert e in warp w, then
                                                          // the exclusive prefix over warps
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int F = T * k;
    int32_t st = 0;
    grid_dep_launch();
    grid_dep_wait();

    if (topk)
        for (int t = warp; t < T; t += kRouteWarps) topk_token(logits, t, E, k, flags, ids, wts, lane, st);
    for (int e = tid; e <= E; e += kRouteThreads) count[e] = 0;
    __syncthreads();

    // -- histogram: lanes with the same expert add once
    for (int base = 0; base < F; base += kRouteThreads) {
        const int f = base + tid;
        const int e = f < F ? ids[f] : -1;
        const bool valid = f < F && e >= 0 && e < E;
        if (f < F && !valid) st |= MILO_DEV_BAD_EXPERT_ID;
        const unsigned same = __match_any_sync(0xFFFFFFFFu, valid ? e : -1);
        if (valid && __ffs(same) - 1 == lane) atomicAdd(&count[e], __popc(same));
    }
    __syncthreads();

    // -- exclusive scan over the experts: warp 0, 32 experts per round
    if (warp == 0) {
        int run = 0;
        for (int b0 = 0; b0 < E; b0 += 32) {
            const int e = b0 + lane;
            const int c = e < E ? count[e] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            if (e < E) {
                offsets[e] = run + incl - c;
                cursor[e] = run + incl - c;
            }
            run += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) offsets[E] = run;
    }
    __syncthreads();

    // -- stable scatter, one chunk of kRouteThreads flat slots at a time: rank
    //    within the warp from match_any, rank across warps from the prefix of
    //    the per-warp counts
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < F; base += kRouteThreads) {
        for (int i = tid; i < kRouteWarps * E; i += kRouteThreads) wcnt[i / E][i % E] = 0;
        __syncthreads();
        const int f = base + tid;
        const int e = f < F ? ids[f] : -1;
        const bool valid = f < F && e >= 0 && e < E;
        const unsigned same = __match_any_sync(0xFFFFFFFFu, valid ? e : -1);
        const int rank = __popc(same & lt_mask);
        if (valid && rank == 0) wcnt[warp][e] = __popc(same);
        __syncthreads();
        for (int x = tid; x < E; x += kRouteThreads) {
            int run = cursor[x];
            for (int w = 0; w < kRouteWarps; ++w) {
                const int c = wcnt[w][x];
                wcnt[w][x] = run;
                run += c;
            }
            cursor[x] = run;
        }
        __syncthreads();
        if (valid) {
            const int p = wcnt[warp][e] + rank;
            if (in_range(dev_status, p >= 0 && p < F)) {
                perm[p] = f;
                inv_perm[f] = p;
            }
        } else if (f < F) {
            inv_perm[f] = -1;
        }
        __syncthreads();
    }
    flag(dev_status, st);
}

}  // namespace milo

using namespace milo;

extern "C" milo_status milo_route(const uint16_t* logits, int32_t T, int32_t E, int32_t k,
                                  uint32_t flags, int32_t* topk_ids, float* topk_w,
                                  int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm,
                                  int32_t* dev_status, void* stream) {
    clear_error();
    if (T < 0) return fail(MILO_ERR_INVALID_ARG, "milo_route: T must be >= 0");
    if (E < 1 || E > MILO_MAX_EXPERTS)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_route: E must be in [1, 256]");
    if (k < 1 || k > E || k > MILO_MAX_TOPK)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_route: k must be in [1, min(E, 16)]");
    if (flags & ~(MILO_ROUTE_RENORM | MILO_ROUTE_IDS_GIVEN))
        return fail(MILO_ERR_INVALID_ARG, "milo_route: unknown flag");
    if (!topk_ids || !expert_offsets || (T > 0 && (!perm || !inv_perm)))
        return fail(MILO_ERR_INVALID_ARG, "milo_route: NULL output");
    if (!(flags & MILO_ROUTE_IDS_GIVEN) && T > 0 && (!logits || !topk_w))
        return fail(MILO_ERR_INVALID_ARG, "milo_route: logits and topk_w are required");
    if (static_cast<long long>(T) * k > MILO_MAX_ROWS)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_route: T*k above MILO_MAX_ROWS");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool want_topk = !(flags & MILO_ROUTE_IDS_GIVEN) && T > 0;
    const bool split = want_topk && T >= kRouteSplitT;
    if (split) {
        milo_status s = check_cuda(launch_pdl(topk_kernel, dim3((T + kTopkWarps - 1) / kTopkWarps), dim3(kTopkThreads),
                                              0, st, logits, T, E, k, flags, topk_ids, topk_w, dev_status),
                                   "milo_route (top-k)");
        if (s != MILO_OK) return s;
    }
    return check_cuda(launch_pdl(route_kernel, dim3(1), dim3(kRouteThreads), 0, st, logits, T, E, k, flags,
                                 (want_topk && !split) ? 1 : 0, topk_ids, topk_w, expert_offsets, perm, inv_perm,
                                 dev_status),
                      "milo_route");
}
