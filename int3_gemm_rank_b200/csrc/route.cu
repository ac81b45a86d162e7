// route.cu -- top-k softmax router and stable expert grouping.
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators", section "Background": an MoE layer activates a subset of its
// experts for each token.  Routing here is the Mixtral-style top-k over the
// router logits, and the grouping (per-expert histogram, exclusive scan,
// stable scatter) turns the top-k ids into per-expert row lists for the
// grouped GEMM.  One thread block does the whole job: the router is a few
// microseconds even for 8192 tokens, and a single block keeps the scatter
// stable without inter-block synchronisation.
#include <cuda_runtime.h>

#include "milo_device.cuh"
#include "milo_host.h"

namespace milo {

constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;

__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel(const uint16_t* __restrict__ logits, int T, int E, int k, uint32_t flags,
             int32_t* __restrict__ ids, float* __restrict__ wts, int32_t* __restrict__ offsets,
             int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
             int32_t* __restrict__ dev_status) {
    __shared__ int count[MILO_MAX_EXPERTS + 1];
    __shared__ int cursor[MILO_MAX_EXPERTS];
    __shared__ int wcnt[kRouteWarps][MILO_MAX_EXPERTS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int F = T * k;
    int32_t st = 0;
    grid_dep_launch();
    grid_dep_wait();

    // -- top-k per token: insertion into a list kept in descending logit order;
    //    a strictly larger logit is needed to pass an entry, so equal logits
    //    keep ascending expert order.
    if (!(flags & MILO_ROUTE_IDS_GIVEN)) {
        for (int t = tid; t < T; t += kRouteThreads) {
            const uint16_t* l = logits + static_cast<size_t>(t) * E;
            float lv[MILO_MAX_TOPK];
            int le[MILO_MAX_TOPK];
            int n = 0;
            for (int e = 0; e < E; ++e) {
                const float v = __half2float(__ushort_as_half(l[e]));
                if (!isfinite(v)) st |= MILO_DEV_NONFINITE;
                if (n == k && !(v > lv[k - 1])) continue;
                int pos = n < k ? n : k - 1;
                while (pos > 0 && v > lv[pos - 1]) {
                    lv[pos] = lv[pos - 1];
                    le[pos] = le[pos - 1];
                    --pos;
                }
                lv[pos] = v;
                le[pos] = e;
                if (n < k) ++n;
            }
            const float m = lv[0];
            float den = 0.0f;
            if (flags & MILO_ROUTE_RENORM) {
                for (int j = 0; j < k; ++j) den += expf(lv[j] - m);
            } else {
                for (int e = 0; e < E; ++e) den += expf(__half2float(__ushort_as_half(l[e])) - m);
            }
            for (int j = 0; j < k; ++j) {
                ids[static_cast<size_t>(t) * k + j] = le[j];
                wts[static_cast<size_t>(t) * k + j] = expf(lv[j] - m) / den;
            }
        }
    }
    for (int e = tid; e <= E; e += kRouteThreads) count[e] = 0;
    __syncthreads();

    // -- histogram
    for (int f = tid; f < F; f += kRouteThreads) {
        const int e = ids[f];
        if (e < 0 || e >= E) st |= MILO_DEV_BAD_EXPERT_ID;
        else atomicAdd(&count[e], 1);
    }
    __syncthreads();

    // -- exclusive scan (E <= 256: one thread is enough)
    if (tid == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            const int c = count[e];
            offsets[e] = run;
            cursor[e] = run;
            run += c;
        }
        offsets[E] = run;
    }
    __syncthreads();

    // -- stable scatter, one chunk of kRouteThreads flat slots at a time:
    //    rank within the warp from match_any, rank across warps from a
    //    per-warp count table.
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < F; base += kRouteThreads) {
        for (int i = tid; i < kRouteWarps * E; i += kRouteThreads) wcnt[i / E][i % E] = 0;
        __syncthreads();
        const int f = base + tid;
        int e = f < F ? ids[f] : -1;
        const bool valid = f < F && e >= 0 && e < E;
        const int key = valid ? e : -1;
        const unsigned same = __match_any_sync(0xFFFFFFFFu, key);
        const int rank = __popc(same & lt_mask);
        if (valid && rank == 0) wcnt[warp][e] = __popc(same);
        __syncthreads();
        if (valid) {
            int p = cursor[e] + rank;
            for (int w = 0; w < warp; ++w) p += wcnt[w][e];
            perm[p] = f;
            inv_perm[f] = p;
        } else if (f < F) {
            inv_perm[f] = -1;
        }
        __syncthreads();
        for (int x = tid; x < E; x += kRouteThreads) {
            int add = 0;
            for (int w = 0; w < kRouteWarps; ++w) add += wcnt[w][x];
            cursor[x] += add;
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
    if (static_cast<long long>(T) * k > 0x3FFFFFFFLL)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_route: T*k too large");
    return check_cuda(launch_pdl(route_kernel, dim3(1), dim3(kRouteThreads), 0, static_cast<cudaStream_t>(stream),
                                 logits, T, E, k, flags, topk_ids, topk_w, expert_offsets, perm, inv_perm,
                                 dev_status),
                      "milo_route");
}
