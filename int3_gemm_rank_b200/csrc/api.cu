// api.cu -- host side of libmilo: argument validation, device tables,
// workspace layout and the launch sequence of the forward.
//
// The sequence for one MoE layer ("MiLo: Efficient Quantized MoE Inference
// with Mixture of Low-Rank Compensators": routed experts, each a quantised
// weight plus a rank-r compensator, outputs mixed by the router weights):
//   few rows per expert (mma.sync GEMMs):
//     prep(x, row bookkeeping) -> gemv<SwiGLU>(w1|w3, t = x V1|V3^T inside)
//        -> prep(h) -> gemv(w2, t = h V2^T inside) -> combine
//   many rows per expert (tcgen05 GEMMs):
//     prep(x, row bookkeeping) -> lorc(x, V1|V3) -> tc<SwiGLU>(w1|w3)
//        -> prep(h) -> lorc(h, V2) -> tc(w2) -> combine
// Every step is a kernel on the caller's stream; the host never waits.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <string>
#include <vector>

#include "milo_host.h"
#include "milo_kernels.h"

namespace milo {

static thread_local std::string g_last_error;
void clear_error() { g_last_error.clear(); }
void set_error(const std::string& msg) { g_last_error = msg; }

// ---------------------------------------------------------------------------
// tensor maps of the tcgen05 GEMM (driver entry point fetched through the
// runtime; no -lcuda)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major tensor [rows, cols] with row pitch `pitch` bytes; box {bcols, brows}.
static milo_status make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols,
                            uint64_t rows, uint64_t pitch, uint32_t bcols, uint32_t brows, const char* what,
                            CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MILO_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {pitch};
    cuuint32_t box[2] = {bcols, brows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MILO_ERR_INVALID_ARG, std::string("tensor map encoding failed for ") + what + " (code " +
                                              std::to_string(static_cast<int>(r)) + ")");
    return MILO_OK;
}

// Measurement hook (milo_set_profile_events).
static cudaEvent_t g_prof[4] = {nullptr, nullptr, nullptr, nullptr};
static int g_prof_n = 0;

static void prof_record(int i, cudaStream_t st) {
    if (i < g_prof_n && g_prof[i]) cudaEventRecord(g_prof[i], st);
}

static int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// ---------------------------------------------------------------------------
// tables
// ---------------------------------------------------------------------------
static milo_status fill_proj(ProjDev* d, const milo_qweight& w, int N, int K, const char* what) {
    memset(d, 0, sizeof(*d));
    if (!w.packed) return fail(MILO_ERR_INVALID_ARG, std::string(what) + ": NULL packed weight");
    if (w.rank < 0 || w.rank % 8 || w.rank > MILO_MAX_RANK)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE,
                    std::string(what) + ": rank must be a multiple of 8 in [0, 64]");
    if (w.rank > 0 && (!w.U || !w.V))
        return fail(MILO_ERR_INVALID_ARG, std::string(what) + ": U and V are required when rank > 0");
    if (!aligned(w.packed, 16) || (w.rank > 0 && (!aligned(w.U, 16) || !aligned(w.V, 16))))
        return fail(MILO_ERR_INVALID_ARG, std::string(what) + ": pointers must be 16-byte aligned");
    if (w.lorc_format != MILO_LORC_F16 && w.lorc_format != MILO_LORC_INT3)
        return fail(MILO_ERR_INVALID_ARG, std::string(what) + ": unknown compensator format");
    const bool int3 = w.rank > 0 && w.lorc_format == MILO_LORC_INT3;
    if (int3 && N % 128)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE,
                    std::string(what) + ": an int3 compensator needs N to be a multiple of 128");
    d->packed = static_cast<const uint8_t*>(w.packed);
    d->U = w.rank > 0 ? static_cast<const uint16_t*>(w.U) : nullptr;
    d->V = w.rank > 0 ? static_cast<const uint16_t*>(w.V) : nullptr;
    d->rank = w.rank;
    d->N = N;
    d->K = K;
    d->lorc3 = int3 ? 1 : 0;
    // fp16 V for the mma.sync GEMM's t-items: 32 rank rows x 64 of K per box
    // (rows past the rank read as zeros)
    if (w.rank > 0 && !int3)
        return make_map(&d->vmap, w.V, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, static_cast<uint64_t>(K), w.rank,
                        static_cast<uint64_t>(K) * 2, 64, 32, "V", CU_TENSOR_MAP_SWIZZLE_128B);
    return MILO_OK;
}

static milo_status check_nk(int N, int K, const std::string& what) {
    if (N <= 0 || K <= 0) return fail(MILO_ERR_INVALID_ARG, what + ": sizes must be positive");
    if (N > kMaxWeightRows) return fail(MILO_ERR_UNSUPPORTED_SHAPE, what + ": N above 2^31 - 64");
    if (K > kMaxProjK) return fail(MILO_ERR_UNSUPPORTED_SHAPE, what + ": K above 2^24");
    if (K % 128) return fail(MILO_ERR_UNSUPPORTED_SHAPE, what + ": K must be a multiple of 128");
    if (N % 16) return fail(MILO_ERR_UNSUPPORTED_SHAPE, what + ": N must be a multiple of 16");
    return MILO_OK;
}

// The shape fields of a grouped projection or a layer as the preparation
// accepts them.  The size queries and the calls check them again, and once
// prepared also max_rank (it sizes the compensator's rows and stages), since
// the planning divides by and multiplies with every one of them.
static milo_status check_linear(const milo_linear* lin, bool prepared, const char* what) {
    const std::string f = what;
    if (lin->group != MILO_GROUP) return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": group must be 64");
    if (lin->n_experts < 1 || lin->n_experts > MILO_MAX_EXPERTS)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": n_experts must be in [1, 256]");
    const milo_status s = check_nk(lin->N, lin->K, f);
    if (s != MILO_OK) return s;
    if (prepared && (lin->max_rank < 0 || lin->max_rank > MILO_MAX_RANK || lin->max_rank % 8))
        return fail(MILO_ERR_INVALID_ARG, f + ": max_rank is not one milo_linear_prepare sets (0..64, multiple of 8)");
    return MILO_OK;
}

static milo_status check_layer(const milo_moe_layer* L, bool prepared, const char* what) {
    const std::string f = what;
    if (L->group != MILO_GROUP) return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": group must be 64");
    if (L->n_routed < 1 || L->n_shared < 0 || L->n_routed > MILO_MAX_EXPERTS || L->n_shared > MILO_MAX_EXPERTS ||
        L->n_routed + L->n_shared > MILO_MAX_EXPERTS)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": experts: need n_routed >= 1 and n_routed + n_shared <= 256");
    if (L->top_k < 1 || L->top_k > L->n_routed || L->top_k > MILO_MAX_TOPK)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": top_k must be in [1, min(n_routed, 16)]");
    milo_status s;
    if ((s = check_nk(L->inter, L->hidden, f + " (w1/w3)")) != MILO_OK) return s;
    if ((s = check_nk(L->hidden, L->inter, f + " (w2)")) != MILO_OK) return s;
    if (L->hidden % 4) return fail(MILO_ERR_UNSUPPORTED_SHAPE, f + ": hidden must be a multiple of 4");
    if (prepared && (L->max_rank < 0 || L->max_rank > MILO_MAX_RANK || L->max_rank % 8))
        return fail(MILO_ERR_INVALID_ARG, f + ": max_rank is not one milo_layer_prepare sets (0..64, multiple of 8)");
    return MILO_OK;
}

static milo_status upload(void* device_table, size_t table_bytes, const std::vector<ProjDev>& t) {
    if (!device_table || !aligned(device_table, 64))
        return fail(MILO_ERR_WORKSPACE, "device table must be a 64-byte aligned device buffer");
    const size_t need = t.size() * sizeof(ProjDev);
    if (table_bytes < need) return fail(MILO_ERR_WORKSPACE, "device table too small");
    return check_cuda(cudaMemcpy(device_table, t.data(), need, cudaMemcpyHostToDevice), "table upload");
}

// Which grouped GEMM runs.  The mma.sync kernel suits a few routed rows per
// expert (decode): a tcgen05.mma of N = 16 costs as much to issue as one of
// N = 64.  With many rows per expert (prefill) the weights are reused across
// 128-row tiles and the tcgen05 kernel takes over.  milo_set_gemm_path (or
// MILO_GEMM=mma|tc in the environment, read once) forces one; both give the
// same results within fp32 rounding.
static std::atomic<int> g_gemm_path{-1};   // -1: not yet read from the environment

static int gemm_path() {
    int v = g_gemm_path.load(std::memory_order_relaxed);
    if (v >= 0) return v;
    static std::once_flag once;
    std::call_once(once, [] {
        const char* e = getenv("MILO_GEMM");
        int m = MILO_GEMM_AUTO;
        if (e && e[0] == 't') m = MILO_GEMM_TC;
        else if (e && e[0] == 'm') m = MILO_GEMM_MMA;
        int unset = -1;
        g_gemm_path.compare_exchange_strong(unset, m);
    });
    return g_gemm_path.load(std::memory_order_relaxed);
}

static bool use_tc(long long routed_rows, int n_routed) {
    const int path = gemm_path();
    if (path == MILO_GEMM_TC) return true;
    if (path == MILO_GEMM_MMA) return false;
    return routed_rows >= 64LL * std::max(1, n_routed);
}

// ---------------------------------------------------------------------------
// workspace layouts
// ---------------------------------------------------------------------------
struct Carve {
    size_t off = 0;
    size_t take(size_t bytes) {
        const size_t o = off;
        off = round_up(off + bytes, 256);
        return o;
    }
};

// Prepared activations and group sums of R rows: chunk-major (K chunks of 256).
static int chunks_of(int K) { return (K + kChunkK - 1) / kChunkK; }
static size_t frag_bytes(int K, int R) {
    // the mma.sync layout; the tcgen05 layout [R][K] fp16 is never larger
    return static_cast<size_t>(chunks_of(K)) * R * kFragRowHalves * 2;
}
// zero-point operand of the tcgen05 path: per row and pair of super-blocks,
// the four group sums as fp16 (hi, lo, hi, lo): [R][chunks][16] fp16
static size_t gsum_bytes(int K, int R) { return static_cast<size_t>(chunks_of(K)) * R * 32; }

struct LorcPlan {
    int splits, row_groups;
};

// slice counters of the compensator kernel: (expert, projection, 16-rank block, row group <= 8)
static int lorc_counters(int n_exp) { return n_exp * 2 * ((MILO_MAX_RANK + 15) / 16) * 8; }

struct LinearWs {
    size_t grp, rows, inv, rscale, frag, gsum, t, tpart, done, part, plain, total;
    int R, splits, tcols, nzero;
    bool tc;
    LorcPlan lp;
};

static int tiles_of(int N, int rows) { return (N + rows - 1) / rows; }

// Split-K factor for the plain kernel: make the estimated item count fill the
// persistent grid in whole waves (the tail "shift" of the work distribution).
static int choose_splits(long long base_items, int chunks) {
    const int slots = 3 * sm_count();
    if (base_items <= 0) return 1;
    int best = 1;
    double best_eff = -1.0;
    for (int s = 1; s <= 16 && s <= chunks; ++s) {
        const double items = static_cast<double>(base_items) * s;
        const double waves = items / slots;
        double eff = waves / std::ceil(waves);
        if (waves < 1.0) eff = waves;                     // under-filled grid
        eff -= 0.004 * (s - 1);                           // partial-sum traffic
        if (eff > best_eff + 1e-9) { best_eff = eff; best = s; }
    }
    // with ceil(chunks / best) chunks per split, every split must get one
    const int cps = (chunks + best - 1) / best;
    return (chunks + cps - 1) / cps;
}

// K slices and row-tile groups of the compensator down-projection.  A block
// handles one 16-row tile of one expert for one K slice, so its latency is a
// couple of staging rounds: slices of about four super-blocks (the last one
// may be shorter) while the row tiles alone do not fill the GPU, and enough
// row groups for the largest possible group (max_rows), capped in blocks.
static LorcPlan lorc_plan(int n_exp, int nproj, int K, long long max_rows) {
    const long long base = static_cast<long long>(n_exp) * nproj * ((MILO_MAX_RANK + 15) / 16);
    const int sb = K / 128;
    const long long tiles = std::max(1LL, (max_rows + 15) / 16);
    LorcPlan pl{1, 1};
    pl.splits = tiles >= 8 ? 1 : std::max(1, (sb + 3) / 4);
    pl.row_groups = static_cast<int>(std::min<long long>(tiles, std::max(1LL, 65536 / (base * pl.splits))));
    if (pl.splits > 1) pl.row_groups = std::min(pl.row_groups, 8);   // the slice counters cover 8 row groups
    return pl;
}

// K slices of the compensator's t-items inside the mma.sync GEMM: at least
// two pipeline stages (256 of K each) per slice, and at most this many slices
// (the kernel takes fewer, longer ones when the t-items outnumber the CTAs).
static int t_slice_len(int) { return 512; }
static int t_slices(int K) { return (K + t_slice_len(K) - 1) / t_slice_len(K); }

// The rows of one call, counted in 64 bits before the 32-bit planning below:
// T*k routed slots (grouped linear), plus n_shared*T shared-expert rows (MoE
// layer).  A call above MILO_MAX_ROWS is refused before anything is planned.
static milo_status check_linear_rows(int T, int k, const char* what) {
    if (static_cast<long long>(T) * k > MILO_MAX_ROWS)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, std::string(what) + ": T*k above MILO_MAX_ROWS");
    return MILO_OK;
}

static milo_status check_moe_rows(const milo_moe_layer* L, int T, const char* what) {
    // top_k and n_shared are in range here (check_layer first)
    if (static_cast<long long>(T) * (L->top_k + L->n_shared) > MILO_MAX_ROWS)
        return fail(MILO_ERR_UNSUPPORTED_SHAPE, std::string(what) + ": T*(top_k + n_shared) above MILO_MAX_ROWS");
    return MILO_OK;
}

static LinearWs linear_ws(const milo_linear* lin, int T, int k) {
    LinearWs w;
    Carve c;
    w.R = T * k;
    w.tc = use_tc(static_cast<long long>(T) * k, lin->n_experts);
    const int n_exp = lin->n_experts;
    const int chunks = (lin->K + kChunkK - 1) / kChunkK;
    const long long groups = std::min<long long>(n_exp, std::max(1LL, static_cast<long long>(T) * k));
    const long long tt = std::max(1LL, (static_cast<long long>(T) * k + kTokTile - 1) / kTokTile);
    w.splits = choose_splits(std::max(groups, tt) * tiles_of(lin->N, kRowsPlain), chunks);
    w.tcols = std::max(8, lin->max_rank);
    w.grp = c.take(static_cast<size_t>(n_exp) * 8);
    w.rows = c.take(static_cast<size_t>(w.R) * 4);
    w.inv = c.take(static_cast<size_t>(w.R) * 4);
    w.rscale = c.take(static_cast<size_t>(w.R) * 4);
    w.frag = c.take(frag_bytes(lin->K, w.R));
    w.gsum = c.take(gsum_bytes(lin->K, w.R));
    w.t = c.take(static_cast<size_t>(w.R) * w.tcols * 2);
    w.lp = lorc_plan(n_exp, 1, lin->K, static_cast<long long>(T) * k);   // at most all rows in one expert
    // the tcgen05 path: the down-projection kernel's K slices; the mma.sync
    // path: its t-items' K slices, the rows' plain copy, and their counters
    const int tslices = w.tc ? w.lp.splits : t_slices(lin->K);
    w.tpart = c.take(static_cast<size_t>(tslices) * w.R * w.tcols * 4);
    w.nzero = lorc_counters(n_exp) + (w.tc ? 0 : gemv_sync_ints(w.R, n_exp));
    w.done = c.take(static_cast<size_t>(w.nzero) * 4);
    w.part = c.take(static_cast<size_t>(w.splits) * w.R * lin->N * 4);
    w.plain = w.tc ? 0 : c.take(static_cast<size_t>(w.R) * lin->K * 2);
    w.total = c.off;
    return w;
}

struct MoeWs {
    size_t grp, rows, xscale, xfrag, xg, t13, h, hscale, hfrag, hg, t2, tpart, done, part, xplain, hplain, total;
    int R, R_routed, splits, tc13, tc2, nzero, sync13, sync2;
    bool tc;
    LorcPlan lp13, lp2;
};

static MoeWs moe_ws(const milo_moe_layer* L, int T) {
    MoeWs w;
    Carve c;
    const int H = L->hidden, I = L->inter;
    w.R_routed = T * L->top_k;
    w.R = w.R_routed + L->n_shared * T;
    w.tc = use_tc(w.R_routed, L->n_routed);
    const int n_exp = L->n_routed + L->n_shared;
    const int chunks = (I + kChunkK - 1) / kChunkK;
    // 16-row token tiles: the routed rows fill at least one per expert they
    // reach and at least R_routed / 16 in all; each shared expert sees all T
    // tokens
    const long long routed_tt = std::max(std::min<long long>(L->n_routed, std::max(1LL, static_cast<long long>(w.R_routed))),
                                         (static_cast<long long>(w.R_routed) + kTokTile - 1) / kTokTile);
    const long long token_tiles = routed_tt + static_cast<long long>(L->n_shared) * ((T + kTokTile - 1) / kTokTile);
    w.splits = choose_splits(token_tiles * tiles_of(H, kRowsPlain), chunks);
    w.tc13 = std::max(8, 2 * L->max_rank);
    w.tc2 = std::max(8, L->max_rank);
    w.grp = c.take(static_cast<size_t>(n_exp) * 8);
    w.rows = c.take(static_cast<size_t>(w.R) * 4);
    w.xscale = c.take(static_cast<size_t>(w.R) * 4);
    w.xfrag = c.take(frag_bytes(H, w.R));
    w.xg = c.take(gsum_bytes(H, w.R));
    w.t13 = c.take(static_cast<size_t>(w.R) * w.tc13 * 2);
    w.h = c.take(static_cast<size_t>(w.R) * I * 2);
    w.hscale = c.take(static_cast<size_t>(w.R) * 4);
    w.hfrag = c.take(frag_bytes(I, w.R));
    w.hg = c.take(gsum_bytes(I, w.R));
    w.t2 = c.take(static_cast<size_t>(w.R) * w.tc2 * 2);
    // a token meets an expert at most once, and a shared expert sees every token
    w.lp13 = lorc_plan(n_exp, 2, H, T);
    w.lp2 = lorc_plan(n_exp, 1, I, T);
    // the down-projection kernels' slices (tcgen05 path) or the t-items' (mma.sync path)
    const size_t s13 = w.tc ? w.lp13.splits : t_slices(H), s2 = w.tc ? w.lp2.splits : t_slices(I);
    w.tpart = c.take(std::max(s13 * w.tc13, s2 * w.tc2) * w.R * 4);
    // counters, all zeroed by the first preparation: the down-projection
    // kernels', then (mma.sync path) those of the w1|w3 and w2 GEMMs
    w.sync13 = w.tc ? 0 : gemv_sync_ints(w.R, n_exp);
    w.sync2 = w.tc ? 0 : gemv_sync_ints(w.R, n_exp);
    w.nzero = lorc_counters(n_exp) + w.sync13 + w.sync2;
    w.done = c.take(static_cast<size_t>(w.nzero) * 4);
    w.part = c.take(static_cast<size_t>(w.splits) * w.R * H * 4);
    w.xplain = w.tc ? 0 : c.take(static_cast<size_t>(w.R) * H * 2);
    w.hplain = w.tc ? 0 : c.take(static_cast<size_t>(w.R) * I * 2);
    w.total = c.off;
    return w;
}

// ---------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------
static void act_ptrs(GemvParams& g, void* frag, void* rscale, void* t, int R, int K, int tcols, bool has_t) {
    g.x = static_cast<const uint16_t*>(frag);
    g.rscale = static_cast<const float*>(rscale);
    g.t = has_t ? static_cast<uint16_t*>(t) : nullptr;
    g.R = R;
    g.K = K;
    g.SB = K / 128;
    g.G = K / MILO_GROUP;
    g.chunks = chunks_of(K);
    g.has_t = has_t;
    g.tcols = tcols;
}

static milo_status run_gemv(GemvParams& g, bool glu, cudaStream_t st, const char* what) {
    return check_cuda(launch_gemv(g, glu, sm_count(), st), what);
}

// The t-items of a grouped GEMM on the mma.sync path: the compensator's t from
// the rows' plain copy, K slices and counters in the workspace.
static milo_status t_items(GemvParams& g, const void* plain, void* tpart, int32_t* sync) {
    g.t_items = g.has_t ? 1 : 0;
    g.src = static_cast<const uint16_t*>(plain);
    g.kslice = t_slice_len(g.K);
    g.nks = t_slices(g.K);
    g.tpart = static_cast<float*>(tpart);
    const int tiles = (g.R + kTokTile - 1) / kTokTile + g.n_exp;   // as gemv_sync_ints
    g.tctr = sync;
    g.tdone = sync + 4 * tiles;
    if (!g.has_t) return MILO_OK;
    return make_map(&g.smap, plain, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, static_cast<uint64_t>(g.K),
                    static_cast<uint64_t>(g.R), static_cast<uint64_t>(g.K) * 2, 64, kTokTile, "plain rows",
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

// The grouped GEMM described by g on the tcgen05 kernel: activations in
// A-column order [R][K] fp16 with the zero-point operand [R][chunks][16] fp16.
static milo_status run_tc(const GemvParams& g, bool glu, void* xcol, void* gsum, cudaStream_t st,
                          const char* what) {
    TcParams p;
    memset(&p, 0, sizeof(p));
    milo_status s;
    const int Rm = std::max(g.R, 1);
    const int chunks = chunks_of(g.K);
    if ((s = make_map(&p.b_map, xcol, CU_TENSOR_MAP_DATA_TYPE_UINT16, g.K, Rm, static_cast<uint64_t>(g.K) * 2, 64,
                      kTcTokens, "activations", CU_TENSOR_MAP_SWIZZLE_128B)) != MILO_OK)
        return s;
    if ((s = make_map(&p.z_map, gsum, CU_TENSOR_MAP_DATA_TYPE_UINT16, 16 * chunks, Rm,
                      static_cast<uint64_t>(chunks) * 32, 16, kTcTokens, "group sums",
                      CU_TENSOR_MAP_SWIZZLE_32B)) != MILO_OK)
        return s;
    if (g.has_t && (s = make_map(&p.t_map, g.t, CU_TENSOR_MAP_DATA_TYPE_UINT16, g.tcols, Rm,
                                 static_cast<uint64_t>(g.tcols) * 2, 64, kTcTokens, "compensator rows",
                                 CU_TENSOR_MAP_SWIZZLE_128B)) != MILO_OK)
        return s;
    p.rscale = g.rscale;
    p.table = g.table;
    p.grp = g.grp;
    p.y_part = g.y_part;
    p.h = g.h;
    p.dev_status = g.dev_status;
    p.stride = g.stride;
    p.proj_a = g.proj_a;
    p.proj_b = g.proj_b;
    p.n_exp = g.n_exp;
    p.N = g.N;
    p.K = g.K;
    p.R = g.R;
    p.SB = g.K / 128;
    p.has_t = g.has_t;
    p.tcols = g.tcols;
    p.t_col_b = g.t_col_b;
    // keep the larger of an expert's routed activations and its weights hot
    // in L2: when the rows outweigh the weights, sweep the weight tiles fastest
    const double act_bytes = static_cast<double>(g.R) / std::max(1, g.n_exp) * g.K * 2.0;
    const double w_bytes = static_cast<double>(g.N) * (glu ? 2 : 1) * g.K * 7.0 / 16.0;
    p.ntile_fast = act_bytes > w_bytes ? 1 : 0;
    return check_cuda(launch_tc_gemm(p, glu, sm_count(), st), what);
}

}  // namespace milo

using namespace milo;

// ===========================================================================
// C ABI
// ===========================================================================

extern "C" const char* milo_status_str(milo_status s) {
    switch (s) {
        case MILO_OK: return "ok";
        case MILO_ERR_INVALID_ARG: return "invalid argument";
        case MILO_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MILO_ERR_WORKSPACE: return "workspace or table too small or misaligned";
        case MILO_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

extern "C" const char* milo_last_error(void) { return g_last_error.c_str(); }

extern "C" int32_t milo_version(void) { return 1; }

extern "C" milo_status milo_set_profile_events(void* const* events, int32_t n) {
    clear_error();
    if (n < 0 || n > 4 || (n > 0 && !events))
        return fail(MILO_ERR_INVALID_ARG, "milo_set_profile_events: n must be in [0, 4]");
    for (int i = 0; i < 4; ++i) g_prof[i] = i < n ? static_cast<cudaEvent_t>(events[i]) : nullptr;
    g_prof_n = n;
    return MILO_OK;
}

extern "C" milo_status milo_set_gemm_path(int32_t mode) {
    clear_error();
    if (mode != MILO_GEMM_AUTO && mode != MILO_GEMM_MMA && mode != MILO_GEMM_TC)
        return fail(MILO_ERR_INVALID_ARG, "milo_set_gemm_path: mode must be MILO_GEMM_AUTO, _MMA or _TC");
    g_gemm_path.store(mode, std::memory_order_relaxed);
    return MILO_OK;
}

extern "C" milo_status milo_table_bytes(int32_t n_projections, size_t* bytes) {
    clear_error();
    if (n_projections < 0 || !bytes) return fail(MILO_ERR_INVALID_ARG, "milo_table_bytes: bad argument");
    *bytes = static_cast<size_t>(n_projections) * sizeof(ProjDev);
    return MILO_OK;
}

extern "C" milo_status milo_linear_prepare(milo_linear* lin, const milo_qweight* weights,
                                           void* device_table, size_t table_bytes) {
    clear_error();
    if (!lin || !weights) return fail(MILO_ERR_INVALID_ARG, "milo_linear_prepare: NULL argument");
    milo_status s = check_linear(lin, false, "milo_linear_prepare");
    if (s != MILO_OK) return s;
    std::vector<ProjDev> t(lin->n_experts);
    int rmax = 0;
    for (int e = 0; e < lin->n_experts; ++e) {
        if ((s = fill_proj(&t[e], weights[e], lin->N, lin->K, "milo_linear_prepare")) != MILO_OK)
            return s;
        rmax = std::max(rmax, weights[e].rank);
    }
    if ((s = upload(device_table, table_bytes, t)) != MILO_OK) return s;
    lin->max_rank = rmax;
    lin->table = device_table;
    return MILO_OK;
}

extern "C" milo_status milo_layer_prepare(milo_moe_layer* L, const milo_expert* experts,
                                          void* device_table, size_t table_bytes) {
    clear_error();
    if (!L || !experts) return fail(MILO_ERR_INVALID_ARG, "milo_layer_prepare: NULL argument");
    milo_status s = check_layer(L, false, "milo_layer_prepare");
    if (s != MILO_OK) return s;
    const int n_exp = L->n_routed + L->n_shared;
    std::vector<ProjDev> t(3 * static_cast<size_t>(n_exp));
    int rmax = 0;
    for (int e = 0; e < n_exp; ++e) {
        if ((s = fill_proj(&t[3 * e + 0], experts[e].w1, L->inter, L->hidden, "w1")) != MILO_OK) return s;
        if ((s = fill_proj(&t[3 * e + 1], experts[e].w3, L->inter, L->hidden, "w3")) != MILO_OK) return s;
        if ((s = fill_proj(&t[3 * e + 2], experts[e].w2, L->hidden, L->inter, "w2")) != MILO_OK) return s;
        rmax = std::max({rmax, experts[e].w1.rank, experts[e].w3.rank, experts[e].w2.rank});
    }
    if ((s = upload(device_table, table_bytes, t)) != MILO_OK) return s;
    L->max_rank = rmax;
    L->table = device_table;
    return MILO_OK;
}

extern "C" milo_status milo_linear_workspace_bytes(const milo_linear* lin, int32_t T, int32_t k,
                                                   size_t* bytes) {
    clear_error();
    if (!lin || !bytes || T < 0 || k < 1) return fail(MILO_ERR_INVALID_ARG, "milo_linear_workspace_bytes");
    milo_status s = check_linear(lin, true, "milo_linear_workspace_bytes");
    if (s != MILO_OK) return s;
    if ((s = check_linear_rows(T, k, "milo_linear_workspace_bytes")) != MILO_OK) return s;
    *bytes = linear_ws(lin, T, k).total;
    return MILO_OK;
}

extern "C" milo_status milo_moe_workspace_bytes(const milo_moe_layer* L, int32_t T, size_t* bytes) {
    clear_error();
    if (!L || !bytes || T < 0) return fail(MILO_ERR_INVALID_ARG, "milo_moe_workspace_bytes");
    milo_status s = check_layer(L, true, "milo_moe_workspace_bytes");
    if (s != MILO_OK) return s;
    if ((s = check_moe_rows(L, T, "milo_moe_workspace_bytes")) != MILO_OK) return s;
    *bytes = moe_ws(L, T).total;
    return MILO_OK;
}

extern "C" size_t milo_moe_h_offset(const milo_moe_layer* L, int32_t T) {
    clear_error();
    if (!L || T < 0 || check_layer(L, true, "milo_moe_h_offset") != MILO_OK ||
        check_moe_rows(L, T, "milo_moe_h_offset") != MILO_OK)
        return 0;
    return moe_ws(L, T).h;
}

extern "C" milo_status milo_grouped_linear(const milo_linear* lin, const void* x, milo_dtype x_dt,
                                           int32_t T, int32_t k, const int32_t* expert_offsets,
                                           const int32_t* perm, void* y, milo_dtype y_dt, void* ws,
                                           size_t ws_bytes, int32_t* dev_status, void* stream) {
    clear_error();
    if (!lin || !lin->table) return fail(MILO_ERR_INVALID_ARG, "milo_grouped_linear: layer not prepared");
    if (const milo_status s0 = check_linear(lin, true, "milo_grouped_linear"); s0 != MILO_OK) return s0;
    if (T < 0 || k < 1 || k > MILO_MAX_TOPK) return fail(MILO_ERR_INVALID_ARG, "milo_grouped_linear: bad T or k");
    if (check_linear_rows(T, k, "milo_grouped_linear") != MILO_OK) return MILO_ERR_UNSUPPORTED_SHAPE;
    if (x_dt != MILO_F16 && x_dt != MILO_BF16) return fail(MILO_ERR_INVALID_ARG, "x must be fp16 or bf16");
    if (y_dt != MILO_F16 && y_dt != MILO_BF16 && y_dt != MILO_F32) return fail(MILO_ERR_INVALID_ARG, "bad y dtype");
    if (!perm && k != 1) return fail(MILO_ERR_INVALID_ARG, "perm may be NULL only with k == 1");
    if (T == 0) return MILO_OK;
    if (!x || !y || !expert_offsets || !ws) return fail(MILO_ERR_INVALID_ARG, "milo_grouped_linear: NULL pointer");
    if (!aligned(x, 16) || !aligned(y, 16)) return fail(MILO_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
    if (!aligned(ws, 256)) return fail(MILO_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (lin->N % 4) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "N must be a multiple of 4");
    const LinearWs w = linear_ws(lin, T, k);
    if (ws_bytes < w.total) return fail(MILO_ERR_WORKSPACE, "milo_grouped_linear: workspace too small");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(ws);
    int32_t* grp = reinterpret_cast<int32_t*>(base + w.grp);
    int32_t* rows = reinterpret_cast<int32_t*>(base + w.rows);
    int32_t* inv = reinterpret_cast<int32_t*>(base + w.inv);

    const bool tc = w.tc;
    float* rscale = reinterpret_cast<float*>(base + w.rscale);
    PrepParams pp = {};
    pp.src = static_cast<const uint16_t*>(x);
    pp.row_src = rows;
    pp.frag = reinterpret_cast<uint16_t*>(base + w.frag);
    pp.gsum = reinterpret_cast<uint16_t*>(base + w.gsum);
    pp.rscale = rscale;
    pp.layout = tc ? 1 : 0;
    pp.dev_status = dev_status;
    pp.R = w.R;
    pp.K = lin->K;
    pp.src_bf16 = x_dt == MILO_BF16;
    pp.rows = 1;
    pp.offsets = expert_offsets;
    pp.perm = perm;
    pp.grp = grp;
    pp.inv = inv;
    pp.T = T;
    pp.k = k;
    pp.E = lin->n_experts;
    pp.S = 0;
    pp.R_routed = w.R;
    pp.zero = reinterpret_cast<int32_t*>(base + w.done);
    pp.nzero = w.nzero;
    pp.plain = tc ? nullptr : reinterpret_cast<uint16_t*>(base + w.plain);
    milo_status s = check_cuda(launch_prep(pp, st), "prep");
    if (s != MILO_OK) return s;

    const bool has_t = lin->max_rank > 0;
    const ProjDev* table = static_cast<const ProjDev*>(lin->table);
    // the tcgen05 path takes t from the down-projection kernel; the mma.sync
    // GEMM computes it itself (t-items) and combines its own output tiles
    if (has_t && tc) {
        LorcParams lp = {};
        lp.src = static_cast<const uint16_t*>(x);
        lp.row_src = rows;
        lp.rscale = rscale;
        lp.table = table;
        lp.grp = grp;
        lp.t = reinterpret_cast<uint16_t*>(base + w.t);
        lp.part = reinterpret_cast<float*>(base + w.tpart);
        lp.done = reinterpret_cast<int32_t*>(base + w.done);
        lp.dev_status = dev_status;
        lp.stride = 1;
        lp.proj_a = 0;
        lp.proj_b = -1;
        lp.n_exp = lin->n_experts;
        lp.K = lin->K;
        lp.R = w.R;
        lp.tcols = w.tcols;
        lp.t_col_b = 0;
        lp.src_bf16 = x_dt == MILO_BF16;
        lp.splits = w.lp.splits;
        lp.row_groups = w.lp.row_groups;
        if ((s = check_cuda(launch_lorc(lp, st), "lorc")) != MILO_OK) return s;
    }

    GemvParams g;
    memset(&g, 0, sizeof(g));
    act_ptrs(g, base + w.frag, rscale, base + w.t, w.R, lin->K, w.tcols, has_t);
    g.table = table;
    g.grp = grp;
    g.y_part = reinterpret_cast<float*>(base + w.part);
    g.dev_status = dev_status;
    g.stride = 1;
    g.proj_a = 0;
    g.proj_b = 0;
    g.n_exp = lin->n_experts;
    g.N = lin->N;
    const int splits = tc ? 1 : w.splits;   // the tcgen05 kernel does not split K
    g.splits = splits;
    g.cps = (g.chunks + splits - 1) / splits;
    CombineParams cp{reinterpret_cast<const float*>(base + w.part), inv, nullptr, y, dev_status,
                     T, k, 0, lin->N, w.R, splits, w.R, static_cast<int>(y_dt), 1};
    prof_record(0, st);
    if (tc) {
        s = run_tc(g, false, base + w.frag, base + w.gsum, st, "tc gemm");
    } else {
        s = t_items(g, base + w.plain, base + w.tpart,
                    reinterpret_cast<int32_t*>(base + w.done) + lorc_counters(lin->n_experts));
        if (s == MILO_OK) s = run_gemv(g, false, st, "gemv");
    }
    if (s != MILO_OK) return s;
    prof_record(1, st);
    return check_cuda(launch_combine(cp, st), "combine");
}

extern "C" milo_status milo_moe_forward(const milo_moe_layer* L, const void* x, milo_dtype x_dt,
                                        int32_t T, const float* topk_w, const int32_t* expert_offsets,
                                        const int32_t* perm, const int32_t* inv_perm, void* y,
                                        milo_dtype y_dt, void* ws, size_t ws_bytes,
                                        int32_t* dev_status, void* stream) {
    clear_error();
    if (!L || !L->table) return fail(MILO_ERR_INVALID_ARG, "milo_moe_forward: layer not prepared");
    if (const milo_status s0 = check_layer(L, true, "milo_moe_forward"); s0 != MILO_OK) return s0;
    if (T < 0) return fail(MILO_ERR_INVALID_ARG, "milo_moe_forward: T must be >= 0");
    if (check_moe_rows(L, T, "milo_moe_forward") != MILO_OK) return MILO_ERR_UNSUPPORTED_SHAPE;
    if (x_dt != MILO_F16 && x_dt != MILO_BF16) return fail(MILO_ERR_INVALID_ARG, "x must be fp16 or bf16");
    if (y_dt != MILO_F16 && y_dt != MILO_BF16 && y_dt != MILO_F32) return fail(MILO_ERR_INVALID_ARG, "bad y dtype");
    if (T == 0) return MILO_OK;
    if (!x || !y || !topk_w || !expert_offsets || !perm || !inv_perm || !ws)
        return fail(MILO_ERR_INVALID_ARG, "milo_moe_forward: NULL pointer");
    if (!aligned(x, 16) || !aligned(y, 16)) return fail(MILO_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
    if (!aligned(ws, 256)) return fail(MILO_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    const MoeWs w = moe_ws(L, T);
    if (ws_bytes < w.total) return fail(MILO_ERR_WORKSPACE, "milo_moe_forward: workspace too small");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(ws);
    const int n_exp = L->n_routed + L->n_shared;
    const int H = L->hidden, I = L->inter;
    int32_t* grp = reinterpret_cast<int32_t*>(base + w.grp);
    int32_t* rows = reinterpret_cast<int32_t*>(base + w.rows);
    const ProjDev* table = static_cast<const ProjDev*>(L->table);
    const bool has_t = L->max_rank > 0;
    milo_status s;

    const bool tc = w.tc;
    int32_t* sync = reinterpret_cast<int32_t*>(base + w.done) + lorc_counters(n_exp);
    float* xscale = reinterpret_cast<float*>(base + w.xscale);
    float* hscale = reinterpret_cast<float*>(base + w.hscale);
    PrepParams px = {};
    px.src = static_cast<const uint16_t*>(x);
    px.row_src = rows;
    px.frag = reinterpret_cast<uint16_t*>(base + w.xfrag);
    px.gsum = reinterpret_cast<uint16_t*>(base + w.xg);
    px.rscale = xscale;
    px.layout = tc ? 1 : 0;
    px.dev_status = dev_status;
    px.R = w.R;
    px.K = H;
    px.src_bf16 = x_dt == MILO_BF16;
    px.rows = 1;
    px.offsets = expert_offsets;
    px.perm = perm;
    px.grp = grp;
    px.inv = nullptr;
    px.T = T;
    px.k = L->top_k;
    px.E = L->n_routed;
    px.S = L->n_shared;
    px.R_routed = w.R_routed;
    px.zero = reinterpret_cast<int32_t*>(base + w.done);
    px.nzero = w.nzero;
    px.plain = tc ? nullptr : reinterpret_cast<uint16_t*>(base + w.xplain);
    if ((s = check_cuda(launch_prep(px, st), "prep x")) != MILO_OK) return s;
    if (has_t && tc) {
        LorcParams lp = {};
        lp.src = static_cast<const uint16_t*>(x);
        lp.row_src = rows;
        lp.rscale = xscale;
        lp.table = table;
        lp.grp = grp;
        lp.t = reinterpret_cast<uint16_t*>(base + w.t13);
        lp.part = reinterpret_cast<float*>(base + w.tpart);
        lp.done = reinterpret_cast<int32_t*>(base + w.done);
        lp.dev_status = dev_status;
        lp.stride = 3;
        lp.proj_a = 0;
        lp.proj_b = 1;
        lp.n_exp = n_exp;
        lp.K = H;
        lp.R = w.R;
        lp.tcols = w.tc13;
        lp.t_col_b = L->max_rank;
        lp.src_bf16 = x_dt == MILO_BF16;
        lp.splits = w.lp13.splits;
        lp.row_groups = w.lp13.row_groups;
        if ((s = check_cuda(launch_lorc(lp, st), "lorc w1|w3")) != MILO_OK) return s;
    }

    GemvParams g1;
    memset(&g1, 0, sizeof(g1));
    act_ptrs(g1, base + w.xfrag, xscale, base + w.t13, w.R, H, w.tc13, has_t);
    g1.table = table;
    g1.grp = grp;
    g1.h = reinterpret_cast<uint16_t*>(base + w.h);
    g1.dev_status = dev_status;
    g1.stride = 3;
    g1.proj_a = 0;
    g1.proj_b = 1;
    g1.n_exp = n_exp;
    g1.N = I;
    g1.splits = 1;
    g1.cps = g1.chunks;
    g1.t_col_b = L->max_rank;
    prof_record(0, st);
    if (tc) {
        s = run_tc(g1, true, base + w.xfrag, base + w.xg, st, "tc gemm w1|w3");
    } else {
        s = t_items(g1, base + w.xplain, base + w.tpart, sync);
        if (s == MILO_OK) s = run_gemv(g1, true, st, "gemv w1|w3");
    }
    if (s != MILO_OK) return s;
    prof_record(1, st);

    PrepParams ph = {};
    ph.src = reinterpret_cast<const uint16_t*>(base + w.h);
    ph.row_src = nullptr;
    ph.frag = reinterpret_cast<uint16_t*>(base + w.hfrag);
    ph.gsum = reinterpret_cast<uint16_t*>(base + w.hg);
    ph.rscale = hscale;
    ph.layout = tc ? 1 : 0;
    ph.dev_status = dev_status;
    ph.R = w.R;
    ph.K = I;
    ph.src_bf16 = 0;
    ph.rows = 0;
    ph.plain = tc ? nullptr : reinterpret_cast<uint16_t*>(base + w.hplain);
    if ((s = check_cuda(launch_prep(ph, st), "prep h")) != MILO_OK) return s;
    if (has_t && tc) {
        LorcParams lp = {};
        lp.src = reinterpret_cast<const uint16_t*>(base + w.h);
        lp.row_src = nullptr;
        lp.rscale = hscale;
        lp.table = table;
        lp.grp = grp;
        lp.t = reinterpret_cast<uint16_t*>(base + w.t2);
        lp.part = reinterpret_cast<float*>(base + w.tpart);
        lp.done = reinterpret_cast<int32_t*>(base + w.done);
        lp.dev_status = dev_status;
        lp.stride = 3;
        lp.proj_a = 2;
        lp.proj_b = -1;
        lp.n_exp = n_exp;
        lp.K = I;
        lp.R = w.R;
        lp.tcols = w.tc2;
        lp.t_col_b = 0;
        lp.src_bf16 = 0;
        lp.splits = w.lp2.splits;
        lp.row_groups = w.lp2.row_groups;
        if ((s = check_cuda(launch_lorc(lp, st), "lorc w2")) != MILO_OK) return s;
    }

    GemvParams g2;
    memset(&g2, 0, sizeof(g2));
    act_ptrs(g2, base + w.hfrag, hscale, base + w.t2, w.R, I, w.tc2, has_t);
    g2.table = table;
    g2.grp = grp;
    g2.y_part = reinterpret_cast<float*>(base + w.part);
    g2.dev_status = dev_status;
    g2.stride = 3;
    g2.proj_a = 2;
    g2.proj_b = 2;
    g2.n_exp = n_exp;
    g2.N = H;
    const int splits = tc ? 1 : w.splits;   // the tcgen05 kernel does not split K
    g2.splits = splits;
    g2.cps = (g2.chunks + splits - 1) / splits;
    CombineParams cp{reinterpret_cast<const float*>(base + w.part), inv_perm, topk_w, y, dev_status,
                     T, L->top_k, L->n_shared, H, w.R, splits, w.R_routed, static_cast<int>(y_dt), 0};
    prof_record(2, st);
    if (tc) {
        s = run_tc(g2, false, base + w.hfrag, base + w.hg, st, "tc gemm w2");
    } else {
        s = t_items(g2, base + w.hplain, base + w.tpart, sync + w.sync13);
        if (s == MILO_OK) s = run_gemv(g2, false, st, "gemv w2");
    }
    if (s != MILO_OK) return s;
    prof_record(3, st);
    return check_cuda(launch_combine(cp, st), "combine");
}
