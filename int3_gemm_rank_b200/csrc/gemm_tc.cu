// gemm_tc.cu -- grouped int3 x fp16 GEMM with the low-rank compensator on the
// 5th-generation tensor cores (tcgen05.mma, tensor memory), sm_100a.
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators": "MiLo Algorithm" (W_out = W_quant + U V, so
// y = x W_quant^T + (x V^T) U^T, rank per expert, possibly 0) and "MiLo Kernel"
// (int3 x FP16 GEMM, dequantisation fused, zero point folded in, global loads
// overlapping the math).
//
// One CTA owns 128 weight rows (w1|w3: 64 features of each) and 16 routed rows
// of one expert; six warps:
//   warp 0      TMA producer: packed codes, scales/zeros, activations (already
//               in the order of the A columns and pre-scaled, 128-byte
//               swizzled) and per-group activation sums, 256 K per stage,
//               four stages;
//   warp 1      allocates 256 TMEM columns; one lane issues tcgen05.mma;
//   warps 2..5  one thread per weight row (TMEM lane): read the row's 12 words
//               of a 128-code super-block, extract 64 code pairs (one LOP3 per
//               pair; values code * 8^i * 2^-24, exact in fp16) and store them
//               with one tcgen05.st as the A operand (three A buffers).  The MMA
//               (M=128, N=16, K=16) accumulates each 64-code scale group into
//               its own TMEM buffer D_g = 2^-24 sum_k x_k q_k (four D buffers);
//               the same threads read D_g back and fold
//                   acc += s * 2^24 * D_g - s * z * sum_k x_k
//               in fp32 registers, only for the routed rows that exist.  The
//               compensator is one more MMA with A = U rows (w1 and w3 rows
//               side by side along K) and B = t = x V^T.  Epilogue: SwiGLU
//               through a shared-memory exchange, or fp32 split-K partials.
// Work items are enumerated on the device from the expert offsets (as in the
// mma.sync kernel); CTAs are persistent, two per SM.
#include <cuda_runtime.h>

#include "milo_device.cuh"
#include "milo_kernels.h"
#include "milo_tc.cuh"

namespace milo {

constexpr int kTcStages = 4;
constexpr int kTcStageBytes = 23552;   // multiple of 1024: swizzled tiles stay aligned
constexpr int kTcOffB = 0;             // activations [2 sb][2 K atoms][16 rows][128 B], swizzled
constexpr int kTcOffQ = 8192;          // packed codes [2 sb][128 rows][12 words]
constexpr int kTcOffS = 20480;         // scales / zeros, 2048 B
constexpr int kTcOffG = 22528;         // group sums [16 rows][4 groups] f32
constexpr int kTcStageTx = 8192 + 12288 + 2048 + 256;
constexpr int kTcOffU = 4096;          // compensator stage: t at kTcOffB (<= 2 atoms), U rows here
constexpr int kTcABufs = 3, kTcDBufs = 4;
constexpr int kTcDCol0 = kTcABufs * 64;
constexpr uint32_t kTcTmemCols = 256;
constexpr int kTcThreads = 192;
constexpr int kTcXch = kTcStages * kTcStageBytes;   // SwiGLU exchange [64][17] f32
constexpr int kTcBar = kTcXch + 4608;
constexpr int kTcNumBars = 2 * kTcStages + 2 * kTcABufs + 2 * kTcDBufs + 3;
constexpr int kTcTab = kTcBar + 8 * kTcNumBars + 16;
constexpr int kTcSmemUsed = kTcTab + 3 * (MILO_MAX_EXPERTS + 1) * 4;
constexpr int kTcSmemBytes = kTcSmemUsed + 1024;   // slack to align the base to 1024 B

static_assert(kTcStageTx <= kTcStageBytes, "stage layout");
static_assert(kTcOffU + 128 * MILO_MAX_RANK * 2 <= kTcStageBytes, "compensator stage");
static_assert(kTcDCol0 + kTcDBufs * 16 <= static_cast<int>(kTcTmemCols), "TMEM budget");

struct TcItem {
    int e, ntile, split, tt;
};

__device__ __forceinline__ TcItem tc_decode(int it, const int* start, const int* cnt, int n_exp,
                                            int splits) {
    int lo = 0, hi = n_exp - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (start[mid] <= it) lo = mid;
        else hi = mid - 1;
    }
    TcItem r;
    r.e = lo;
    const int local = it - start[lo];
    const int tte = (cnt[lo] + kTokTile - 1) / kTokTile;
    r.tt = local % tte;
    const int rest = local / tte;
    r.split = rest % splits;
    r.ntile = rest / splits;
    return r;
}

// Register R (0..15) of a unit goes to A column 32*(R/8) + 8*C + R%8: the
// first scale group's registers fill columns 0..31, the second's 32..63.
template <int C, int R>
__device__ __forceinline__ void tc_unit_reg(const uint32_t (&w)[3], const uint32_t (&hw)[3],
                                            uint32_t (&a)[64]) {
    constexpr int s = 4 * (R / 8) + (R % 8) / 2, hh = R % 2;
    a[32 * (R / 8) + 8 * C + (R % 8)] = unit_reg<sched_word(s, hh), sched_field(s, hh)>(w, hw);
}

template <int C>
__device__ __forceinline__ void tc_unit(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t (&a)[64]) {
    const uint32_t w[3] = {w0, w1, w2};
    const uint32_t hw[3] = {w0 >> 9, w1 >> 9, w2 >> 9};
    tc_unit_reg<C, 0>(w, hw, a);
    tc_unit_reg<C, 1>(w, hw, a);
    tc_unit_reg<C, 2>(w, hw, a);
    tc_unit_reg<C, 3>(w, hw, a);
    tc_unit_reg<C, 4>(w, hw, a);
    tc_unit_reg<C, 5>(w, hw, a);
    tc_unit_reg<C, 6>(w, hw, a);
    tc_unit_reg<C, 7>(w, hw, a);
    tc_unit_reg<C, 8>(w, hw, a);
    tc_unit_reg<C, 9>(w, hw, a);
    tc_unit_reg<C, 10>(w, hw, a);
    tc_unit_reg<C, 11>(w, hw, a);
    tc_unit_reg<C, 12>(w, hw, a);
    tc_unit_reg<C, 13>(w, hw, a);
    tc_unit_reg<C, 14>(w, hw, a);
    tc_unit_reg<C, 15>(w, hw, a);
}

// acc[tok] += s24 * D[tok] + nsz * xg[tok] for the first NT routed rows.
template <int NT>
__device__ __forceinline__ void tc_fold(float (&acc)[16], uint32_t d_addr, float s24, float nsz,
                                        const float* gs, int grp) {
    uint32_t d[NT];
    tc_ld<NT>(d_addr, d);
    tc_wait_ld();
#pragma unroll
    for (int i = 0; i < NT; ++i)
        acc[i] = fmaf(nsz, gs[i * 4 + grp], fmaf(s24, __uint_as_float(d[i]), acc[i]));
}

template <int NT>
__device__ __forceinline__ void tc_add(float (&acc)[16], uint32_t d_addr) {
    uint32_t d[NT];
    tc_ld<NT>(d_addr, d);
    tc_wait_ld();
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i] += __uint_as_float(d[i]);
}

// Bounded wait that all lanes of a warp leave together (tcgen05.ld/st that
// follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xFFFFFFFFu, ok);
}

struct TcRowState {
    int stage, ab, db;
    uint32_t phase, aph, dph, xph;
};

// Fold the two scale groups of super-block `sbl` of stage `st` into acc.
template <bool GLU>
__device__ __forceinline__ bool tc_fold_sb(TcRowState& rs, float (&acc)[16], const uint8_t* st, int sbl,
                                           int row, int lane, uint32_t lane_base, uint64_t* dfull,
                                           uint64_t* dempty, int ntcls) {
    const float* gs = reinterpret_cast<const float*>(st + kTcOffG);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (!warp_wait(&dfull[rs.db], rs.dph)) return false;
        tc_fence_after();
        const int grp = 2 * sbl + h;
        const __half* S;
        int idx;
        if (GLU) {
            S = reinterpret_cast<const __half*>(st + kTcOffS + (row >> 6) * 1024);
            idx = grp * 64 + (row & 63);
        } else {
            S = reinterpret_cast<const __half*>(st + kTcOffS);
            idx = grp * 128 + row;
        }
        const __half* Z = S + (GLU ? 256 : 512);
        const float sv = __half2float(S[idx]);
        const float zv = __half2float(Z[idx]);
        const float s24 = sv * 16777216.0f, nsz = -sv * zv;
        const uint32_t d_addr = lane_base + kTcDCol0 + 16 * rs.db;
        if (ntcls == 0) tc_fold<4>(acc, d_addr, s24, nsz, gs, grp);
        else if (ntcls == 1) tc_fold<8>(acc, d_addr, s24, nsz, gs, grp);
        else tc_fold<16>(acc, d_addr, s24, nsz, gs, grp);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dempty[rs.db]);
        if (++rs.db == kTcDBufs) { rs.db = 0; rs.dph ^= 1; }
    }
    return true;
}

template <bool GLU>
__global__ void __launch_bounds__(kTcThreads, 2) tc_gemm_kernel(const __grid_constant__ TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTcBar);
    uint64_t* empty = full + kTcStages;
    uint64_t* afull = empty + kTcStages;
    uint64_t* aempty = afull + kTcABufs;
    uint64_t* dfull = aempty + kTcABufs;
    uint64_t* dempty = dfull + kTcDBufs;
    uint64_t* done_bar = dempty + kTcDBufs;
    uint64_t* xfull = done_bar + 1;    // SwiGLU exchange: w3 rows -> w1 rows
    uint64_t* xempty = done_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 3);
    int* start = reinterpret_cast<int*>(smem + kTcTab);
    int* cnt = start + (MILO_MAX_EXPERTS + 1);
    int* row0s = cnt + (MILO_MAX_EXPERTS + 1);

    constexpr int RA = GLU ? kRowsGlu : kRowsPlain;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (p.N + RA - 1) / RA;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + 4);
        }
        for (int b = 0; b < kTcABufs; ++b) {
            mbar_init(&afull[b], 4);
            mbar_init(&aempty[b], 1);
        }
        for (int b = 0; b < kTcDBufs; ++b) {
            mbar_init(&dfull[b], 1);
            mbar_init(&dempty[b], 4);
        }
        mbar_init(done_bar, 1);
        mbar_init(xfull, 2);
        mbar_init(xempty, 2);
        fence_barrier_init();
        int run = 0;
        for (int e = 0; e < p.n_exp; ++e) {
            const int r0 = p.grp[2 * e], m = p.grp[2 * e + 1];
            const bool ok = m > 0 && r0 >= 0 && r0 + m <= p.R;
            start[e] = run;
            cnt[e] = ok ? m : 0;
            row0s[e] = r0;
            if (ok) run += ((m + kTokTile - 1) / kTokTile) * n_tiles * p.splits;
        }
        start[p.n_exp] = run;
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTcTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const int n_items = start[p.n_exp];
    const uint32_t idesc = f16_idesc(128, 16);

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t last_phase[kTcStages];
            bool used[kTcStages] = {false, false, false, false};
            bool fail = false;
            for (int it = blockIdx.x; it < n_items && !fail; it += gridDim.x) {
                const TcItem w = tc_decode(it, start, cnt, p.n_exp, p.splits);
                const ProjDev* pa = p.table + w.e * p.stride + p.proj_a;
                const ProjDev* pb = p.table + w.e * p.stride + p.proj_b;
                const int n0 = w.ntile * RA;
                const int row0 = row0s[w.e] + w.tt * kTokTile;
                const int c0 = w.split * p.cps, c1 = min(p.chunks, c0 + p.cps);
                tmap_acquire(&pa->q_map);
                tmap_acquire(&pa->s_map);
                tmap_acquire(&pa->z_map);
                if (GLU) {
                    tmap_acquire(&pb->q_map);
                    tmap_acquire(&pb->s_map);
                    tmap_acquire(&pb->z_map);
                }
                for (int ch = c0; ch < c1; ++ch) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { fail = true; break; }
                    uint8_t* st = smem + stage * kTcStageBytes;
                    uint64_t* fb = &full[stage];
                    mbar_arrive_expect_tx(fb, kTcStageTx);
#pragma unroll
                    for (int sbl = 0; sbl < 2; ++sbl) {
                        const int sb = 2 * ch + sbl;
                        tma_load_2d(st + kTcOffB + (2 * sbl) * 2048, &p.b_map, fb, 128 * sb, row0);
                        tma_load_2d(st + kTcOffB + (2 * sbl + 1) * 2048, &p.b_map, fb, 128 * sb + 64, row0);
                        if (GLU) {
                            tma_load_2d(st + kTcOffQ + sbl * 6144, &pa->q_map, fb, 12 * sb, n0);
                            tma_load_2d(st + kTcOffQ + sbl * 6144 + 3072, &pb->q_map, fb, 12 * sb, n0);
                        } else {
                            tma_load_2d(st + kTcOffQ + sbl * 6144, &pa->q_map, fb, 12 * sb, n0);
                        }
                    }
                    if (GLU) {
                        tma_load_2d(st + kTcOffS, &pa->s_map, fb, n0, 4 * ch);
                        tma_load_2d(st + kTcOffS + 512, &pa->z_map, fb, n0, 4 * ch);
                        tma_load_2d(st + kTcOffS + 1024, &pb->s_map, fb, n0, 4 * ch);
                        tma_load_2d(st + kTcOffS + 1536, &pb->z_map, fb, n0, 4 * ch);
                    } else {
                        tma_load_2d(st + kTcOffS, &pa->s_map, fb, n0, 4 * ch);
                        tma_load_2d(st + kTcOffS + 1024, &pa->z_map, fb, n0, 4 * ch);
                    }
                    tma_load_2d(st + kTcOffG, &p.g_map, fb, 4 * ch, row0);
                    used[stage] = true;
                    last_phase[stage] = phase;
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
                const int ra = pa->rank, rb = GLU ? pb->rank : 0;
                if (!fail && w.split == 0 && p.has_t && (ra > 0 || rb > 0)) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { fail = true; break; }
                    uint8_t* st = smem + stage * kTcStageBytes;
                    uint64_t* fb = &full[stage];
                    const int nbox = (p.tcols + 63) / 64;
                    const uint32_t bytes = nbox * 2048 + ra * RA * 2 + (GLU ? rb * RA * 2 : 0);
                    mbar_arrive_expect_tx(fb, bytes);
                    for (int j = 0; j < nbox; ++j)
                        tma_load_2d(st + kTcOffB + j * 2048, &p.t_map, fb, 64 * j, row0);
                    if (ra > 0) {
                        tmap_acquire(&pa->u_map);
                        tma_load_2d(st + kTcOffU, &pa->u_map, fb, 0, n0);
                    }
                    if (GLU && rb > 0) {
                        tmap_acquire(&pb->u_map);
                        tma_load_2d(st + kTcOffU + RA * MILO_MAX_RANK * 2, &pb->u_map, fb, 0, n0);
                    }
                    used[stage] = true;
                    last_phase[stage] = phase;
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
            }
            if (fail) flag(p.dev_status, MILO_DEV_TIMEOUT);
            // every issued copy has landed before the CTA can leave
            for (int s = 0; s < kTcStages; ++s)
                if (used[s] && !mbar_wait(&full[s], last_phase[s])) flag(p.dev_status, MILO_DEV_TIMEOUT);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0, ab = 0, db = 0;
            uint32_t phase = 0, aph = 0, dph = 0;
            bool fail = false;
            for (int it = blockIdx.x; it < n_items && !fail; it += gridDim.x) {
                const TcItem w = tc_decode(it, start, cnt, p.n_exp, p.splits);
                const ProjDev* pa = p.table + w.e * p.stride + p.proj_a;
                const ProjDev* pb = p.table + w.e * p.stride + p.proj_b;
                const int c0 = w.split * p.cps, c1 = min(p.chunks, c0 + p.cps);
                for (int ch = c0; ch < c1 && !fail; ++ch) {
                    if (!mbar_wait(&full[stage], phase)) { fail = true; break; }
                    const uint32_t sb_addr = smem_u32(smem + stage * kTcStageBytes) + kTcOffB;
                    for (int sbl = 0; sbl < 2 && !fail; ++sbl) {
                        if (!mbar_wait(&afull[ab], aph)) { fail = true; break; }
                        tc_fence_after();
                        for (int h = 0; h < 2; ++h) {
                            if (!mbar_wait(&dempty[db], dph ^ 1)) { fail = true; break; }
                            tc_fence_after();
                            const uint32_t d_addr = tbase + kTcDCol0 + 16 * db;
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                tc_mma_ts(d_addr, tbase + 64 * ab + 32 * h + 8 * q,
                                          sw128_kmajor_desc(sb_addr + (2 * sbl + h) * 2048 + 32 * q), idesc,
                                          q > 0 ? 1u : 0u);
                            tc_commit(&dfull[db]);
                            if (++db == kTcDBufs) { db = 0; dph ^= 1; }
                        }
                        tc_commit(&aempty[ab]);
                        if (++ab == kTcABufs) { ab = 0; aph ^= 1; }
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
                const int ra = pa->rank, rb = GLU ? pb->rank : 0;
                if (!fail && w.split == 0 && p.has_t && (ra > 0 || rb > 0)) {
                    if (!mbar_wait(&full[stage], phase) || !mbar_wait(&afull[ab], aph) ||
                        !mbar_wait(&dempty[db], dph ^ 1)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t t_addr = smem_u32(smem + stage * kTcStageBytes) + kTcOffB;
                    const uint32_t d_addr = tbase + kTcDCol0 + 16 * db;
                    const int steps = (p.tcols + 15) / 16;
                    for (int q = 0; q < steps; ++q)
                        tc_mma_ts(d_addr, tbase + 64 * ab + 8 * q,
                                  sw128_kmajor_desc(t_addr + (q / 4) * 2048 + (q % 4) * 32), idesc,
                                  q > 0 ? 1u : 0u);
                    tc_commit(&dfull[db]);
                    if (++db == kTcDBufs) { db = 0; dph ^= 1; }
                    tc_commit(&aempty[ab]);
                    if (++ab == kTcABufs) { ab = 0; aph ^= 1; }
                    tc_commit(&empty[stage]);
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
            }
            if (fail) flag(p.dev_status, MILO_DEV_TIMEOUT);
            // every issued MMA has completed before TMEM is released
            tc_commit(done_bar);
            if (!mbar_wait(done_bar, 0)) flag(p.dev_status, MILO_DEV_TIMEOUT);
        }
    } else {
        // ---------------------------------------------------------------- rows
        const int quarter = warp & 3;
        const int row = 32 * quarter + lane;
        const uint32_t lane_base = tbase + (static_cast<uint32_t>(32 * quarter) << 16);
        float* xch = reinterpret_cast<float*>(smem + kTcXch);
        TcRowState rs{0, 0, 0, 0u, 0u, 0u, 0u};
        int32_t st_bits = 0;
        bool fail = false;
        for (int it = blockIdx.x; it < n_items && !fail; it += gridDim.x) {
            const TcItem w = tc_decode(it, start, cnt, p.n_exp, p.splits);
            const ProjDev* pa = p.table + w.e * p.stride + p.proj_a;
            const ProjDev* pb = p.table + w.e * p.stride + p.proj_b;
            const int n0 = w.ntile * RA;
            const int row0 = row0s[w.e] + w.tt * kTokTile;
            const int ntok = min(kTokTile, cnt[w.e] - w.tt * kTokTile);
            const int ntcls = ntok <= 4 ? 0 : (ntok <= 8 ? 1 : 2);
            const int c0 = w.split * p.cps, c1 = min(p.chunks, c0 + p.cps);
            float acc[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
            const uint8_t* prev_st = nullptr;
            int prev_stage = 0, prev_sbl = 0;
            for (int ch = c0; ch < c1 && !fail; ++ch) {
                if (!warp_wait(&full[rs.stage], rs.phase)) { fail = true; break; }
                const uint8_t* st = smem + rs.stage * kTcStageBytes;
                for (int sbl = 0; sbl < 2; ++sbl) {
                    const uint4* qv = reinterpret_cast<const uint4*>(st + kTcOffQ + (sbl * 128 + row) * 48);
                    const uint4 v0 = qv[0], v1 = qv[1], v2 = qv[2];
                    uint32_t a[64];
                    tc_unit<0>(v0.x, v0.y, v0.z, a);
                    tc_unit<1>(v0.w, v1.x, v1.y, a);
                    tc_unit<2>(v1.z, v1.w, v2.x, a);
                    tc_unit<3>(v2.y, v2.z, v2.w, a);
                    if (!warp_wait(&aempty[rs.ab], rs.aph ^ 1)) { fail = true; break; }
                    tc_fence_after();
                    tc_st64(lane_base + 64 * rs.ab, a);
                    tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&afull[rs.ab]);
                    if (++rs.ab == kTcABufs) { rs.ab = 0; rs.aph ^= 1; }
                    if (prev_st) {
                        if (!tc_fold_sb<GLU>(rs, acc, prev_st, prev_sbl, row, lane, lane_base, dfull, dempty,
                                             ntcls)) { fail = true; break; }
                        if (prev_sbl == 1) {
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&empty[prev_stage]);
                        }
                    }
                    prev_st = st;
                    prev_stage = rs.stage;
                    prev_sbl = sbl;
                }
                if (++rs.stage == kTcStages) { rs.stage = 0; rs.phase ^= 1; }
            }
            if (fail) break;
            if (prev_st) {
                if (!tc_fold_sb<GLU>(rs, acc, prev_st, prev_sbl, row, lane, lane_base, dfull, dempty, ntcls)) {
                    fail = true;
                    break;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[prev_stage]);
            }
            const int ra = pa->rank, rb = GLU ? pb->rank : 0;
            if (w.split == 0 && p.has_t && (ra > 0 || rb > 0)) {
                if (!warp_wait(&full[rs.stage], rs.phase)) { fail = true; break; }
                const uint8_t* st = smem + rs.stage * kTcStageBytes;
                // A row of the compensator step: this row's U values at the K slots
                // of its projection's t columns, zeros elsewhere.
                const uint16_t* src;
                int lo, r;
                if (GLU && row >= 64) {
                    src = reinterpret_cast<const uint16_t*>(st + kTcOffU + RA * MILO_MAX_RANK * 2) + (row - 64) * rb;
                    lo = p.t_col_b;
                    r = rb;
                } else {
                    src = reinterpret_cast<const uint16_t*>(st + kTcOffU) + row * ra;
                    lo = 0;
                    r = ra;
                }
                uint32_t a[64];
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const int slot = 2 * j;
                    a[j] = (slot >= lo && slot < lo + r) ? *reinterpret_cast<const uint32_t*>(src + (slot - lo)) : 0u;
                }
                if (!warp_wait(&aempty[rs.ab], rs.aph ^ 1)) { fail = true; break; }
                tc_fence_after();
                tc_st64(lane_base + 64 * rs.ab, a);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&afull[rs.ab]);
                    mbar_arrive(&empty[rs.stage]);
                }
                if (++rs.ab == kTcABufs) { rs.ab = 0; rs.aph ^= 1; }
                if (++rs.stage == kTcStages) { rs.stage = 0; rs.phase ^= 1; }
                if (!warp_wait(&dfull[rs.db], rs.dph)) { fail = true; break; }
                tc_fence_after();
                const uint32_t d_addr = lane_base + kTcDCol0 + 16 * rs.db;
                if (ntcls == 0) tc_add<4>(acc, d_addr);
                else if (ntcls == 1) tc_add<8>(acc, d_addr);
                else tc_add<16>(acc, d_addr);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dempty[rs.db]);
                if (++rs.db == kTcDBufs) { rs.db = 0; rs.dph ^= 1; }
            }

            // ------------------------------------------------------------ epilogue
            if constexpr (GLU) {
                // rows 64..127 (w3) hand b to rows 0..63 (w1) through shared memory
                if (row >= 64) {
                    if (!warp_wait(xempty, rs.xph ^ 1)) { fail = true; break; }
#pragma unroll
                    for (int i = 0; i < 16; ++i) xch[(row - 64) * 17 + i] = acc[i];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(xfull);
                } else {
                    if (!warp_wait(xfull, rs.xph)) { fail = true; break; }
                    const int f = n0 + row;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float bv = xch[row * 17 + i];
                        if (i < ntok && f < p.N) {
                            const float av = acc[i];
                            const float hv = av / (1.0f + expf(-av)) * bv;
                            const __half hh = __float2half_rn(hv);
                            if (!isfinite(hv)) st_bits |= MILO_DEV_NONFINITE;
                            else if (__hisinf(hh)) st_bits |= MILO_DEV_FP16_RANGE;
                            p.h[static_cast<size_t>(row0 + i) * p.N + f] = __half_as_ushort(hh);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(xempty);
                }
                rs.xph ^= 1;
            } else {
                float* out = p.y_part + static_cast<size_t>(w.split) * p.R * p.N;
                const int n = n0 + row;
                if (n < p.N) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (i < ntok) out[static_cast<size_t>(row0 + i) * p.N + n] = acc[i];
                }
            }
        }
        if (fail) st_bits |= MILO_DEV_TIMEOUT;
        flag(p.dev_status, st_bits);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTcTmemCols);
    }
}

size_t tc_smem_bytes() { return kTcSmemBytes; }

cudaError_t launch_tc_gemm(const TcParams& p, bool glu, int grid, cudaStream_t s) {
    static bool configured[64][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !configured[dev][glu]) {
        e = glu ? cudaFuncSetAttribute(tc_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes)
                : cudaFuncSetAttribute(tc_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev][glu] = true;
    }
    if (glu) tc_gemm_kernel<true><<<grid, kTcThreads, kTcSmemBytes, s>>>(p);
    else tc_gemm_kernel<false><<<grid, kTcThreads, kTcSmemBytes, s>>>(p);
    return cudaGetLastError();
}

}  // namespace milo
