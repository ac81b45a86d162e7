// gemm_tc.cu -- grouped int3 x fp16 GEMM with the low-rank compensator on the
// 5th-generation tensor cores (tcgen05, TMEM), for experts with many routed
// rows (prefill, large batches) (sm_100a).
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators": W_out = W_quant + U V ("MiLo Algorithm"), an int3 x FP16 GEMM
// with dequantisation and the asymmetric zero point fused in ("MiLo Kernel").
//
// Design (B200):
//   - A work item is (expert, 128 weight rows, kTcTok routed rows); a stage is
//     one 128-code super-block.  The producer warp brings the activations
//     (2-D TMA, 128-byte swizzle: the K-major B operand), the two 64-row
//     blob blocks (1-D bulk copies: codes, scales, zeros) and, on the second
//     stage of each super-block pair, the pair's group-sum tile.
//   - Four extraction warps (one thread per weight row) turn the row's 32
//     code pairs into exact fp16 patterns code * 2^e * 2^-24 (one LOP3 per
//     pair; the activations carry 2^(6 - e) and their row's scale 2^a) and
//     store them to TMEM: the A operand.  They also write -s_g * z_g of the
//     row's groups, times a power of two of the row (zp_scale) and split into
//     fp16 hi + lo, to shared memory (32-byte swizzle).
//   - The MMA warp issues tcgen05.mma M=128, N=kTcTok, K=16 (one elected lane)
//     with A from TMEM and B from shared memory, per 64-code scale group into
//     its own TMEM accumulator D_g (several in flight), and once per pair a
//     zero-point step Z += (-s z)_hi,lo x (X_g)_hi,lo over the pair's four
//     groups (four K slots each: the four hi/lo cross products).
//   - Eight fold warps (two per weight row: kTcTok / 2 routed rows and fp32
//     accumulators each) read D_g and fold acc += s * 2^18 * D_g (packed
//     FFMA2), then add Z once per item and multiply each routed row by its
//     2^-a, so the scale and the zero point cost no per-weight work; -s z
//     splits exactly, X_g to 2^-22 relative, and the rest is fp32
//     accumulation.
//   - The compensator is one more stage: A = U rows, B = t = x V^T.
//   - Epilogue: SwiGLU through a shared-memory exchange between the w1 and w3
//     rows of each output feature (each side finishes half the tokens), or
//     the fp32 output rows.
//   - Every wait is bounded; on a timeout the kernel flags MILO_DEV_TIMEOUT,
//     drains its copies and MMAs and frees TMEM before leaving.
#include <cuda_runtime.h>

#include <atomic>

#include "milo_device.cuh"
#include "milo_host.h"
#include "milo_kernels.h"
#include "milo_tc.cuh"

namespace milo {

constexpr int kTcTok = kTcTokens;           // routed rows per item (MMA N)
constexpr int kTcHalf = kTcTok / 2;         // routed rows per fold warp
constexpr int kTcRows = 128;                // weight rows per item (MMA M)
constexpr int kTcAlign(int b) { return (b + 1023) / 1024 * 1024; }
constexpr int kTcOffB = 0;                  // activations: 2 swizzled atoms [kTcTok rows][128 B]
constexpr int kTcAtom = kTcTok * 128;
constexpr int kTcOffW = 2 * kTcAtom;        // two blob blocks (rows 0-63, 64-127)
// zero-point step, once per pair of super-blocks (four groups, four K slots
// each): B = group sums X_g as fp16 hi, lo [kTcTok routed rows][32 B], A =
// -s*z as fp16 hi, lo [128 weight rows][32 B], both with the 32-byte swizzle
constexpr int kTcOffZB = kTcAlign(kTcOffW + 2 * kBlockSB);
constexpr int kTcZTile = kTcTok * 32;
constexpr int kTcOffZA = kTcAlign(kTcOffZB + kTcZTile);
constexpr int kTcZATile = kTcRows * 32;
constexpr int kTcStageTx = 2 * kTcAtom;     // plus the blob blocks (and the B_z tile)
constexpr int kTcOffUA = kTcOffW;           // compensator stage: U rows of w1 (or 128 rows)
constexpr int kTcOffUB = kTcOffW + 64 * MILO_MAX_RANK * 2;   // U rows of w3
constexpr int kTcMax(int a, int b) { return a > b ? a : b; }
constexpr int kTcStage = kTcAlign(kTcMax(kTcOffZA + kTcZATile, kTcOffUA + kTcRows * MILO_MAX_RANK * 2));   // bytes per stage
constexpr int kTcStages = kTcTok == 128 ? 3 : 4;
constexpr int kTcXch = kTcStages * kTcStage;             // SwiGLU exchange, per token half: [48 tokens][64 rows] f32
constexpr int kTcXchHalf = kTcHalf * 64;                  // floats per half
constexpr int kTcBar = kTcXch + 2 * kTcXchHalf * 4;
constexpr int kTcDBufs = (512 - 128 - kTcTok) / kTcTok;   // TMEM accumulators D_g in flight between MMA and fold
constexpr int kTcNumBars = 2 * kTcStages + 2 * 2 + 2 * kTcDBufs + 1 + 4 + 1;   // + done, xfull[2], xempty[2], zempty
constexpr int kTcTab = kTcBar + 8 * kTcNumBars + 16;
constexpr int kTcSmemUsed = kTcTab + 3 * (MILO_MAX_EXPERTS + 1) * 4;
constexpr int kTcSmemBytes = kTcSmemUsed + 1024;        // slack to align the base to 1024 B
constexpr int kTcFoldWarps = 8;             // two per TMEM lane quarter, kTcHalf routed rows each
constexpr int kTcThreads = 32 * (2 + 4 + kTcFoldWarps);   // producer, MMA, extraction, fold
constexpr uint32_t kTcTmemCols = 512;       // A: 2 x 64 columns, D_g: kTcDBufs x kTcTok, Z: kTcTok
constexpr int kTcACol = 0, kTcDCol = 128, kTcZCol = kTcDCol + kTcDBufs * kTcTok;

static_assert(kTcOffW + 2 * kBlockSB <= kTcOffZB && kTcOffZB + kTcZTile <= kTcOffZA, "stage layout");
static_assert(kTcOffZA + kTcZATile <= kTcStage && kTcOffZB % 1024 == 0 && kTcOffZA % 1024 == 0, "stage layout");
static_assert(kTcAtom % 1024 == 0 && kTcTok % 32 == 0 && kTcHalf % 16 == 0, "tile shapes");
static_assert(kTcDCol % 32 == 0 && kTcTok % 32 == 0 && kTcZCol % 32 == 0, "accumulator columns");
static_assert(kTcOffUB + 64 * MILO_MAX_RANK * 2 <= kTcStage, "compensator stage: U rows");
static_assert(kTcOffUA + kTcRows * MILO_MAX_RANK * 2 <= kTcStage, "compensator stage: plain U rows");
static_assert(kTcSmemBytes <= 227 * 1024, "shared memory");
static_assert(kTcZCol + kTcTok <= static_cast<int>(kTcTmemCols), "TMEM columns");

struct TcItem {
    int e, ntile, tt;
};

__device__ __forceinline__ TcItem tc_decode(int it, const int* start, const int* cnt, int n_exp, int n_tiles,
                                           int ntile_fast) {
    int lo = 0, hi = n_exp - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (start[mid] <= it) lo = mid;
        else hi = mid - 1;
    }
    TcItem r;
    r.e = lo;
    const int local = it - start[lo];
    const int tte = (cnt[lo] + kTcTok - 1) / kTcTok;
    if (ntile_fast) {
        r.ntile = local % n_tiles;
        r.tt = local / n_tiles;
    } else {
        r.tt = local % tte;
        r.ntile = local / tte;
    }
    return r;
}

// Register R (0..15) of unit C goes to A column 32 * (R / 8) + 8 * C + R % 8:
// the first scale group's registers fill columns 0..31, the second's 32..63
// (R = 2 * step + half of the eight-step register schedule).
template <int C, int R>
__device__ __forceinline__ void tc_unit_reg(const uint32_t (&w)[3], const uint32_t (&hw)[3], uint32_t (&a)[64]) {
    constexpr int s = R / 2, hh = R % 2;
    a[32 * (R / 8) + 8 * C + (R % 8)] = unit_reg<sched_word(s, hh), sched_field(s, hh)>(w, hw);
}

template <int C>
__device__ __forceinline__ void tc_unit(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t (&a)[64]) {
    const uint32_t w[3] = {w0, w1, w2};
    const uint32_t hw[3] = {w0 >> word_shift(0), w1 >> word_shift(1), w2 >> word_shift(2)};
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

// fp16 pair (U[n][rho], U[n][rho + 1]) from an int3 U^T block (128 features):
// feature nl's codes of rank rows rho and rho + 1, (q - z) * s.
__device__ __forceinline__ uint32_t lorc3_value_pair(const uint8_t* blk, int rho, int nl) {
    float v[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(blk + lorc_words_off(rho + q, 0, blob_unit(nl)));
        const uint32_t w3[3] = {wp[0], wp[1], wp[2]};
        const uint32_t sz = *reinterpret_cast<const uint32_t*>(blk + lorc_sz_off(rho + q, nl >> 6));
        v[q] = (static_cast<float>(unit_code(w3, blob_code(nl))) - sz_zero(sz)) * sz_scale(sz);
    }
    return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[0]))) |
           (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[1]))) << 16);
}

// Power of two 2^c that brings a weight row's first group scale s into
// [2^-3, 2^-2).  The zero-point operand -s z 2^c of each of the row's groups
// (|s z| <= 7 s for codes 0..7) then splits into normal fp16 hi + lo however
// small the weights are; the fold multiplies the row's Z by 2^-c.  Extraction
// and fold warps derive it from the same s; 1 for a zero row.
__device__ __forceinline__ float zp_scale(float s) {
    const uint32_t b = __float_as_uint(s);
    if (!(s > 0.0f) || b >= 0x7F800000u) return 1.0f;
    return __uint_as_float(static_cast<uint32_t>(127 + 124 - static_cast<int>(b >> 23)) << 23);
}

// A fold warp reads its kTcHalf accumulator columns in chunks of kTcChunk
// (48: three x16 loads in flight; 32: one x32 load), the caller waiting with
// tc_wait_ld.
constexpr int kTcChunk = kTcHalf % 32 == 0 ? 32 : 48;
constexpr int kTcChunks = kTcHalf / kTcChunk;
static_assert(kTcHalf % kTcChunk == 0, "fold chunks");

template <int C>
__device__ __forceinline__ void tc_ld_chunk(uint32_t taddr, uint32_t (&d)[C]) {
    if constexpr (C == 32) {
        tc_ld<32>(taddr, d);
    } else {
        tc_ld<16>(taddr, reinterpret_cast<uint32_t(&)[16]>(d[0]));
        tc_ld<16>(taddr + 16, reinterpret_cast<uint32_t(&)[16]>(d[16]));
        tc_ld<16>(taddr + 32, reinterpret_cast<uint32_t(&)[16]>(d[32]));
    }
}

template <bool GLU>
__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm_kernel(const __grid_constant__ TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTcBar);
    uint64_t* empty = full + kTcStages;
    uint64_t* afull = empty + kTcStages;
    uint64_t* aempty = afull + 2;
    uint64_t* dfull = aempty + 2;
    uint64_t* dempty = dfull + kTcDBufs;
    uint64_t* done_bar = dempty + kTcDBufs;
    uint64_t* xfull = done_bar + 1;      // [2] SwiGLU exchange, per token half: w3 rows -> w1 rows
    uint64_t* xempty = xfull + 2;        // [2]
    uint64_t* zempty = xempty + 2;       // the fold warps have read the item's Z accumulator
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(zempty + 1);
    int* start = reinterpret_cast<int*>(smem + kTcTab);
    int* cnt = start + (MILO_MAX_EXPERTS + 1);
    int* row0s = cnt + (MILO_MAX_EXPERTS + 1);
    float* xch = reinterpret_cast<float*>(smem + kTcXch);

    constexpr int RA = GLU ? kRowsGlu : kRowsPlain;   // output features per item
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (p.N + RA - 1) / RA;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + 4 + kTcFoldWarps);   // MMA commit, extraction warps, fold warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&afull[b], 4);
            mbar_init(&aempty[b], 1);
        }
        for (int b = 0; b < kTcDBufs; ++b) {
            mbar_init(&dfull[b], 1);
            mbar_init(&dempty[b], kTcFoldWarps);
        }
        mbar_init(done_bar, 1);
        mbar_init(zempty, kTcFoldWarps);
        for (int rd = 0; rd < 2; ++rd) {
            mbar_init(&xfull[rd], 4);    // the four fold warps of the token half
            mbar_init(&xempty[rd], 4);
        }
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTcTmemCols);
    grid_dep_wait();
    // item table: all threads load the expert groups, warp 0 scans the item counts
    for (int e = threadIdx.x; e < p.n_exp; e += blockDim.x) {
        const int r0 = p.grp[2 * e], m = p.grp[2 * e + 1];
        const bool ok = m > 0 && r0 >= 0 && r0 + m <= p.R;
        cnt[e] = ok ? m : 0;
        row0s[e] = r0;
    }
    __syncthreads();
    if (warp == 0) {
        int run = 0;
        for (int base = 0; base < p.n_exp; base += 32) {
            const int e = base + lane;
            const int m = e < p.n_exp ? cnt[e] : 0;
            const int items = m > 0 ? ((m + kTcTok - 1) / kTcTok) * n_tiles : 0;
            int incl = items;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            if (e < p.n_exp) start[e] = run + incl - items;
            run += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) start[p.n_exp] = run;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const int n_items = start[p.n_exp];

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // the whole warp runs the loop; one elected lane issues the copies
        {
            // weights keep the default L2 policy here: every weight tile serves
            // all of its expert's routed-row tiles (an evict-first hint, right
            // for the decode GEMM that reads each tile once, made them re-read)
            int stage = 0;
            uint32_t phase = 0, filled = 0, fph = 0;
            bool fail = false;
            for (int it = blockIdx.x; it < n_items && !fail; it += gridDim.x) {
                const TcItem w = tc_decode(it, start, cnt, p.n_exp, n_tiles, p.ntile_fast);
                const ProjDev* pa = p.table + w.e * p.stride + p.proj_a;
                const ProjDev* pb = p.table + w.e * p.stride + p.proj_b;
                const int n0 = w.ntile * RA;
                const int tile0 = n0 / kTileRows;
                const int ntl = GLU ? 2 : min(2, (p.N - n0 + kTileRows - 1) / kTileRows);
                const int row0 = row0s[w.e] + w.tt * kTcTok;
                for (int b = 0; b < p.SB; ++b) {
                    if (!warp_wait(&empty[stage], phase ^ 1)) {
                        fail = true;
                        break;
                    }
                    uint8_t* st = smem + stage * kTcStage;
                    uint64_t* fb = &full[stage];
                    filled |= 1u << stage;
                    fph = (fph & ~(1u << stage)) | (phase << stage);
                    const bool zs = (b & 1) || b == p.SB - 1;    // last stage of a super-block pair
                    const uint8_t* w0 = pa->packed + (static_cast<size_t>(tile0) * p.SB + b) * kBlockSB;
                    const uint8_t* w1 = GLU ? pb->packed + (static_cast<size_t>(tile0) * p.SB + b) * kBlockSB
                                            : w0 + static_cast<size_t>(p.SB) * kBlockSB;
                    if (elect_one()) {
                        // each blob's ceil(N / 64) tiles of SB blocks (SwiGLU: tile
                        // tile0 of w1's and of w3's), the routed rows
                        if (in_range(p.dev_status, tile0 + (GLU ? 1 : ntl) <= (p.N + kTileRows - 1) / kTileRows &&
                                                       row0 >= 0 &&
                                                       row0 < p.R)) {
                            mbar_arrive_expect_tx(fb, kTcStageTx + ntl * kBlockSB + (zs ? kTcZTile : 0));
                            tma_load_2d(st + kTcOffB, &p.b_map, fb, 128 * b, row0);
                            tma_load_2d(st + kTcOffB + kTcAtom, &p.b_map, fb, 128 * b + 64, row0);
                            bulk_load(st + kTcOffW, w0, kBlockSB, fb);
                            if (ntl == 2) bulk_load(st + kTcOffW + kBlockSB, w1, kBlockSB, fb);
                            if (zs) tma_load_2d(st + kTcOffZB, &p.z_map, fb, 16 * (b >> 1), row0);
                        } else {
                            mbar_arrive(fb);
                        }
                    }
                    __syncwarp();
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
                if (fail) break;
                const int ra = pa->rank, rb = GLU ? pb->rank : 0;
                if (p.has_t && (ra > 0 || rb > 0)) {
                    if (!warp_wait(&empty[stage], phase ^ 1)) {
                        fail = true;
                        break;
                    }
                    uint8_t* st = smem + stage * kTcStage;
                    uint64_t* fb = &full[stage];
                    filled |= 1u << stage;
                    fph = (fph & ~(1u << stage)) | (phase << stage);
                    const int nbox = (p.tcols + 63) / 64;
                    const int urows = min(RA, p.N - n0);
                    // fp16 U rows, or the int3 U^T block holding the item's features
                    const uint32_t ua = ra == 0 ? 0u : pa->lorc3 ? kBlockSB : urows * ra * 2;
                    const uint32_t ub = rb == 0 ? 0u : pb->lorc3 ? kBlockSB : urows * rb * 2;
                    const uint8_t* usa = pa->lorc3 ? reinterpret_cast<const uint8_t*>(pa->U) + (n0 >> 7) * kBlockSB
                                                   : reinterpret_cast<const uint8_t*>(pa->U + static_cast<size_t>(n0) * ra);
                    const uint8_t* usb = !GLU ? usa
                                         : pb->lorc3 ? reinterpret_cast<const uint8_t*>(pb->U) + (n0 >> 7) * kBlockSB
                                                     : reinterpret_cast<const uint8_t*>(pb->U + static_cast<size_t>(n0) * rb);
                    if (elect_one()) {
                        // U rows n0 .. n0 + urows or the int3 U^T block of
                        // super-block n0 / 128, and the stage's room for them
                        if (in_range(p.dev_status, n0 + urows <= p.N && nbox <= 2 && row0 >= 0 && row0 < p.R &&
                                                       ua <= (GLU ? kTcOffUB : kTcStage) - kTcOffUA && kTcOffUB + ub <= kTcStage &&
                                                       (!(ra && pa->lorc3) || (n0 >> 7) < p.N / 128) &&
                                                       (!(rb && pb->lorc3) || (n0 >> 7) < p.N / 128))) {
                            mbar_arrive_expect_tx(fb, nbox * kTcAtom + ua + ub);
                            for (int j = 0; j < nbox; ++j)
                                tma_load_2d(st + kTcOffB + j * kTcAtom, &p.t_map, fb, 64 * j, row0);
                            if (ua) bulk_load(st + kTcOffUA, usa, ua, fb);
                            if (ub) bulk_load(st + kTcOffUB, usb, ub, fb);
                        } else {
                            mbar_arrive(fb);
                        }
                    }
                    __syncwarp();
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
            }
            // no copy may still be landing in shared memory when the CTA leaves
            for (int s2 = 0; s2 < kTcStages; ++s2)
                if (((filled >> s2) & 1u) && !warp_wait(&full[s2], (fph >> s2) & 1u)) fail = true;
            if (fail && lane == 0) flag(p.dev_status, MILO_DEV_TIMEOUT);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // the whole warp runs the loop (uniform operands); one lane issues
        {
            const uint32_t idesc = f16_idesc(kTcRows, kTcTok);
            int stage = 0, ab = 0, db = 0;
            uint32_t phase = 0, aph = 0, dph = 0, zph = 0;
            bool fail = false;
            for (int it = blockIdx.x; it < n_items && !fail; it += gridDim.x) {
                const TcItem w = tc_decode(it, start, cnt, p.n_exp, n_tiles, p.ntile_fast);
                const ProjDev* pa = p.table + w.e * p.stride + p.proj_a;
                const ProjDev* pb = p.table + w.e * p.stride + p.proj_b;
                for (int b = 0; b < p.SB && !fail; ++b) {
                    if (!warp_wait(&full[stage], phase) || !warp_wait(&afull[ab], aph)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sb_addr = smem_u32(smem + stage * kTcStage) + kTcOffB;
                    const bool zs = (b & 1) || b == p.SB - 1;
                    for (int h = 0; h < 2; ++h) {
                        if (!warp_wait(&dempty[db], dph ^ 1)) {
                            fail = true;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d_addr = tbase + kTcDCol + kTcTok * db;
                        tc_mma_ts4(d_addr, tbase + kTcACol + 64 * ab + 32 * h,
                                   sw128_kmajor_desc(sb_addr + h * kTcAtom), idesc, 0u);
                        if (h == 1 && zs) {
                            // zero-point step of the pair into Z; the first one of an
                            // item waits until the fold has read the previous item's Z.
                            // Committed with this group's D_g, so a fold warp that saw
                            // the item's last D_g may read Z.
                            if (b < 2) {
                                if (!warp_wait(zempty, zph ^ 1)) {
                                    fail = true;
                                    break;
                                }
                                zph ^= 1;
                                tc_fence_after();
                            }
                            tc_mma_ss(tbase + kTcZCol, sw32_kmajor_desc(sb_addr - kTcOffB + kTcOffZA),
                                      sw32_kmajor_desc(sb_addr - kTcOffB + kTcOffZB), idesc, b >= 2 ? 1u : 0u);
                        }
                        tc_commit(&dfull[db]);
                        if (++db == kTcDBufs) { db = 0; dph ^= 1; }
                    }
                    if (fail) break;
                    tc_commit(&aempty[ab]);
                    if (++ab == 2) { ab = 0; aph ^= 1; }
                    tc_commit(&empty[stage]);
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
                if (fail) break;
                const int ra = pa->rank, rb = GLU ? pb->rank : 0;
                if (p.has_t && (ra > 0 || rb > 0)) {
                    if (!warp_wait(&full[stage], phase) || !warp_wait(&afull[ab], aph) ||
                        !warp_wait(&dempty[db], dph ^ 1)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t t_addr = smem_u32(smem + stage * kTcStage) + kTcOffB;
                    const uint32_t d_addr = tbase + kTcDCol + kTcTok * db;
                    const int steps = (p.tcols + 15) / 16;
                    for (int q = 0; q < steps; ++q)
                        tc_mma_ts(d_addr, tbase + kTcACol + 64 * ab + 8 * q,
                                  sw128_kmajor_desc(t_addr + (q / 4) * kTcAtom + (q % 4) * 32), idesc,
                                  q > 0 ? 1u : 0u);
                    tc_commit(&dfull[db]);
                    if (++db == kTcDBufs) { db = 0; dph ^= 1; }
                    tc_commit(&aempty[ab]);
                    if (++ab == 2) { ab = 0; aph ^= 1; }
                    tc_commit(&empty[stage]);
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
            }
            if (fail && lane == 0) flag(p.dev_status, MILO_DEV_TIMEOUT);
            // every issued MMA has completed before TMEM is released
            tc_commit(done_bar);
            if (!warp_wait(done_bar, 0) && lane == 0) flag(p.dev_status, MILO_DEV_TIMEOUT);
        }
    } else if (warp < 6) {
        // ---------------------------------------------------------------- extraction (A operand)
        const int quarter = warp & 3;
        const int row = 32 * quarter + lane;               // TMEM lane = weight row of the item
        const uint32_t lane_base = tbase + (static_cast<uint32_t>(32 * quarter) << 16);
        const int half = row >> 6, r64 = row & 63;
        // byte offset of this row's (s, z) pair inside a group's 256 bytes
        const int pair_off = (((r64 >> 4) * 8 + (r64 & 7)) * 4 + ((r64 >> 3) & 1) * 2) * 2;
        int stage = 0, ab = 0;
        uint32_t phase = 0, aph = 0;
        bool fail = false;
        int32_t st_bits = 0;
        uint4 zprev = make_uint4(0u, 0u, 0u, 0u);   // A_z slots of the pair's first super-block
        float zsc = 1.0f;                           // the item's zero-point scale 2^c of this row
        for (int it = blockIdx.x; it < n_items && !fail; it += gridDim.x) {
            const TcItem w = tc_decode(it, start, cnt, p.n_exp, n_tiles, p.ntile_fast);
            const ProjDev* pa = p.table + w.e * p.stride + p.proj_a;
            const ProjDev* pb = p.table + w.e * p.stride + p.proj_b;
            // a plain item's second 64-row block is not loaded when the tile
            // ends first: those rows compute garbage that is never stored
            const bool live = GLU || w.ntile * RA + 64 * half < p.N;
            for (int b = 0; b < p.SB; ++b) {
                if (!warp_wait(&full[stage], phase)) {
                    fail = true;
                    break;
                }
                const uint8_t* st = smem + stage * kTcStage;
                const uint4* qv = reinterpret_cast<const uint4*>(st + kTcOffW + half * kBlockSB + r64 * 48);
                const uint4 v0 = qv[0], v1 = qv[1], v2 = qv[2];
                uint32_t a[64];
                tc_unit<0>(v0.x, v0.y, v0.z, a);
                tc_unit<1>(v0.w, v1.x, v1.y, a);
                tc_unit<2>(v1.z, v1.w, v2.x, a);
                tc_unit<3>(v2.y, v2.z, v2.w, a);
                // -s*z of the two groups, split exactly into fp16 hi + lo, in the
                // K slots (hi, hi, lo, lo) that meet (X hi, X lo, X hi, X lo)
                uint32_t zw[4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t szv = *reinterpret_cast<const uint32_t*>(
                        st + kTcOffW + half * kBlockSB + kQTileSBWords * 4 + h * kGroupBytes + pair_off);
                    const float sv = __half2float(__ushort_as_half(static_cast<uint16_t>(szv & 0xFFFFu)));
                    if (b == 0 && h == 0) zsc = zp_scale(sv);
                    const float c = live ? -(sv * __half2float(__ushort_as_half(static_cast<uint16_t>(szv >> 16)))) * zsc
                                         : 0.0f;
                    const __half hi = __float2half_rn(c);
                    const __half lo = __float2half_rn(c - __half2float(hi));
                    if (__hisinf(hi)) st_bits |= MILO_DEV_FP16_RANGE;
                    zw[2 * h] = static_cast<uint32_t>(__half_as_ushort(hi)) * 0x10001u;
                    zw[2 * h + 1] = static_cast<uint32_t>(__half_as_ushort(lo)) * 0x10001u;
                }
                const bool zs = (b & 1) || b == p.SB - 1;
                if (zs) {
                    uint8_t* za = smem + stage * kTcStage + kTcOffZA;
                    const uint4 cur = make_uint4(zw[0], zw[1], zw[2], zw[3]);
                    const bool second = b & 1;
                    *reinterpret_cast<uint4*>(za + sw32_offset(row, 0)) = second ? zprev : cur;
                    *reinterpret_cast<uint4*>(za + sw32_offset(row, 1)) = second ? cur : make_uint4(0u, 0u, 0u, 0u);
                    fence_proxy_async_smem();
                } else {
                    zprev = make_uint4(zw[0], zw[1], zw[2], zw[3]);
                }
                if (!warp_wait(&aempty[ab], aph ^ 1)) {
                    fail = true;
                    break;
                }
                tc_fence_after();
                tc_st64(lane_base + kTcACol + 64 * ab, a);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&afull[ab]);
                    mbar_arrive(&empty[stage]);
                }
                if (++ab == 2) { ab = 0; aph ^= 1; }
                if (++stage == kTcStages) { stage = 0; phase ^= 1; }
            }
            if (fail) break;
            const int ra = pa->rank, rb = GLU ? pb->rank : 0;
            if (p.has_t && (ra > 0 || rb > 0)) {
                if (!warp_wait(&full[stage], phase)) {
                    fail = true;
                    break;
                }
                // this row's U values at the K slots of its projection's t columns
                const uint8_t* st = smem + stage * kTcStage;
                const uint16_t* src;
                int lo, r;
                bool u3;
                if (GLU && row >= 64) {
                    src = reinterpret_cast<const uint16_t*>(st + kTcOffUB) + (row - 64) * rb;
                    lo = p.t_col_b;
                    r = rb;
                    u3 = pb->lorc3 != 0;
                } else {
                    src = reinterpret_cast<const uint16_t*>(st + kTcOffUA) + row * ra;
                    lo = 0;
                    r = ra;
                    u3 = pa->lorc3 != 0;
                }
                if (!warp_wait(&aempty[ab], aph ^ 1)) {
                    fail = true;
                    break;
                }
                tc_fence_after();
                if (u3) {
                    // int3 U^T block: this row's feature, each rank row's code of
                    // it, eight TMEM columns at a time (a rolled loop keeps the
                    // code small)
                    const uint8_t* blk = st + ((GLU && row >= 64) ? kTcOffUB : kTcOffUA);
                    const int nl = ((w.ntile * RA) & 127) + (GLU ? (row & 63) : row);
#pragma unroll 1
                    for (int j0 = 0; j0 < 64; j0 += 8) {
                        uint32_t v8[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int slot = 2 * (j0 + i);
                            v8[i] = (slot >= lo && slot < lo + r) ? lorc3_value_pair(blk, slot - lo, nl) : 0u;
                        }
                        tc_st8(lane_base + kTcACol + 64 * ab + j0, v8);
                    }
                } else {
                    uint32_t a[64];
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        const int slot = 2 * j;
                        a[j] = (slot >= lo && slot < lo + r) ? *reinterpret_cast<const uint32_t*>(src + (slot - lo)) : 0u;
                    }
                    tc_st64(lane_base + kTcACol + 64 * ab, a);
                }
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&afull[ab]);
                    mbar_arrive(&empty[stage]);
                }
                if (++ab == 2) { ab = 0; aph ^= 1; }
                if (++stage == kTcStages) { stage = 0; phase ^= 1; }
            }
        }
        if (fail) st_bits |= MILO_DEV_TIMEOUT;
        flag(p.dev_status, st_bits);
    } else {
        // ---------------------------------------------------------------- fold + epilogue
        const int quarter = warp & 3;
        const int th = (warp - 6) >> 2;                    // routed rows kTcHalf * th .. kTcHalf * (th + 1) - 1
        const int row = 32 * quarter + lane;
        const uint32_t lane_base = tbase + (static_cast<uint32_t>(32 * quarter) << 16);
        const int half = row >> 6, r64 = row & 63;
        // byte offset of this row's (s, z) pair inside a group's 256 bytes
        const int pair_off = (((r64 >> 4) * 8 + (r64 & 7)) * 4 + ((r64 >> 3) & 1) * 2) * 2;
        int stage = 0, db = 0;
        uint32_t phase = 0, dph = 0;
        uint32_t xi = 0;        // items done: the exchange barriers complete one phase per item
        bool fail = false;
        int32_t st_bits = 0;
        for (int it = blockIdx.x; it < n_items && !fail; it += gridDim.x) {
            const TcItem w = tc_decode(it, start, cnt, p.n_exp, n_tiles, p.ntile_fast);
            const ProjDev* pa = p.table + w.e * p.stride + p.proj_a;
            const ProjDev* pb = p.table + w.e * p.stride + p.proj_b;
            const int n0 = w.ntile * RA;
            const int row0 = row0s[w.e] + w.tt * kTcTok;
            const int ntok = min(kTcTok, cnt[w.e] - w.tt * kTcTok);
            float2 acc[kTcHalf / 2];      // routed rows kTcHalf * th + 2i, +1
            float zinv = 1.0f;            // 2^-c of the row's zero-point scale (zp_scale)
#pragma unroll
            for (int i = 0; i < kTcHalf / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);

            for (int b = 0; b < p.SB; ++b) {
                if (!warp_wait(&full[stage], phase)) {
                    fail = true;
                    break;
                }
                const uint8_t* st = smem + stage * kTcStage;
                float s24[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float sv = __half2float(*reinterpret_cast<const __half*>(
                        st + kTcOffW + half * kBlockSB + kQTileSBWords * 4 + h * kGroupBytes + pair_off));
                    if (b == 0 && h == 0) zinv = inv_pow2(zp_scale(sv));
                    s24[h] = kFoldScale * sv;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
                if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                for (int h = 0; h < 2; ++h) {
                    if (!warp_wait(&dfull[db], dph)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    const float2 s2 = make_float2(s24[h], s24[h]);
                    const uint32_t dcol = lane_base + kTcDCol + kTcTok * db + kTcHalf * th;
#pragma unroll
                    for (int j = 0; j < kTcChunks; ++j) {
                        uint32_t d[kTcChunk];
                        tc_ld_chunk(dcol + kTcChunk * j, d);
                        tc_wait_ld();
                        if (j == kTcChunks - 1) {
                            // the last values are in registers: hand the buffer back first
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&dempty[db]);
                        }
#pragma unroll
                        for (int i = 0; i < kTcChunk / 2; ++i)
                            acc[kTcChunk / 2 * j + i] = __ffma2_rn(
                                s2, make_float2(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1])),
                                acc[kTcChunk / 2 * j + i]);
                    }
                    if (++db == kTcDBufs) { db = 0; dph ^= 1; }
                }
                if (fail) break;
            }
            if (fail) break;
            // the zero-point sums Z = 2^c sum_g (-s_g z_g) X_g: the last D_g's
            // commit covered the item's last zero-point step
#pragma unroll
            for (int j = 0; j < kTcChunks; ++j) {
                uint32_t d[kTcChunk];
                tc_ld_chunk(lane_base + kTcZCol + kTcHalf * th + kTcChunk * j, d);
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < kTcChunk / 2; ++i) {
                    acc[kTcChunk / 2 * j + i].x = fmaf(__uint_as_float(d[2 * i]), zinv, acc[kTcChunk / 2 * j + i].x);
                    acc[kTcChunk / 2 * j + i].y = fmaf(__uint_as_float(d[2 * i + 1]), zinv, acc[kTcChunk / 2 * j + i].y);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(zempty);
            const int ra = pa->rank, rb = GLU ? pb->rank : 0;
            if (p.has_t && (ra > 0 || rb > 0)) {
                // the compensator stage holds nothing this warp reads: release it once filled
                if (!warp_wait(&full[stage], phase)) {
                    fail = true;
                    break;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
                if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                if (!warp_wait(&dfull[db], dph)) {
                    fail = true;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < kTcChunks; ++j) {
                    uint32_t d[kTcChunk];
                    tc_ld_chunk(lane_base + kTcDCol + kTcTok * db + kTcHalf * th + kTcChunk * j, d);
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < kTcChunk / 2; ++i) {
                        acc[kTcChunk / 2 * j + i].x += __uint_as_float(d[2 * i]);
                        acc[kTcChunk / 2 * j + i].y += __uint_as_float(d[2 * i + 1]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dempty[db]);
                if (++db == kTcDBufs) { db = 0; dph ^= 1; }
            }

            // undo the rows' scale 2^a: token kTcHalf * th + 32 u + lane's scale
            // in register u of that lane, broadcast to the whole warp
            {
                float sc[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int t = kTcHalf * th + 32 * u + lane;
                    sc[u] = t < ntok && in_range(p.dev_status, row0 + t < p.R) ? inv_pow2(p.rscale[row0 + t]) : 0.0f;
                }
#pragma unroll
                for (int i = 0; i < kTcHalf / 2; ++i) {
                    const float s0 = __shfl_sync(0xFFFFFFFFu, sc[(2 * i) >> 5], (2 * i) & 31);
                    const float s1 = __shfl_sync(0xFFFFFFFFu, sc[(2 * i + 1) >> 5], (2 * i + 1) & 31);
                    acc[i].x *= s0;
                    acc[i].y *= s1;
                }
            }

            // ------------------------------------------------------------ epilogue
            if constexpr (GLU) {
                // SwiGLU h = silu(a) * b for output feature n0 + c: a is in TMEM
                // lane c (w1 row), b in lane 64 + c (w3 row), different warps.  Per
                // token half th the four warps of the half swap through their own
                // buffer [48 tokens][64 columns]: the w3 warps post b of the
                // first 24 tokens, the w1 warps a of the last 24, then each side
                // finishes its 24 tokens.  xfull / xempty (four arrivals) complete
                // one phase per item.
                const bool is_w1 = row < 64;
                const int c = row & 63;
                float* R = xch + th * kTcXchHalf;
                if (!warp_wait(&xempty[th], (xi + 1) & 1u)) {
                    fail = true;
                    break;
                }
                const int post0 = is_w1 ? kTcHalf / 2 : 0;     // tokens this side posts
#pragma unroll
                for (int i = 0; i < kTcHalf / 4; ++i) {
                    const float2 v = is_w1 ? acc[kTcHalf / 4 + i] : acc[i];
                    R[(post0 + 2 * i) * 64 + c] = v.x;
                    R[(post0 + 2 * i + 1) * 64 + c] = v.y;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&xfull[th]);
                if (!warp_wait(&xfull[th], xi & 1u)) {
                    fail = true;
                    break;
                }
                const int own0 = is_w1 ? 0 : kTcHalf / 2;       // tokens this side finishes
                const int f = n0 + c;
#pragma unroll
                for (int i = 0; i < kTcHalf / 4; ++i) {
                    const float2 mine = is_w1 ? acc[i] : acc[kTcHalf / 4 + i];   // tokens own0 + 2i, +1
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int tl = own0 + 2 * i + u;
                        const float other = R[tl * 64 + c];
                        const float own = u ? mine.y : mine.x;
                        const float av = is_w1 ? own : other;
                        const float bv = is_w1 ? other : own;
                        const int t = kTcHalf * th + tl;
                        if (t < ntok && f < p.N && in_range(p.dev_status, row0 + t < p.R)) {
                            const float hv = __fdividef(av, 1.0f + __expf(-av)) * bv;
                            const __half hh = __float2half_rn(hv);
                            if (!isfinite(hv)) st_bits |= MILO_DEV_NONFINITE;
                            else if (__hisinf(hh)) st_bits |= MILO_DEV_FP16_RANGE;
                            // streaming: h (R x I fp16) is far larger than L2 and is
                            // read once, by the next kernel
                            __stcs(p.h + static_cast<size_t>(row0 + t) * p.N + f, __half_as_ushort(hh));
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&xempty[th]);
                ++xi;
            } else {
                const int n = n0 + row;
                if (n < p.N) {
#pragma unroll
                    for (int i = 0; i < kTcHalf; ++i) {
                        const int t = kTcHalf * th + i;
                        if (t < ntok && in_range(p.dev_status, row0 + t < p.R))
                            // streaming stores: the output is read once, by the
                            // combine, and must not push the routed rows out of L2
                            __stcs(p.y_part + static_cast<size_t>(row0 + t) * p.N + n,
                                   (i & 1) ? acc[i >> 1].y : acc[i >> 1].x);
                    }
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
    static std::atomic<bool> configured[64][2];   // set once per device and kernel (a repeat is harmless)
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !configured[dev][glu].load(std::memory_order_acquire)) {
        e = glu ? cudaFuncSetAttribute(tc_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes)
                : cudaFuncSetAttribute(tc_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev][glu].store(true, std::memory_order_release);
    }
    // normal stream ordering, like the other persistent GEMM
    if (glu) tc_gemm_kernel<true><<<grid, kTcThreads, kTcSmemBytes, s>>>(p);
    else tc_gemm_kernel<false><<<grid, kTcThreads, kTcSmemBytes, s>>>(p);
    return cudaGetLastError();
}

}  // namespace milo
