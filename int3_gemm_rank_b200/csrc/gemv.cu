// gemv.cu -- grouped int3 x fp16 GEMM with the low-rank compensator, for
// decode-sized rows per expert (sm_100a).
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators":
//   - "MiLo Algorithm: Mixture of Low-Rank Compensators": W_out = W_quant + U V,
//     so y = x W_quant^T + (x V^T) U^T; the rank differs per expert and may be 0.
//   - "MiLo Kernel: Efficient Int3 Quantized GEMM Backend": int3 x FP16 GEMM
//     with dequantisation fused in (no separate dequantisation pass),
//     asynchronous global loads overlapping the math, and the asymmetric zero
//     point folded into the kernel.
//
// B200 design (not a translation of the page's kernel):
//   - One producer thread streams each CTA's weight tile into a 3-stage
//     shared-memory ring guarded by mbarriers.  The packed weights are stored
//     as (64-row tile, K chunk) blocks holding codes, scales and zeros
//     (milo.h), and the prepared activations of the item's routed rows (group
//     sums in the row padding) are contiguous too, so a stage is two or three
//     1-D bulk copies of the TMA engine.  Each copy instruction costs the
//     issuing thread about the same whatever its size, so the layout keeps
//     their number minimal.  Weights are read from HBM exactly once per token
//     tile, with an evict-first L2 policy.
//   - Four consumer warps each own 32 weight rows.  A lane reads its 3-word
//     unit of two rows and extracts code pairs with one LOP3 each (plus one
//     shift per word): the masked fp16 pattern already is code * 2^e * 2^-24,
//     and 2^(6 - e) is folded into the activations, which are shared by all
//     rows (as is the row's own scale 2^a, see kFoldScale).  mma.sync m16n8k16
//     (A = codes, B = tokens) accumulates D_g = 2^-18 * sum_k x'_k q_k per
//     scale group g; after each group the lane folds
//     acc += s * 2^18 * D_g - s * z * sum_k x'_k  in fp32, and the epilogue
//     multiplies by 2^-a.  The zero point thus costs nothing per weight and
//     the result is exact to fp32 rounding.
//   - The compensator runs as extra K-steps on the same accumulators:
//     A = U rows (fp16, or decoded from the int3 U^T blob), B = t = x V^T
//     (fp16).  t itself comes from "t-items" of the same launch, which every
//     CTA runs first (see decode_titem): the rows' plain copy times V by
//     ldmatrix + mma.sync from TMA boxes (fp16 V), or the V blob decoded by
//     this kernel's own chunk code (int3 V).
//   - Epilogue: SwiGLU h = silu(a) * b in the w1|w3 kernel (both rows live in
//     the same lane), or fp32 partial sums per K split for the plain one.
//   - A K chunk is two super-blocks; when K/128 is odd the last chunk has one,
//     and only the bytes that exist are copied and computed.
//   - Work items (expert, row tile, K split, 16-row token tile) are enumerated
//     on the device from the expert offsets, so the host never synchronises;
//     CTAs are persistent (three per SM) and walk the items round-robin, the
//     token tiles of one weight tile being adjacent so that they share L2.
//     The consumers learn each item, and what the producer decoded for it,
//     from a header the producer writes into the item's first stage; the
//     experts take turns in order of routed rows, most first, so that the
//     partial last round holds the cheapest items.
#include <cuda_runtime.h>

#include <atomic>

#include "milo_device.cuh"
#include "milo_host.h"
#include "milo_kernels.h"

namespace milo {

constexpr int kStages = 3;
constexpr int kConsumerWarps = 4;
constexpr int kGemvThreads = 32 * (kConsumerWarps + 1);
// Stage layout (bytes).  Two weight regions of kTileBlk bytes, each the nsb
// (tile, super-block) blocks of the packed blob: per super-block the codes
// [64 rows][12 words], then its two groups' (s, z) pairs (GLU: w1's tile,
// then w3's; plain: rows 0-63, then 64-127).  Then the activations
// [16 rows][272 fp16].  Stages are 1024-byte aligned for the t-items' swizzled
// TMA boxes, which fill a whole stage.
constexpr int kTileBlk = 2 * kBlockSB;                    // 7168
constexpr int kOffQ = 0;
constexpr int kOffX = 2 * kTileBlk;                       // 14336
constexpr int kStageBytes = 23552;
constexpr int kOffUA = 0, kOffUB = 8192, kOffT = 16384;   // compensator stage
constexpr int kBarOffset = kStages * kStageBytes;
// barriers, then the item tables cnt, row0s, tpos, tstart [MILO_MAX_EXPERTS +
// 1], the stage headers (kHdrInts each), the consumers' broadcast word and
// the expert order ord, pos [MILO_MAX_EXPERTS] (bytes); 1 KB of slack to
// align the base
constexpr int kHdrInts = 8;
constexpr int kSmemBytes = kBarOffset + 2 * kStages * 8 + 4 * (MILO_MAX_EXPERTS + 1) * 4 + kStages * kHdrInts * 4 + 16 +
                           2 * MILO_MAX_EXPERTS + 1024;
static_assert(MILO_MAX_EXPERTS <= 256, "expert order in bytes");

static_assert(kOffX + kTokTile * kFragRowHalves * 2 <= kStageBytes, "GEMM stage");
static_assert(kStageBytes % 1024 == 0, "stage alignment");
static_assert(3 * (kSmemBytes + 1024) <= 228 * 1024, "three CTAs per SM (1 KB reserved per CTA)");
static_assert(kStageBytes % 16 == 0 && kOffX % 16 == 0 && kTileBlk % 16 == 0, "bulk-copy alignment");
static_assert(kOffT >= kRowsPlain * MILO_MAX_RANK * 2, "compensator stage: U rows");
static_assert(kOffT + kTokTile * 2 * MILO_MAX_RANK * 2 <= kStageBytes, "compensator stage: t rows");

struct Item {
    int e, ntile, split, tt;
};

// Largest e in [0, n_exp) with first[e] * mul <= it (first[] non-decreasing).
__device__ __forceinline__ int find_expert(int it, const int* first, int mul, int n_exp) {
    int lo = 0, hi = n_exp - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (first[mid] * mul <= it) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// GEMM item `it`: the experts take turns in the order ord (most routed rows
// first); the expert at position k owns items [tpos[k], tpos[k+1]) * n_tiles
// * splits (tpos: prefix of the 16-row token tiles in that order), its token
// tiles fastest, then the K splits, then the weight-row tiles.
__device__ __forceinline__ Item decode_item(int it, const int* tpos, const uint8_t* ord, const int* cnt, int n_exp,
                                            int n_tiles, int splits) {
    Item r;
    const int k = find_expert(it, tpos, n_tiles * splits, n_exp);
    r.e = ord[k];
    const int local = it - tpos[k] * n_tiles * splits;
    const int tte = (cnt[r.e] + kTokTile - 1) / kTokTile;
    r.tt = local % tte;
    const int rest = local / tte;
    r.split = rest % splits;
    r.ntile = rest / splits;
    return r;
}

// t-items of a projection per token tile and K slice: one per 32 ranks of an
// fp16 V, one for an int3 V (its one 64-row tile).
__device__ __forceinline__ int rank_blocks(int r) { return (r + 31) >> 5; }
__device__ __forceinline__ int t_blocks(const ProjDev* P) {
    const int r = P->rank;
    return r == 0 ? 0 : P->lorc3 ? 1 : rank_blocks(r);
}

// Named barrier of the four consumer warps (the producer warp is not in it).
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// GPU-scope counters: an acquire-release add (returns the old value) and a
// release add.  A CTA barrier before them orders the CTA's other threads'
// writes too (the release is cumulative).
__device__ __forceinline__ int atom_add_acq_rel(int32_t* p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void red_add_release(int32_t* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// A t-item: t[row][col] = fp16(sum_k x'[row][k] V[rank][k]) for the 16 rows
// of one token tile of expert e, 32 ranks of one projection (8 per consumer
// warp) and one K slice; x' is the prepared rows' plain fp16 copy (already
// times their scale 2^a).  Items j of expert e are [tstart[e], tstart[e+1])
// * nks, K slices fastest, then rank blocks, then token tiles.
struct TItem {
    const ProjDev* P;     // the projection whose V it multiplies
    int e, ks, tt;        // expert, K slice, token tile
    int rb;               // first rank of the block
    int col;              // column of that rank in t
};

template <bool GLU>
__device__ __forceinline__ TItem decode_titem(const GemvParams& p, int j, int nks, const int* tstart) {
    TItem t;
    t.e = find_expert(j, tstart, nks, p.n_exp);
    const ProjDev* pa = p.table + t.e * p.stride + p.proj_a;
    const ProjDev* pb = p.table + t.e * p.stride + p.proj_b;
    const int na = t_blocks(pa), nb = GLU ? t_blocks(pb) : 0;
    const int local = j - tstart[t.e] * nks;
    t.ks = local % nks;
    const int rest = local / nks;
    const int rbi = rest % (na + nb);
    t.tt = rest / (na + nb);
    const bool second = rbi >= na;
    t.P = second ? pb : pa;
    t.rb = 32 * (second ? rbi - na : rbi);
    t.col = (second ? p.t_col_b : 0) + t.rb;
    return t;
}

// t-item stage (fp16 V): per 64 of K one TMA box of the 16 rows' plain copy
// and one of the block's 32 V rows, both 128-byte rows with the 128-byte
// swizzle; three of each per stage.
constexpr int kTBoxes = 3;
constexpr int kTStageK = 64 * kTBoxes;                    // 192
// K slices are whole stages of both kinds of t-item (192 of K with fp16 V,
// one 256 chunk with int3 V)
constexpr int kTSliceAlign = 768;
static_assert(kTSliceAlign % kTStageK == 0 && kTSliceAlign % kChunkK == 0, "t-item slices");
constexpr int kOffTX = 0, kTXBox = kTokTile * 128;        // 2048
constexpr int kOffTV = kTBoxes * kTXBox, kTVBox = 32 * 128;   // 6144, 4096
static_assert(kOffTV + kTBoxes * kTVBox <= kStageBytes && kOffTV % 1024 == 0, "t-item stage");

// Consumer side of a t-item with fp16 V: its stages (the first one already
// waited for) as m16n8k16 MMAs, A = the 16 rows (ldmatrix), B = the warp's 8
// V rows (ldmatrix), each stage released after use.  False on a timeout.
__device__ bool titem_tma(const TItem& ti, int kb0, int kb1, const uint8_t* smem, uint64_t* full,
                          uint64_t* empty, int& stage, uint32_t& phase, int warp, int lane, float (&acc)[4]) {
    const bool active = ti.rb + 8 * warp < ti.P->rank;   // the warp's 8 ranks exist
    const int arow = (lane & 7) + 8 * ((lane >> 3) & 1), achk = lane >> 4;
    const int brow = 8 * warp + (lane & 7), bchk = lane >> 3;
    for (int kc = kb0; kc < kb1; kc += kTStageK) {
        if (kc != kb0 && !warp_wait(&full[stage], phase)) return false;
        const uint8_t* st = smem + stage * kStageBytes;
        const int nbox = min(kTBoxes, (kb1 - kc) / 64);
        if (active) {
#pragma unroll
            for (int q = 0; q < kTBoxes; ++q) {
                if (q == nbox) break;
                const uint8_t* xb = st + kOffTX + q * kTXBox;
                const uint8_t* vb = st + kOffTV + q * kTVBox;
#pragma unroll
                for (int s2 = 0; s2 < 4; s2 += 2) {
                    uint32_t b[4];
                    ldmatrix_x4(b, vb + swz128(brow, 2 * s2 + bchk));
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t a[4];
                        ldmatrix_x4(a, xb + swz128(arow, 2 * (s2 + h) + achk));
                        mma16816(acc, a[0], a[1], a[2], a[3], b[2 * h], b[2 * h + 1]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
    }
    return true;
}

// End of t-item j: the lane's n results v[i] of token tok[i] and rank rk[i]
// (only those of the tile's tokens and the projection's ranks are stored).
// One slice: t directly.  Otherwise the slice's f32 partials go to tpart;
// the slice that counts last adds the slices in order (deterministic) and
// writes t.  The CTA that writes t then counts the t-item done for the token
// tile.
template <bool GLU, int N>
__device__ void titem_finish(const GemvParams& p, const TItem& ti, int j, int nks, int row0, int ntok,
                             const int* tpos, const uint8_t* pos, const float (&v)[N], const int (&tok)[N],
                             const int (&rk)[N],
                             volatile int* bcast) {
    const int r = ti.P->rank, col0 = ti.col - ti.rb;
    const int n_ttiles = (p.R + kTokTile - 1) / kTokTile + p.n_exp;   // as gemv_sync_ints
    int32_t st = 0;
    bool ok[N];
#pragma unroll
    for (int i = 0; i < N; ++i)
        ok[i] = tok[i] < ntok && rk[i] < r &&
                in_range(p.dev_status, row0 + tok[i] >= 0 && row0 + tok[i] < p.R && col0 + rk[i] < p.tcols &&
                                           ti.ks < p.nks);
    if (nks == 1) {
#pragma unroll
        for (int i = 0; i < N; ++i)
            if (ok[i]) p.t[static_cast<size_t>(row0 + tok[i]) * p.tcols + col0 + rk[i]] = t_half(v[i], st);
    } else {
        float* part = p.tpart + static_cast<size_t>(ti.ks) * p.R * p.tcols;
#pragma unroll
        for (int i = 0; i < N; ++i)
            if (ok[i]) part[static_cast<size_t>(row0 + tok[i]) * p.tcols + col0 + rk[i]] = v[i];
        // the CTA's partials, then one thread's acquire-release count: the last
        // slice to count sees every other slice's partials
        consumer_sync();
        if (threadIdx.x == 0)
            *bcast = in_range(p.dev_status, j / nks < 4 * n_ttiles) && atom_add_acq_rel(&p.tctr[j / nks], 1) == nks - 1;
        consumer_sync();
        const bool last = *bcast != 0;
        if (last) {
            const size_t slice = static_cast<size_t>(p.R) * p.tcols;
#pragma unroll
            for (int i = 0; i < N; ++i)
                if (ok[i]) {
                    const size_t o = static_cast<size_t>(row0 + tok[i]) * p.tcols + col0 + rk[i];
                    float a = 0.0f;
                    for (int s2 = 0; s2 < nks; ++s2) a += __ldcg(p.tpart + s2 * slice + o);
                    p.t[o] = t_half(a, st);
                }
        }
        consumer_sync();          // every warp has read bcast before it is reused
        if (!last) {
            flag(p.dev_status, st);
            return;
        }
    }
    consumer_sync();          // t is written; one release publishes it
    const int tile = tpos[pos[ti.e]] + ti.tt;   // the token tile's slot
    if (threadIdx.x == 0 && in_range(p.dev_status, tile < n_ttiles)) red_add_release(&p.tdone[tile], 1);
    flag(p.dev_status, st);
}

// One k16 step of the code part: extract the A fragments of both row tiles
// and multiply them with the prepared activation fragments of NT n8 tiles.
template <int S, int NT, int NTI>
__device__ __forceinline__ void code_step(const uint32_t (&wd)[2][2][3], const uint32_t (&hw)[2][2][3],
                                          const uint8_t* xs, int g, int c, float (&dz)[2][2][4]) {
    constexpr int t0 = sched_word(S, 0), f0 = sched_field(S, 0);
    constexpr int t1 = sched_word(S, 1), f1 = sched_field(S, 1);
    static_assert(S < kSteps, "schedule");
    uint2 b[NT];
#pragma unroll
    for (int n8 = 0; n8 < NT; ++n8)
        b[n8] = *reinterpret_cast<const uint2*>(xs + ((n8 * 8 + g) * kFragRowHalves + S * 16 + c * 4) * 2);
#pragma unroll
    for (int ti = 0; ti < NTI; ++ti) {
        const uint32_t a0 = unit_reg<t0, f0>(wd[ti][0], hw[ti][0]);
        const uint32_t a1 = unit_reg<t0, f0>(wd[ti][1], hw[ti][1]);
        const uint32_t a2 = unit_reg<t1, f1>(wd[ti][0], hw[ti][0]);
        const uint32_t a3 = unit_reg<t1, f1>(wd[ti][1], hw[ti][1]);
#pragma unroll
        for (int n8 = 0; n8 < NT; ++n8) {
            if constexpr (S == 0 || S == 4) mma16816_zc(dz[ti][n8], a0, a1, a2, a3, b[n8].x, b[n8].y);
            else mma16816(dz[ti][n8], a0, a1, a2, a3, b[n8].x, b[n8].y);
        }
    }
}

// Per m16 tile ti of a consumer warp: byte offset of its weight region in the
// stage and its first row inside the 64-row tile.
template <bool GLU>
struct TileMap {
    int reg[2], r[2];
    __device__ __forceinline__ explicit TileMap(int warp) {
#pragma unroll
        for (int ti = 0; ti < 2; ++ti) {
            if (GLU) {
                reg[ti] = ti * kTileBlk;
                r[ti] = 16 * warp;
            } else {
                reg[ti] = (warp >> 1) * kTileBlk;
                r[ti] = 32 * (warp & 1) + 16 * ti;
            }
        }
    }
};

// acc += s * 2^18 * D_g - s * z * X_g for group `grp` (0..3) of the chunk;
// super-block grp / 2's scales follow its codes, as (s, z) pairs of rows j and
// j + 8 of each 16-row block, so one 64-bit load brings the lane's two rows.
// xg[n8][j]: X_g of its tokens.
template <int NT, int NTI>
__device__ __forceinline__ void fold_group(float (&acc)[2][2][4], const float (&dz)[2][2][4],
                                           const uint8_t* st, int grp, const int (&reg)[2],
                                           const int (&rbase)[2], int g, const float (&xg)[NT][2]) {
#pragma unroll
    for (int ti = 0; ti < NTI; ++ti) {
        const uint2 q = *reinterpret_cast<const uint2*>(st + reg[ti] + (grp >> 1) * kBlockSB + kQTileSBWords * 4 +
                                                        (grp & 1) * kGroupBytes + ((rbase[ti] >> 4) * 8 + g) * 8);
        float s24[2], nsz[2];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const uint32_t v = rr ? q.y : q.x;
            const float sv = __half2float(__ushort_as_half(static_cast<uint16_t>(v & 0xFFFFu)));
            const float zv = __half2float(__ushort_as_half(static_cast<uint16_t>(v >> 16)));
            s24[rr] = sv * kFoldScale;
            nsz[rr] = -sv * zv;
        }
#pragma unroll
        for (int n8 = 0; n8 < NT; ++n8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int rr = i >> 1;
                acc[ti][n8][i] = fmaf(nsz[rr], xg[n8][i & 1], fmaf(s24[rr], dz[ti][n8][i], acc[ti][n8][i]));
            }
        }
    }
}

// One stage's K chunk (nsb super-blocks) on the warp's NTI m16 row tiles
// (NTI = 1: only tile 0, for the int3 compensator's t-items).
template <bool GLU, int NT, int NTI = 2>
__device__ __forceinline__ void chunk_compute(const uint8_t* st, float (&acc)[2][2][4], const TileMap<GLU>& tm,
                                              int nsb, int lane) {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int sbl = 0; sbl < 2; ++sbl) {
        if (sbl == nsb) break;
        uint32_t wd[2][2][3], hw[2][2][3];
#pragma unroll
        for (int ti = 0; ti < NTI; ++ti) {
            const uint32_t* qt = reinterpret_cast<const uint32_t*>(st + tm.reg[ti] + sbl * kBlockSB);
#pragma unroll
            for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                for (int t = 0; t < 3; ++t) {
                    wd[ti][rr][t] = qt[(tm.r[ti] + g + 8 * rr) * 12 + 3 * c + t];
                    hw[ti][rr][t] = wd[ti][rr][t] >> word_shift(t);
                }
        }
        const uint8_t* xs = st + kOffX + sbl * kFragHalvesPerSB * 2;
        // group sums of this super-block's two groups for the lane's tokens
        float xa[NT][2], xb[NT][2];
#pragma unroll
        for (int n8 = 0; n8 < NT; ++n8)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int tok = n8 * 8 + 2 * c + j;
                const float2 v = *reinterpret_cast<const float2*>(
                    st + kOffX + (tok * kFragRowHalves + kGsumHalf) * 2 + sbl * 8);
                xa[n8][j] = v.x;
                xb[n8][j] = v.y;
            }
        float dz[2][2][4];
        code_step<0, NT, NTI>(wd, hw, xs, g, c, dz);
        code_step<1, NT, NTI>(wd, hw, xs, g, c, dz);
        code_step<2, NT, NTI>(wd, hw, xs, g, c, dz);
        code_step<3, NT, NTI>(wd, hw, xs, g, c, dz);
        fold_group<NT, NTI>(acc, dz, st, 2 * sbl, tm.reg, tm.r, g, xa);
        code_step<4, NT, NTI>(wd, hw, xs, g, c, dz);
        code_step<5, NT, NTI>(wd, hw, xs, g, c, dz);
        code_step<6, NT, NTI>(wd, hw, xs, g, c, dz);
        code_step<7, NT, NTI>(wd, hw, xs, g, c, dz);
        fold_group<NT, NTI>(acc, dz, st, 2 * sbl + 1, tm.reg, tm.r, g, xb);
    }
}

// Values of rank row rho of an int3 U^T block (128 features) at features nl
// and nl + 8 (nl % 16 < 8: the same unit, codes 8 apart): (q - z) * s.
__device__ __forceinline__ float2 lorc3_pair(const uint8_t* blk, int rho, int nl) {
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(blk + lorc_words_off(rho, 0, blob_unit(nl)));
    const uint32_t w3[3] = {wp[0], wp[1], wp[2]};
    const uint32_t sz = *reinterpret_cast<const uint32_t*>(blk + lorc_sz_off(rho, nl >> 6));
    const float s = sz_scale(sz), z = sz_zero(sz);
    const int m = blob_code(nl);
    return make_float2((static_cast<float>(unit_code(w3, m)) - z) * s,
                       (static_cast<float>(unit_code(w3, m + 8)) - z) * s);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(lo))) |
           (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(hi))) << 16);
}

// Compensator K-steps: acc += U_tile * t^T over the rank (multiple of 8).  U
// rows are fp16 [rows][r] in the stage, or (u3a for w1 / the plain
// projection, u3b for w3) the item's int3 U^T block, whose features start at
// `nb0` inside the block.
template <bool GLU, int NT>
__device__ __forceinline__ void lorc_compute(const uint8_t* st, float (&acc)[2][2][4], int warp,
                                             int lane, int ra, int rb, int tcols, int t_col_b, bool u3a, bool u3b,
                                             int nb0) {
    const int g = lane >> 2, c = lane & 3;
    const uint16_t* tt = reinterpret_cast<const uint16_t*>(st + kOffT);
#pragma unroll
    for (int ti = 0; ti < 2; ++ti) {
        const int r = (GLU && ti == 1) ? rb : ra;
        const uint16_t* U = reinterpret_cast<const uint16_t*>(st + ((GLU && ti == 1) ? kOffUB : kOffUA));
        const int rbase = GLU ? 16 * warp : 32 * warp + 16 * ti;
        const int tc0 = (GLU && ti == 1) ? t_col_b : 0;
        for (int kk = 0; kk < r; kk += 16) {
            const int col = kk + 2 * c;
            const bool upper = col + 8 < r;
            uint32_t a0, a1, a2 = 0u, a3 = 0u;
            if ((GLU && ti == 1) ? u3b : u3a) {
                const uint8_t* blk = reinterpret_cast<const uint8_t*>(U);
                const int nl = nb0 + rbase + g;
                const float2 v0 = lorc3_pair(blk, col, nl), v1 = lorc3_pair(blk, col + 1, nl);
                a0 = pack_half2(v0.x, v1.x);
                a1 = pack_half2(v0.y, v1.y);
                if (upper) {
                    const float2 v8 = lorc3_pair(blk, col + 8, nl), v9 = lorc3_pair(blk, col + 9, nl);
                    a2 = pack_half2(v8.x, v9.x);
                    a3 = pack_half2(v8.y, v9.y);
                }
            } else {
                a0 = *reinterpret_cast<const uint32_t*>(U + (rbase + g) * r + col);
                a1 = *reinterpret_cast<const uint32_t*>(U + (rbase + g + 8) * r + col);
                if (upper) {
                    a2 = *reinterpret_cast<const uint32_t*>(U + (rbase + g) * r + col + 8);
                    a3 = *reinterpret_cast<const uint32_t*>(U + (rbase + g + 8) * r + col + 8);
                }
            }
#pragma unroll
            for (int n8 = 0; n8 < NT; ++n8) {
                const uint16_t* trow = tt + (n8 * 8 + g) * tcols + tc0;
                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(trow + col);
                const uint32_t b1 = upper ? *reinterpret_cast<const uint32_t*>(trow + col + 8) : 0u;
                mma16816(acc[ti][n8], a0, a1, a2, a3, b0, b1);
            }
        }
    }
}

// A GEMM item's stage header: its index, what the producer decoded for it,
// and its projections' ranks and compensator formats (info).
__device__ __forceinline__ void write_hdr(volatile int* h, int it, const Item& w, int info) {
    h[1] = w.e;
    h[2] = w.ntile;
    h[3] = w.tt | (w.split << 16);
    h[4] = info;
    h[0] = it;
}

template <bool GLU>
__global__ void __launch_bounds__(kGemvThreads, 3) gemv_kernel(const __grid_constant__ GemvParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
    uint64_t* empty = full + kStages;
    int* cnt = reinterpret_cast<int*>(empty + kStages);
    int* row0s = cnt + (MILO_MAX_EXPERTS + 1);
    int* tpos = row0s + (MILO_MAX_EXPERTS + 1);      // prefix of the token tiles in expert order ord
    int* tstart = tpos + (MILO_MAX_EXPERTS + 1);     // prefix of the experts' t-items (expert index order)
    // header of each stage: the work item whose first stage it is (-1: no more
    // items, -2 - j: t-item j), then for a GEMM item what the producer decoded
    // for it (expert, weight tile, token tile and K split, the ranks and
    // compensator formats), so that the consumers need no global loads for it
    volatile int* hdr = tstart + (MILO_MAX_EXPERTS + 1);
    volatile int* bcast = hdr + kStages * kHdrInts;   // consumers' broadcast word
    // the GEMM items' expert order (most routed rows first, then by index) and
    // each expert's position in it
    uint8_t* ord = reinterpret_cast<uint8_t*>(const_cast<int*>(bcast) + 4);
    uint8_t* pos = ord + MILO_MAX_EXPERTS;

    constexpr int RA = GLU ? kRowsGlu : kRowsPlain;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (p.N + RA - 1) / RA;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_barrier_init();
    }
    grid_dep_wait();
    // Item tables from the expert groups: all threads load the groups (and the
    // ranks, for the t-items), then warp 0 scans the token tiles and t-items.
    for (int e = threadIdx.x; e < p.n_exp; e += blockDim.x) {
        const int r0 = p.grp[2 * e], m = p.grp[2 * e + 1];
        const bool ok = m > 0 && r0 >= 0 && r0 + m <= p.R;
        cnt[e] = ok ? m : 0;
        row0s[e] = r0;
        const int tte = ok ? (m + kTokTile - 1) / kTokTile : 0;
        int nt = 0;
        if (p.t_items && tte > 0) {
            const int na = t_blocks(p.table + e * p.stride + p.proj_a);
            const int nb = GLU ? t_blocks(p.table + e * p.stride + p.proj_b) : 0;
            nt = tte * (na + nb);
        }
        tstart[e] = nt;
    }
    __syncthreads();
    // Whole waves of round-robin items are even; the last, partial one is not,
    // so the costlier items (more routed rows: 16-token tiles, several tiles)
    // go first and the last wave holds the cheapest.
    for (int e = threadIdx.x; e < p.n_exp; e += blockDim.x) {
        int rank = 0;
        for (int f = 0; f < p.n_exp; ++f) rank += cnt[f] > cnt[e] || (cnt[f] == cnt[e] && f < e);
        pos[e] = static_cast<uint8_t>(rank);
        ord[rank] = static_cast<uint8_t>(e);
    }
    __syncthreads();
    for (int k = threadIdx.x; k < p.n_exp; k += blockDim.x) tpos[k] = (cnt[ord[k]] + kTokTile - 1) / kTokTile;
    __syncthreads();
    if (warp == 0) {
        int run = 0, trun = 0;
        for (int base = 0; base < p.n_exp; base += 32) {
            const int e = base + lane;
            const int a = e < p.n_exp ? tpos[e] : 0, b = e < p.n_exp ? tstart[e] : 0;
            int ia = a, ib = b;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int ya = __shfl_up_sync(0xFFFFFFFFu, ia, o);
                const int yb = __shfl_up_sync(0xFFFFFFFFu, ib, o);
                if (lane >= o) { ia += ya; ib += yb; }
            }
            if (e < p.n_exp) {
                tpos[e] = run + ia - a;
                tstart[e] = trun + ib - b;
            }
            run += __shfl_sync(0xFFFFFFFFu, ia, 31);
            trun += __shfl_sync(0xFFFFFFFFu, ib, 31);
        }
        if (lane == 0) {
            tpos[p.n_exp] = run;
            tstart[p.n_exp] = trun;
        }
    }
    __syncthreads();
    const int n_items = tpos[p.n_exp] * n_tiles * p.splits;
    // K slices of the t-items: about one t-item per CTA (each slice pays a
    // fixed cost in counting and partial sums), at most p.nks slices, each a
    // whole number of stages; every CTA derives the same values from the same
    // tables
    int nks = 1, kslice = p.K;
    if (p.t_items && tstart[p.n_exp] > 0) {
        nks = max(1, min(p.nks, static_cast<int>(gridDim.x) / tstart[p.n_exp]));
        kslice = (((p.K + nks - 1) / nks) + kTSliceAlign - 1) / kTSliceAlign * kTSliceAlign;
        nks = (p.K + kslice - 1) / kslice;
    }
    const int n_t = tstart[p.n_exp] * nks;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        // The whole warp runs the loop (warp-uniform operands); one elected
        // lane issues the copies: issued from a divergent single-lane branch a
        // bulk copy costs the thread about 200 cycles.
        const uint64_t pol = l2_evict_first();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t filled = 0, fph = 0;     // per stage: has a fill, parity of its last fill
        bool fail = false;
        // This CTA's t-items first (j = G - 1 - b, + G, ...: one per CTA from
        // the last one down, so that every t is ready early; the last CTAs
        // have the fewest GEMM items), then its GEMM items, taken round-robin
        // (item b, b + G, ...).  A global work queue balanced the skewed
        // DeepSeekMoE-shaped layer no better and cost the Mixtral-shaped one
        // 15 %; the static split is kept.
        const int S = static_cast<int>(gridDim.x);
        int tj = S - 1 - static_cast<int>(blockIdx.x);
        int next = blockIdx.x;
        for (;;) {
            if (tj < n_t) {
                // a t-item: with fp16 V its stages of plain rows and V rows by
                // TMA; with an int3 V, like a GEMM item, its V-blob chunks and
                // the rows' prepared activations by bulk copies
                const TItem ti = decode_titem<GLU>(p, tj, nks, tstart);
                const int kb0 = ti.ks * kslice, kb1 = min(p.K, kb0 + kslice);
                const int trow0 = row0s[ti.e] + kTokTile * ti.tt;
                const bool l3 = ti.P->lorc3 != 0;
                // stages of 192 of K (fp16 V) or of one K chunk (int3 V)
                const int kstep = l3 ? kChunkK : kTStageK;
                const int tntok = min(kTokTile, cnt[ti.e] - kTokTile * ti.tt);
                for (int kc = kb0; kc < kb1; kc += kstep) {
                    if (!warp_wait(&empty[stage], phase ^ 1)) {
                        fail = true;
                        break;
                    }
                    uint8_t* st = smem + stage * kStageBytes;
                    uint64_t* fb = &full[stage];
                    filled |= 1u << stage;
                    fph = (fph & ~(1u << stage)) | (phase << stage);
                    if (elect_one()) {
                        if (kc == kb0) hdr[stage * kHdrInts] = -2 - tj;
                        if (l3) {
                            // the V blob's K chunk (its one 64-row tile) and the
                            // rows' prepared activations, as for a GEMM item
                            const int ch = kc / kChunkK;
                            const uint32_t vb = min(2, p.SB - 2 * ch) * kBlockSB;
                            const uint32_t xb = tntok * kFragRowHalves * 2;
                            if (in_range(p.dev_status, ch < p.chunks && 2 * ch < p.SB && tntok > 0 && trow0 >= 0 &&
                                                           trow0 + tntok <= p.R)) {
                                mbar_arrive_expect_tx(fb, vb + xb);
                                bulk_load_hint(st + kOffQ,
                                               reinterpret_cast<const uint8_t*>(ti.P->V) + 2 * ch * kBlockSB, vb, fb,
                                               pol);
                                bulk_load(st + kOffX, p.x + (static_cast<size_t>(ch) * p.R + trow0) * kFragRowHalves,
                                          xb, fb);
                            } else {
                                mbar_arrive(fb);
                            }
                        } else {
                            const int nbox = min(kTBoxes, (kb1 - kc) / 64);
                            if (!in_range(p.dev_status, kc + 64 * nbox <= p.K && trow0 >= 0 && trow0 < p.R &&
                                                            ti.rb < ti.P->rank)) {
                                mbar_arrive(fb);
                            } else {
                            mbar_arrive_expect_tx(fb, nbox * (kTXBox + kTVBox));
                            for (int q = 0; q < nbox; ++q) {
                                tma_load_2d(st + kOffTX + q * kTXBox, &p.smap, fb, kc + 64 * q, trow0);
                                tma_load_2d(st + kOffTV + q * kTVBox, &ti.P->vmap, fb, kc + 64 * q, ti.rb);
                            }
                            }
                        }
                    }
                    __syncwarp();
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
                if (fail) break;
                tj += S;
                continue;
            }
            const int it = next;
            if (it < 0 || it >= n_items) break;
            next += gridDim.x;
            bool header = false;      // the item's first stage has been filled
            const Item w = decode_item(it, tpos, ord, cnt, p.n_exp, n_tiles, p.splits);
            const ProjDev* pa = p.table + w.e * p.stride + p.proj_a;
            const ProjDev* pb = p.table + w.e * p.stride + p.proj_b;
            const int n0 = w.ntile * RA;
            const int tile0 = n0 / kTileRows;
            const int ntl = GLU ? 2 : min(2, (p.N - n0 + kTileRows - 1) / kTileRows);
            const int row0 = row0s[w.e] + w.tt * kTokTile;
            const int ntok = min(kTokTile, cnt[w.e] - w.tt * kTokTile);
            const int c0 = w.split * p.cps;
            const int c1 = min(p.chunks, c0 + p.cps);
            // the compensator stage's fields, loaded with the item's first ones
            const int ra = pa->rank, rb = GLU ? pb->rank : 0;
            const bool l3a = pa->lorc3 != 0, l3b = GLU ? pb->lorc3 != 0 : false;
            const int hinfo = ra | (rb << 8) | (l3a ? 1 << 16 : 0) | (l3b ? 1 << 17 : 0);
            const uint16_t* Ua = pa->U;
            const uint16_t* Ub = pb->U;
            for (int ch = c0; ch < c1; ++ch) {
                if (!warp_wait(&empty[stage], phase ^ 1)) {
                    fail = true;
                    break;
                }
                uint8_t* st = smem + stage * kStageBytes;
                uint64_t* fb = &full[stage];
                filled |= 1u << stage;
                fph = (fph & ~(1u << stage)) | (phase << stage);
                const int nsb = min(2, p.SB - 2 * ch);
                const uint32_t wb = nsb * kBlockSB;                  // one tile's block
                const uint32_t xb = ntok * kFragRowHalves * 2;
                const uint8_t* w0 = pa->packed + (static_cast<size_t>(tile0) * p.SB + 2 * ch) * kBlockSB;
                const uint8_t* w1 = GLU ? pb->packed + (static_cast<size_t>(tile0) * p.SB + 2 * ch) * kBlockSB
                                        : w0 + static_cast<size_t>(p.SB) * kBlockSB;
                const uint16_t* xsrc = p.x + (static_cast<size_t>(ch) * p.R + row0) * kFragRowHalves;
                if (elect_one()) {
                    if (!header) write_hdr(hdr + stage * kHdrInts, it, w, hinfo);
                    // each blob holds ceil(N / 64) tiles of SB blocks (SwiGLU: tile
                    // tile0 of w1's and of w3's; plain: tiles tile0 and tile0 + 1
                    // of one); the rows exist
                    if (in_range(p.dev_status, tile0 + (GLU ? 1 : ntl) <= (p.N + kTileRows - 1) / kTileRows &&
                                                   2 * ch + nsb <= p.SB && ch < p.chunks && ntok > 0 &&
                                                   row0 >= 0 && row0 + ntok <= p.R)) {
                        mbar_arrive_expect_tx(fb, ntl * wb + xb);
                        bulk_load_hint(st + kOffQ, w0, wb, fb, pol);
                        if (ntl == 2) bulk_load_hint(st + kOffQ + kTileBlk, w1, wb, fb, pol);
                        bulk_load(st + kOffX, xsrc, xb, fb);
                    } else {
                        mbar_arrive(fb);
                    }
                }
                __syncwarp();
                header = true;
                if (++stage == kStages) { stage = 0; phase ^= 1; }
            }
            if (fail) break;
            if (w.split == 0 && p.has_t && (ra > 0 || rb > 0)) {
                if (p.t_items) {
                    // this token tile's t comes from t-items of this launch:
                    // wait (bounded) until all its rank blocks are done
                    const int need = (ra == 0 ? 0 : l3a ? 1 : rank_blocks(ra)) +
                                     (GLU && rb > 0 ? (l3b ? 1 : rank_blocks(rb)) : 0);
                    const int32_t* done = p.tdone + tpos[pos[w.e]] + w.tt;
                    const int n_ttiles = (p.R + kTokTile - 1) / kTokTile + p.n_exp;   // as gemv_sync_ints
                    const bool dok = in_range(p.dev_status, tpos[pos[w.e]] + w.tt < n_ttiles);
                    if (dok && ld_acquire(done) < need) {
                        const long long t0 = clock64();
                        while (ld_acquire(done) < need) {
                            if (clock64() - t0 > kWaitCycles) {
                                fail = true;
                                break;
                            }
                            __nanosleep(64);
                        }
                    }
                    fail = __any_sync(0xFFFFFFFFu, fail);
                    if (fail) break;
                    // t was written by ordinary stores; the bulk copy reads it
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
                if (!warp_wait(&empty[stage], phase ^ 1)) {
                    fail = true;
                    break;
                }
                uint8_t* st = smem + stage * kStageBytes;
                uint64_t* fb = &full[stage];
                filled |= 1u << stage;
                fph = (fph & ~(1u << stage)) | (phase << stage);
                const int urows = min(RA, p.N - n0);
                // fp16 U rows, or the int3 U^T block holding the item's features
                const uint32_t ua = ra == 0 ? 0u : l3a ? kBlockSB : urows * ra * 2;
                const uint32_t ub = rb == 0 ? 0u : l3b ? kBlockSB : urows * rb * 2;
                const uint8_t* usa = l3a ? reinterpret_cast<const uint8_t*>(Ua) + (n0 >> 7) * kBlockSB
                                         : reinterpret_cast<const uint8_t*>(Ua + static_cast<size_t>(n0) * ra);
                const uint8_t* usb = !GLU ? usa : l3b ? reinterpret_cast<const uint8_t*>(Ub) + (n0 >> 7) * kBlockSB
                                                      : reinterpret_cast<const uint8_t*>(Ub + static_cast<size_t>(n0) * rb);
                const uint32_t tb = ntok * p.tcols * 2;
                if (elect_one()) {
                    if (!header) write_hdr(hdr + stage * kHdrInts, it, w, hinfo);
                    // U rows n0 .. n0 + urows (fp16) or the int3 U^T block of
                    // super-block n0 / 128 (N / 128 of them), the rows' t, and
                    // the stage's room for each
                    if (in_range(p.dev_status, n0 + urows <= p.N && ua <= (GLU ? kOffUB : kOffT) - kOffUA && ub <= kOffT - kOffUB &&
                                                   (!l3a || (n0 >> 7) < p.N / 128) &&
                                                   (!l3b || (n0 >> 7) < p.N / 128) && row0 >= 0 &&
                                                   row0 + ntok <= p.R && tb <= kStageBytes - kOffT)) {
                        mbar_arrive_expect_tx(fb, ua + ub + tb);
                        if (ua) bulk_load_hint(st + kOffUA, usa, ua, fb, pol);
                        if (ub) bulk_load_hint(st + kOffUB, usb, ub, fb, pol);
                        bulk_load(st + kOffT, p.t + static_cast<size_t>(row0) * p.tcols, tb, fb);
                    } else {
                        mbar_arrive(fb);
                    }
                }
                __syncwarp();
                header = true;
                if (++stage == kStages) { stage = 0; phase ^= 1; }
            }
            if (!fail && !header) {   // an item with no stage of its own: a header-only stage
                if (!warp_wait(&empty[stage], phase ^ 1)) {
                    fail = true;
                    break;
                }
                filled |= 1u << stage;
                fph = (fph & ~(1u << stage)) | (phase << stage);
                if (elect_one()) {
                    write_hdr(hdr + stage * kHdrInts, it, w, hinfo);
                    mbar_arrive(&full[stage]);
                }
                __syncwarp();
                if (++stage == kStages) { stage = 0; phase ^= 1; }
            }
            if (fail) break;
        }
        // end of the queue for this CTA's consumers
        if (!fail) {
            if (warp_wait(&empty[stage], phase ^ 1)) {
                filled |= 1u << stage;
                fph = (fph & ~(1u << stage)) | (phase << stage);
                if (elect_one()) {
                    hdr[stage * kHdrInts] = -1;
                    mbar_arrive(&full[stage]);
                }
                __syncwarp();
            } else {
                fail = true;
            }
        }
        // No copy may still be landing in shared memory when the CTA leaves.
        for (int s2 = 0; s2 < kStages; ++s2)
            if (((filled >> s2) & 1u) && !warp_wait(&full[s2], (fph >> s2) & 1u)) fail = true;
        if (fail && lane == 0) flag(p.dev_status, MILO_DEV_TIMEOUT);
        return;
    }

    // -------------------------------------------------------------- consumers
    int stage = 0;
    uint32_t phase = 0;
    const int g = lane >> 2, c = lane & 3;
    const TileMap<GLU> tm(warp);
    for (;;) {
        // the item's first stage carries its index in the stage header
        if (!warp_wait(&full[stage], phase)) {
            flag(p.dev_status, MILO_DEV_TIMEOUT);
            return;
        }
        const int it = hdr[stage * kHdrInts];
        if (it == -1) break;
        if (it < -1) {           // a t-item
            const int j = -2 - it;
            const TItem ti = decode_titem<GLU>(p, j, nks, tstart);
            const int kb0 = ti.ks * kslice, kb1 = min(p.K, kb0 + kslice);
            const int trow0 = row0s[ti.e] + kTokTile * ti.tt;
            const int tntok = min(kTokTile, cnt[ti.e] - kTokTile * ti.tt);
            if (ti.P->lorc3) {
                // int3 V: the GEMM's own decode of the V blob (rows = ranks)
                // against the rows' prepared activations; acc[0][n8][i] is
                // rank 16 warp + g + 8 (i >> 1) of token 8 n8 + 2c + (i & 1),
                // already times the row's 2^a
                float acc[2][2][4] = {};
                const TileMap<true> tmv(warp);
                const bool active = 16 * warp < ti.P->rank;
                for (int kc = kb0; kc < kb1; kc += kChunkK) {
                    if (kc != kb0 && !warp_wait(&full[stage], phase)) {
                        flag(p.dev_status, MILO_DEV_TIMEOUT);
                        return;
                    }
                    const int nsb = min(2, p.SB - 2 * (kc / kChunkK));
                    if (active) {
                        if (tntok > 8) chunk_compute<true, 2, 1>(smem + stage * kStageBytes, acc, tmv, nsb, lane);
                        else chunk_compute<true, 1, 1>(smem + stage * kStageBytes, acc, tmv, nsb, lane);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[stage]);
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
                float v[8];
                int tok[8], rk[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int n8 = q >> 2, i = q & 3;
                    v[q] = acc[0][n8][i];
                    tok[q] = 8 * n8 + 2 * c + (i & 1);
                    rk[q] = 16 * warp + g + 8 * (i >> 1);
                }
                titem_finish<GLU, 8>(p, ti, j, nks, trow0, tntok, tpos, pos, v, tok, rk, bcast);
            } else {
                float tacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                if (!titem_tma(ti, kb0, kb1, smem, full, empty, stage, phase, warp, lane, tacc)) {
                    flag(p.dev_status, MILO_DEV_TIMEOUT);
                    return;
                }
                // tacc[i]: token g + 8 (i >> 1), rank 8 warp + 2c + (i & 1) of the block
                int tok[4], rk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    tok[i] = g + 8 * (i >> 1);
                    rk[i] = ti.rb + 8 * warp + 2 * c + (i & 1);
                }
                titem_finish<GLU, 4>(p, ti, j, nks, trow0, tntok, tpos, pos, tacc, tok, rk, bcast);
            }
            continue;
        }
        bool waited = true;       // the next stage's barrier has been passed already
        Item w;
        int ra, rb;
        bool u3a, u3b;
        {
            const volatile int* h = hdr + stage * kHdrInts;
            w.e = h[1];
            w.ntile = h[2];
            w.tt = h[3] & 0xFFFF;
            w.split = h[3] >> 16;
            const int info = h[4];
            ra = info & 255;
            rb = (info >> 8) & 255;
            u3a = (info >> 16) & 1;
            u3b = GLU ? (info >> 17) & 1 : u3a;
        }
        const int n0 = w.ntile * RA;
        const int row0 = row0s[w.e] + w.tt * kTokTile;
        const int ntok = min(kTokTile, cnt[w.e] - w.tt * kTokTile);
        const int c0 = w.split * p.cps;
        const int c1 = min(p.chunks, c0 + p.cps);
        // the lane's tokens n8 * 8 + 2c + j: 2^-a undoes their rows' scale
        // 2^a; it sits in every activation row's padding (the first stage)
        float inv[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
        float acc[2][2][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[a][b][i] = 0.0f;

        for (int ch = c0; ch < c1; ++ch) {
            if (!waited && !warp_wait(&full[stage], phase)) {
                flag(p.dev_status, MILO_DEV_TIMEOUT);
                return;
            }
            waited = false;
            const uint8_t* st = smem + stage * kStageBytes;
            const int nsb = min(2, p.SB - 2 * ch);
            if (ch == c0) {
#pragma unroll
                for (int n8 = 0; n8 < 2; ++n8)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int tok = n8 * 8 + 2 * c + j;
                        inv[n8][j] = tok < ntok ? reinterpret_cast<const float*>(
                                                      st + kOffX + (tok * kFragRowHalves + kGsumHalf) * 2)[kInvSlot]
                                                : 0.0f;
                    }
            }
            if (ntok > 8) chunk_compute<GLU, 2>(st, acc, tm, nsb, lane);
            else chunk_compute<GLU, 1>(st, acc, tm, nsb, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (w.split == 0 && p.has_t && (ra > 0 || rb > 0)) {
            if (!waited && !warp_wait(&full[stage], phase)) {
                flag(p.dev_status, MILO_DEV_TIMEOUT);
                return;
            }
            waited = false;
            const uint8_t* st = smem + stage * kStageBytes;
            // int3 U^T blocks: the item's features start at n0 & 127 inside them
            if (ntok > 8) lorc_compute<GLU, 2>(st, acc, warp, lane, ra, rb, p.tcols, p.t_col_b, u3a, u3b, n0 & 127);
            else lorc_compute<GLU, 1>(st, acc, warp, lane, ra, rb, p.tcols, p.t_col_b, u3a, u3b, n0 & 127);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (waited) {   // a header-only stage: release it
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == kStages) { stage = 0; phase ^= 1; }
        }

        // ------------------------------------------------------------ epilogue
        if constexpr (GLU) {
            int32_t st = 0;
#pragma unroll
            for (int n8 = 0; n8 < 2; ++n8)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int f = n0 + 16 * warp + g + 8 * (i >> 1);
                    const int tok = n8 * 8 + 2 * c + (i & 1);
                    if (tok < ntok && f < p.N && in_range(p.dev_status, row0 + tok < p.R)) {
                        const float a = acc[0][n8][i] * inv[n8][i & 1], b = acc[1][n8][i] * inv[n8][i & 1];
                        const float hv = __fdividef(a, 1.0f + __expf(-a)) * b;
                        const __half hh = __float2half_rn(hv);
                        if (!isfinite(hv)) st |= MILO_DEV_NONFINITE;
                        else if (__hisinf(hh)) st |= MILO_DEV_FP16_RANGE;
                        p.h[static_cast<size_t>(row0 + tok) * p.N + f] = __half_as_ushort(hh);
                    }
                }
            flag(p.dev_status, st);
        } else {
            float* out = p.y_part + static_cast<size_t>(w.split) * p.R * p.N;
#pragma unroll
            for (int ti = 0; ti < 2; ++ti)
#pragma unroll
                for (int n8 = 0; n8 < 2; ++n8)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = n0 + 32 * warp + 16 * ti + g + 8 * (i >> 1);
                        const int tok = n8 * 8 + 2 * c + (i & 1);
                        if (tok < ntok && n < p.N && in_range(p.dev_status, row0 + tok < p.R && w.split < p.splits))
                            out[static_cast<size_t>(row0 + tok) * p.N + n] = acc[ti][n8][i] * inv[n8][i & 1];
                    }
        }
    }
}

size_t gemv_smem_bytes(bool) { return kSmemBytes; }

// Resident CTAs per SM of the kernel (its shared memory opted in), per device.
static int gemv_occupancy(bool glu, int dev) {
    static std::atomic<int> occ[64][2];
    int v = dev >= 0 && dev < 64 ? occ[dev][glu].load(std::memory_order_acquire) : 0;
    if (v > 0) return v;
    cudaError_t e = glu ? cudaFuncSetAttribute(gemv_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes)
                        : cudaFuncSetAttribute(gemv_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return -static_cast<int>(e);
    int n = 0;
    e = glu ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_kernel<true>, kGemvThreads, kSmemBytes)
            : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_kernel<false>, kGemvThreads, kSmemBytes);
    if (e != cudaSuccess) return -static_cast<int>(e);
    if (n < 1) return -static_cast<int>(cudaErrorInvalidConfiguration);
    if (dev >= 0 && dev < 64) occ[dev][glu].store(n, std::memory_order_release);
    return n;
}

cudaError_t launch_gemv(const GemvParams& p, bool glu, int sms, cudaStream_t s) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int occ = gemv_occupancy(glu, dev);
    if (occ < 0) return static_cast<cudaError_t>(-occ);
    // A normal (not programmatic) launch: the persistent grid starts once the
    // previous kernel has left every SM, so its CTAs are spread evenly over
    // the SMs (an early, programmatic launch places them wherever resources
    // free up first, and the per-SM load of the static item split then goes
    // uneven).  When CTAs wait on one another (t-items), the launch is
    // cooperative: every CTA is resident at once.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(occ * sms));
    cfg.blockDim = dim3(kGemvThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    return glu ? cudaLaunchKernelEx(&cfg, gemv_kernel<true>, p) : cudaLaunchKernelEx(&cfg, gemv_kernel<false>, p);
}

}  // namespace milo
