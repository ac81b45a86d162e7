// milo_kernels.h -- device-table entries, kernel parameter blocks and launch
// declarations shared by the host API (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/milo.h"

namespace milo {

// Tile shapes of the grouped int3 GEMM.
constexpr int kRowsPlain = 128;    // output rows per CTA, plain projection
constexpr int kRowsGlu = 64;       // output features per CTA, w1|w3 + SwiGLU (128 weight rows)
constexpr int kTokTile = 16;       // routed rows per work item (two n8 MMA tiles)
constexpr int kChunkK = 256;       // K per pipeline stage (two 128-code super-blocks)

// Prepared activations: per row and K chunk (two super-blocks), for each
// super-block 8 MMA steps x 4 lanes-in-quad x 4 fp16, then 16 fp16 of padding
// so that the rows of a 16-row tile fall on different shared-memory banks
// (row pitch 136 words, 8 mod 32): 272 fp16 (544 bytes).
// The first 8 padding fp16 hold the chunk's four group sums (f32).
//
// Row scaling: every activation row v (an x row or an h row) is multiplied by
// a power of two 2^a chosen from its largest magnitude (max |v| 2^a in [1, 2))
// before it is rounded to fp16, so that small rows keep their precision and
// large ones fit; the power of two of the int3 field it meets is then applied
// upwards (x 2^(6 - e), exact: the values stay below 2^7).  The products in
// the MMA are thus 2^a * 2^-18 * v * code, the group sums are sums of
// fp16(v 2^a), the compensator's t = fp16(2^a v V^T), and the GEMM epilogue
// multiplies the row's result by 2^-a.  Both factors are exact.
constexpr float kFoldScale = 262144.0f;   // 2^18: undoes the 2^-18 of the code operand
constexpr int kFragHalvesPerSB = 128;
constexpr int kFragRowHalves = 2 * kFragHalvesPerSB + 16;
constexpr int kGsumHalf = 2 * kFragHalvesPerSB;
// Row padding of a chunk (f32 slots from kGsumHalf): the chunk's four group
// sums, then the row's 2^-a.
constexpr int kInvSlot = 4;

// Packed weights (milo.h): rows in tiles of 64; each (tile, super-block)
// block -- the codes, then the two groups' scales and zeros -- is contiguous,
// and consecutive super-blocks of a tile are adjacent, so one bulk copy brings
// a tile's K chunk.  kBlockSB bytes per tile and super-block.
constexpr int kTileRows = 64;
constexpr int kQTileSBWords = kTileRows * 12;       // codes of one tile, one super-block: 3072 bytes
constexpr int kGroupBytes = kTileRows * 2 * 2;      // scales and zeros of one tile, one group: 256 bytes
constexpr int kBlockSB = kQTileSBWords * 4 + 2 * kGroupBytes;   // 3584
constexpr int kTcTokens = 128;               // routed rows per tcgen05 work item (the TMA box height)

// One projection in the device table (device pointers and shape).
struct alignas(64) ProjDev {
    CUtensorMap vmap;           // fp16 V [rank][K]: box {64, 32}, 128-byte swizzle (unset for lorc3 or rank 0)
    const uint8_t* packed;      // blob of ceil(N/64) * (K/128) * kBlockSB bytes
    const uint16_t* U;          // [N][rank] fp16, or (lorc3) the blob of U^T [rank][N]; NULL when rank == 0
    const uint16_t* V;          // [rank][K] fp16, or (lorc3) the blob of V [rank][K]; NULL when rank == 0
    int32_t rank, N, K, lorc3;  // lorc3: the compensator is int3 (both blobs one 64-row tile high)
};

struct CombineParams {
    const float* y_part;        // [splits][R][H]
    const int32_t* inv_perm;    // [T*k] row of each flat slot (-1 = dropped)
    const float* w;             // [T*k] combine weights (NULL: 1, and k slots are rows)
    void* y;                    // output
    int32_t* dev_status;
    int T, k, S, H, R, splits, R_routed, y_dt;
    int per_slot;               // 1: y row per flat slot (grouped linear), 0: per token
};

struct GemvParams {
    CUtensorMap smap;           // the rows' plain fp16 copy `src` [R][K]: box {64, 16}, 128-byte swizzle
    const uint16_t* x;          // prepared activations [chunks][R][kFragRowHalves] fp16
                                // (group sums and 2^-a in each row's padding, see kGsumHalf)
    const float* rscale;        // [R]: the row's activation scale 2^a (see kFoldScale)
    uint16_t* t;                // LoRC down-projection [R][tcols] fp16 (times the row's 2^a)
    const ProjDev* table;       // device table
    const int32_t* grp;         // [n_exp][2]: first row, row count of each group (expert)
    float* y_part;              // plain: [splits][R][N] f32 partial sums
    uint16_t* h;                // SwiGLU: [R][N] fp16
    int32_t* dev_status;
    int stride, proj_a, proj_b; // table entries per expert; entry of A (w1 / the projection), B (w3)
    int n_exp, N, K, R, SB, G;  // G = K / 64 groups
    int splits, chunks, cps;    // split-K count, K chunks, chunks per split
    int has_t, tcols, t_col_b;  // LoRC activations present; row width; first column of w3's
    // Compensator down-projection computed in the kernel ("t-items", first on
    // the CTAs with the fewest GEMM items): t = fp16(x' V^T) per (expert,
    // projection, 32 ranks, 16-row token tile, K slice); the slice that
    // finishes last adds the slices in order, and a GEMM item waits (bounded)
    // until its token tile's t is complete before copying it.
    int t_items;                // 0: t was computed beforehand
    const uint16_t* src;        // the rows' plain fp16 copy [R][K] (times their scale 2^a)
    int nks, kslice;            // the most K slices per t-item and their least length (multiple of
                                // 256): the kernel picks fewer, longer slices when t-items are many
    float* tpart;               // [nks][R][tcols] f32 slice partials
    int32_t* tctr;              // per (expert, token tile, rank block): slices finished (0 on entry)
    int32_t* tdone;             // per (expert, token tile): rank blocks finished (0 on entry)
};

// Ints of the t-item counters of a grouped GEMM over R rows and n_exp experts
// (zeroed before each launch).
inline int gemv_sync_ints(int R, int n_exp) {
    const int tiles = (R + kTokTile - 1) / kTokTile + n_exp;   // token tiles of all experts, at most
    return tiles * 4 + tiles;
}

// Parameters of the tcgen05 grouped GEMM for large per-expert row counts
// (gemm_tc.cu).  Activations in MMA column order [R][K] fp16 and their group
// sums [R][4 * chunks] f32 arrive by 2-D TMA; weights as blob blocks.
struct TcParams {
    CUtensorMap b_map;          // activations [R][K] fp16, box {64, kTcTokens}, 128-byte swizzle
    CUtensorMap z_map;          // group sums [R][chunks][16] fp16 (hi, lo, hi, lo per group), box {16, kTcTokens}
    CUtensorMap t_map;          // LoRC down-projection [R][tcols] fp16, box {64, kTcTokens}, 128-byte swizzle
    const float* rscale;        // [R]: the row's activation scale 2^a
    const ProjDev* table;
    const int32_t* grp;
    float* y_part;              // plain: [R][N] f32
    uint16_t* h;                // SwiGLU: [R][N] fp16
    int32_t* dev_status;
    int stride, proj_a, proj_b;
    int n_exp, N, K, R, SB;
    int has_t, tcols, t_col_b;
    int ntile_fast;             // item order inside an expert: 1 = weight tiles fastest (routed-row tile
                                // stays hot in L2), 0 = routed-row tiles fastest (weight tile stays hot)
};

struct PrepParams {
    const uint16_t* src;        // [*, K] bf16/fp16 (or fp16 h)
    int32_t* row_src;           // row p -> source row; built here when `rows` is set, else
                                // read (NULL: identity); -1 = zero row
    uint16_t* frag;             // layout 0: [chunks][R][kFragRowHalves] fp16, chunks = ceil(K/256);
                                // layout 1: [R][K] fp16 in tcgen05 A-column order
    uint16_t* gsum;             // layout 1: group sums [R][chunks][16] fp16: per group (hi, lo, hi, lo)
    float* rscale;              // [R]: written, the row's scale 2^a (1 for a zero row)
    uint16_t* plain;            // optional [R][K]: written, the row's fp16 values times 2^a
    int layout;
    int32_t* dev_status;
    int R, K, src_bf16;
    // Row bookkeeping (first preparation of a call only): routed rows come from
    // the router's offsets/perm, the n_shared*T shared-expert rows follow them.
    int rows;                   // 1: build grp / row_src / inv from offsets and perm
    const int32_t* offsets;     // [E+1]
    const int32_t* perm;        // [T*k] or NULL (identity)
    int32_t* grp;               // [E+S][2]: first row, row count
    int32_t* inv;               // optional [T*k] inverse of perm (-1 = dropped)
    int T, k, E, S, R_routed;
    int32_t* zero;              // optional: `nzero` ints set to 0 (the compensator's slice counters)
    int nzero;
};

struct LorcParams {
    const uint16_t* src;        // [*, K] bf16/fp16 rows
    const int32_t* row_src;     // row p -> source row (NULL: identity); -1 = zero row
    const float* rscale;        // [R]: the row's activation scale 2^a (written by prep)
    const ProjDev* table;
    const int32_t* grp;         // [n_exp][2]
    uint16_t* t;                // [R, tcols] fp16: 2^a x V^T
    float* part;                // [splits][R][tcols] f32 partial sums over K slices
    int32_t* done;              // per (expert, projection, rank block, row group): slices finished; 0 on entry
    int32_t* dev_status;
    int stride, proj_a, proj_b; // proj_b < 0: single projection
    int n_exp, K, R, tcols, t_col_b, src_bf16;
    int splits, row_groups;     // K slices of ceil(K/128 / splits) super-blocks; row-tile strides
};

// Counters lorc_partial_kernel needs when it splits K (then at most 8 row
// groups); zeroed by prep_kernel and left at zero.
constexpr int kLorcCounters = MILO_MAX_EXPERTS * 2 * ((MILO_MAX_RANK + 15) / 16) * 8;


size_t tc_smem_bytes();
cudaError_t launch_tc_gemm(const TcParams& p, bool glu, int grid, cudaStream_t s);
size_t gemv_smem_bytes(bool glu);
cudaError_t launch_gemv(const GemvParams& p, bool glu, int grid, cudaStream_t s);
cudaError_t launch_prep(const PrepParams& p, cudaStream_t s);
cudaError_t launch_lorc(const LorcParams& p, cudaStream_t s);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t s);

}  // namespace milo
