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

// One projection in the device table.  The tensor maps are encoded on the
// host at prepare time; the kernels read them from global memory.
struct alignas(64) ProjDev {
    CUtensorMap q_map;   // Q u32 [N, 3K/32], box {12 words, tile rows}
    CUtensorMap s_map;   // scale fp16 [K/64, N], box {tile rows, 4 groups}
    CUtensorMap z_map;   // zero  fp16 [K/64, N], box {tile rows, 4 groups}
    CUtensorMap u_map;   // U fp16 [N, r], box {r, tile rows}; unused when rank == 0
    const uint32_t* q;
    const uint16_t* scale;
    const uint16_t* zero;
    const uint16_t* U;
    const uint16_t* V;
    int32_t rank, N, K, tile_rows;
};

struct GemvParams {
    CUtensorMap x_map;          // prepared activations [R, SB*144] fp16, box {144, 16}
    CUtensorMap g_map;          // group sums [R, Gpad] f32, box {4, 16}
    CUtensorMap t_map;          // LoRC down-projection [R, tcols] fp16, box {tcols, 16}
    const ProjDev* table;       // device table
    const int32_t* grp;         // [n_exp][2]: first row, row count of each group (expert)
    float* y_part;              // plain: [splits][R][N] f32 partial sums
    uint16_t* h;                // SwiGLU: [R][N] fp16
    int32_t* dev_status;
    int stride, proj_a, proj_b; // table entries per expert; entry of A (w1 / the projection), B (w3)
    int n_exp, N, K, R;
    int splits, chunks, cps;    // split-K count, K chunks, chunks per split
    int has_t, tcols, t_col_b;  // LoRC activations present; row width; first column of w3's
};

struct PrepParams {
    const uint16_t* src;        // [*, K] bf16/fp16 (or fp16 h)
    int32_t* row_src;           // row p -> source row; built here when `rows` is set, else
                                // read (NULL: identity); -1 = zero row
    uint16_t* frag;             // [R, SB*144] fp16
    float* gsum;                // [R, Gpad] f32
    int32_t* dev_status;
    int R, K, gpad, src_bf16;
    int layout;                 // 0: mma.sync fragments [R][K/128][144]; 1: tcgen05 A-column order [R][K]
    // Row bookkeeping (first preparation of a call only): routed rows come from
    // the router's offsets/perm, the n_shared*T shared-expert rows follow them.
    int rows;                   // 1: build grp / row_src / inv from offsets and perm
    const int32_t* offsets;     // [E+1]
    const int32_t* perm;        // [T*k] or NULL (identity)
    int32_t* grp;               // [E+S][2]: first row, row count
    int32_t* inv;               // optional [T*k] inverse of perm (-1 = dropped)
    int T, k, E, S, R_routed;
};

struct LorcParams {
    const uint16_t* src;        // [*, K] bf16/fp16 rows
    const int32_t* row_src;     // row p -> source row (NULL: identity); -1 = zero row
    const ProjDev* table;
    const int32_t* grp;         // [n_exp][2]
    uint16_t* t;                // [R, tcols] fp16
    float* part;                // [splits][R][tcols] f32 partial sums over K slices
    int32_t* dev_status;
    int stride, proj_a, proj_b; // proj_b < 0: single projection
    int n_exp, K, R, tcols, t_col_b, src_bf16;
    int splits, row_groups;     // K slices (each a multiple of 128); row-tile strides
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

// Parameters of the tcgen05 grouped GEMM (gemm_tc.cu).
struct TcParams {
    CUtensorMap b_map;          // activations in A-column order [R, K] fp16, box {64, 16}, 128B swizzle
    CUtensorMap g_map;          // group sums [R, Gpad] f32, box {4, 16}
    CUtensorMap t_map;          // compensator activations [R, tcols] fp16, box {64, 16}, 128B swizzle
    const ProjDev* table;
    const int32_t* grp;
    float* y_part;
    uint16_t* h;
    int32_t* dev_status;
    int stride, proj_a, proj_b;
    int n_exp, N, K, R;
    int splits, chunks, cps;
    int has_t, tcols, t_col_b;
};

size_t tc_smem_bytes();
cudaError_t launch_tc_gemm(const TcParams& p, bool glu, int grid, cudaStream_t s);
size_t gemv_smem_bytes(bool glu);
cudaError_t launch_gemv(const GemvParams& p, bool glu, int grid, cudaStream_t s);
cudaError_t launch_prep(const PrepParams& p, cudaStream_t s);
cudaError_t launch_lorc(const LorcParams& p, cudaStream_t s);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t s);

}  // namespace milo
