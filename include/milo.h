/*
 * milo.h -- C ABI of the B200 (sm_100a) int3 + low-rank-compensator MoE forward.
 *
 * The operation is the inference hot path of "MiLo: Efficient Quantized MoE
 * Inference with Mixture of Low-Rank Compensators":
 *
 *   - section "MiLo Algorithm: Mixture of Low-Rank Compensators": every expert
 *     weight is W_out = W_quant + U V, a quantised matrix plus a rank-r
 *     compensator, with a rank that may differ per expert (and may be 0).  For
 *     an out x in weight this library stores U [N, r] and V [r, K] and computes
 *         y = x W_quant^T + (x V^T) U^T ;
 *   - section "MiLo Kernel: Efficient Int3 Quantized GEMM Backend": int3
 *     weights times FP16 activations (W3A16), 32 three-bit values packed in
 *     three 32-bit words without a wasted bit, dequantisation asymmetric with a
 *     zero point and fused into the GEMM;
 *   - sections "Background" and "Experimental Setup & Results": the MoE layer
 *     routes each token to a subset of experts (Mixtral-8x7B-style top-k).
 *
 * Conventions (all entry points):
 *   - Pointers are device pointers owned by the caller unless a comment says
 *     "host".  The library never allocates device memory and never
 *     synchronises the host, except milo_*_prepare (documented below).
 *   - Raw 16-bit floats are passed as uint16_t (fp16 or bf16 bit patterns).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued on it; results are ready when the stream reaches that point.
 *   - Argument errors are returned synchronously as milo_status and nothing is
 *     enqueued.  Data-dependent errors found on the device are OR-ed into the
 *     caller's `dev_status` word (MILO_DEV_* bits); the caller zeroes it and
 *     reads it after the stream completes.  `dev_status` may be NULL only where
 *     stated.
 *   - Every call is deterministic: identical inputs give identical bits.
 *   - Calls sharing one workspace must not overlap.
 */
#ifndef MILO_H
#define MILO_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MILO_API __attribute__((visibility("default")))
#else
#define MILO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MILO_F16 = 0, MILO_BF16 = 1, MILO_F32 = 2 } milo_dtype;

typedef enum {
    MILO_OK = 0,
    MILO_ERR_INVALID_ARG = 1,       /* NULL pointer, negative size, bad enum */
    MILO_ERR_UNSUPPORTED_SHAPE = 2, /* e.g. K not a multiple of 128, group != 64 */
    MILO_ERR_WORKSPACE = 3,         /* workspace or table too small / misaligned */
    MILO_ERR_CUDA = 4               /* a CUDA runtime call failed (see milo_last_error) */
} milo_status;

/* Device status bits, OR-ed into *dev_status by the kernels. */
#define MILO_DEV_BAD_EXPERT_ID 0x1  /* a routed id outside [0, E): the slot is dropped */
#define MILO_DEV_NONFINITE 0x2      /* NaN/Inf in weights, logits or activations */
#define MILO_DEV_FP16_RANGE 0x4     /* a value does not fit fp16 (s, z, h, an fp16 output) */
#define MILO_DEV_TIMEOUT 0x8        /* a bounded pipeline wait gave up; outputs invalid */
/* Checked build only (libmilo_checked.so, compiled with MILO_CHECKED): an
 * index or copy range fell outside its buffer; that access was skipped and
 * the outputs are invalid.  The normal build performs no such checks. */
#define MILO_DEV_BOUNDS 0x10

/* Router flags. */
#define MILO_ROUTE_RENORM 0x1u      /* renormalise the softmax over the k picked experts */
#define MILO_ROUTE_IDS_GIVEN 0x2u   /* topk_ids are inputs (logits NULL, topk_w untouched) */

/* Compile-time limits of the library. */
#define MILO_GROUP 64               /* scale/zero group along K */
#define MILO_MAX_RANK 64            /* compensator rank, a multiple of 8 */
#define MILO_MAX_EXPERTS 256        /* routed + shared */
#define MILO_MAX_TOPK 16
/* Rows of one call: T*k for milo_route and milo_grouped_linear, T*(top_k +
 * n_shared) for milo_moe_forward.  Row indices and counts are 32-bit on the
 * device; a call above this returns MILO_ERR_UNSUPPORTED_SHAPE. */
#define MILO_MAX_ROWS 0x3FFFFFFF

MILO_API const char* milo_status_str(milo_status s);
/* Host string describing the last failure on the calling thread ("" if none). */
MILO_API const char* milo_last_error(void);
MILO_API int32_t milo_version(void);

/* ------------------------------------------------------------------------ */
/* Packed int3 weights                                                      */
/* ------------------------------------------------------------------------ */
/*
 * Packing format (self-defined; the page describes three 32-bit words holding
 * 32 three-bit values with no wasted bit but its bit positions are garbled):
 * a row of K codes, K a multiple of 128, is cut into super-blocks of 128 codes
 * (two scale groups of 64).  Super-block b occupies words 12b..12b+11 of the
 * row, as four 3-word units.  Unit c (0..3) carries the 32 codes
 *     u_m = q[128b + 16c + m]             m = 0..15   (first group)
 *     u_m = q[128b + 64 + 16c + m - 16]   m = 16..31  (second group)
 * and word t (0..2) of the unit holds, for i = 0..4,
 *     bits [3i, 3i+3) = u_{10t+2i},   bits [16+3i, 16+3i+3) = u_{10t+2i+1},
 * bit 15 = bit t of u_30, bit 31 = bit t of u_31.
 *
 * Device layout: one blob per weight.  Rows are grouped in tiles of 64 (the
 * last tile padded with zero rows).  The (tile t, super-block b) block starts
 * at byte (t * K/128 + b) * 3584 and holds
 *     the words u32 [64 rows][12]      (word j of row 64t+r = word 12b+j above)
 * then, for groups 2b and 2b+1, 256 bytes each: for each 16-row block m
 * (0..3) and j (0..7) the fp16 quadruple s, z of row 16m+j, s, z of row 16m+j+8
 * so that the kernels fetch one or more consecutive super-blocks of a tile --
 * codes, scales and zeros -- with one copy.
 * Dequantisation: w_hat[n, k] = (q[n, k] - z[n, k/64]) * s[n, k/64].
 * The blob has ceil(N/64) * (K/128) * 3584 bytes (milo_packed_bytes).
 * N is at most 2^31 - 64, so that the padded row count stays a 32-bit
 * integer (UNSUPPORTED_SHAPE above).
 */

/* Bytes of the packed blob of a weight [N, K] (K % 128 == 0), written to the
 * host size_t *bytes.  Errors: K % 128 != 0 or N above 2^31 - 64 ->
 * UNSUPPORTED_SHAPE; N, K <= 0 or bytes NULL -> INVALID_ARG. */
MILO_API milo_status milo_packed_bytes(int32_t N, int32_t K, size_t* bytes);

/*
 * milo_pack -- quantise W fp16 [N, K] (row-major) to int3 and pack it.
 * Round-to-nearest asymmetric min/max per group of 64 along K (the paper's HQQ
 * initialisation is milo_hqq_pack / milo_quantize_lorc; with one iteration HQQ
 * gives exactly this):
 *     s = fp16((max - min) / 7)   (s := 1 when it rounds to 0)
 *     z = fp16(-min / s)
 *     q = clamp(rint(w / s + z), 0, 7)    (fp32, ties to even, no FMA)
 * Writes the blob in the device layout above, padding rows included (size
 * from milo_packed_bytes; 16-byte aligned).
 * Errors: group != 64, K % 128 != 0 or N above 2^31 - 64 -> UNSUPPORTED_SHAPE;
 * N, K <= 0, NULL pointers or a packed buffer not 16-byte aligned ->
 * INVALID_ARG.  Device: NONFINITE for NaN/Inf weights, FP16_RANGE when s or z
 * overflows fp16.  dev_status may be NULL.  W and packed are caller-owned
 * device memory; stream-ordered.
 */
MILO_API milo_status milo_pack(const uint16_t* W, int32_t N, int32_t K, int32_t group, void* packed,
                      int32_t* dev_status, void* stream);

/*
 * milo_unpack -- extract the codes of a packed blob (device layout above)
 * into codes u8 [N, K] row-major, with the same register-level field
 * extraction the GEMM kernels use.  packed (4-byte aligned) and codes are
 * caller-owned device memory; stream-ordered.
 * Errors: K % 128 != 0 or N above 2^31 - 64 -> UNSUPPORTED_SHAPE; N, K <= 0,
 * NULL or misaligned pointers -> INVALID_ARG.
 */
MILO_API milo_status milo_unpack(const void* packed, int32_t N, int32_t K, uint8_t* codes,
                        void* stream);

/*
 * milo_dequantize -- the dequantised weights of a packed blob, as fp16:
 * W_hat[n, k] = fp16((q[n, k] - z[n, k/64]) * s[n, k/64]), row-major [N, K],
 * rounded once to nearest even (the product is formed exactly).  This is the
 * first pass of the unfused pipeline the paper compares its fused kernel
 * against ("Experimental Setup & Results": the int3 GEMM is several times
 * faster than the unfused implementation, a dequantisation pass followed by
 * an FP16 GEMM); the fused GEMMs of this library never materialise W_hat.
 *   packed: the blob (16-byte aligned); W_hat: fp16 [N, K] (16-byte aligned).
 * Errors: K % 128 != 0 or N above 2^31 - 64 -> UNSUPPORTED_SHAPE; N, K <= 0,
 * NULL or misaligned pointers -> INVALID_ARG.  Stream-ordered.
 */
MILO_API milo_status milo_dequantize(const void* packed, int32_t N, int32_t K, uint16_t* W_hat, void* stream);

/* ------------------------------------------------------------------------ */
/* Offline MiLo quantiser                                                   */
/* ------------------------------------------------------------------------ */
/*
 * "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
 * Compensators", section "MiLo Algorithm: Mixture of Low-Rank Compensators":
 * (1) the weights are quantised with HQQ (half-quadratic quantisation, no
 * calibration data); (2) the residual W - W_quant is approximated by the top-r
 * singular triplets of its SVD, U V; then quantisation and compensation are
 * refined in turn: W_quant from W - U V, U V from the new residual.
 *
 * HQQ here (per group of 64 along K, all fp32 in this order, no FMA):
 *     s = fp16((max - min) / 7) (1 when it rounds to 0), z = -min / s, beta = hqq_beta
 *     repeat hqq_iters times:
 *         q = clamp(rint(t * (1/s) + z), 0, 7);  e = t - (q - z) s
 *         L1 = sum |e| (index order); remember z if L1 is the lowest so far
 *         w_e = sign(e) max(|e| - 1 / (sqrt|e| beta), 0)     (lp shrinkage, p = 1/2)
 *         z = (sum over the group of q - (t - w_e) * (1/s)) * (1/64);  beta *= hqq_kappa
 *     z := fp16(remembered z); q = clamp(rint(t / s + z), 0, 7)  (as milo_pack)
 * With hqq_iters <= 1 this is exactly milo_pack's round-to-nearest quantiser.
 */

/*
 * milo_hqq_pack -- HQQ-quantise the target t = W - U V and pack it.
 *   W fp16 [N, K] row-major (K % 128 == 0).  U fp16 [N, rank], V fp16
 *   [rank, K] row-major, or rank = 0 and both NULL (t = W).  The target is
 *   formed in fp32 one rank term at a time: t = W, then for p = 0..rank-1
 *   t = t - U[n, p] * V[p, k] (product and difference each rounded to fp32).
 *   packed: the blob of milo_packed_bytes(N, K) bytes (16-byte aligned).
 *   residual: NULL, or f32 [N, K] receiving W - (q - z) s (fp32: the
 *   difference q - z, the product, then W minus it), the residual a
 *   compensator approximates.
 * Errors: K % 128 != 0, rank > 64, N or K above 2^22 or N * K above 2^34 ->
 * UNSUPPORTED_SHAPE; N, K <= 0, rank < 0,
 * hqq_iters outside 0..1000, beta or kappa not finite and positive, NULL W or
 * packed, U or V NULL with rank > 0 -> INVALID_ARG.  Device: NONFINITE for
 * NaN/Inf targets, FP16_RANGE when s or z overflows fp16.  All pointers are
 * caller-owned device memory; stream-ordered, no host synchronisation.
 */
MILO_API milo_status milo_hqq_pack(const uint16_t* W, const uint16_t* U, const uint16_t* V, int32_t rank,
                                   int32_t N, int32_t K, int32_t hqq_iters, float hqq_beta,
                                   float hqq_kappa, void* packed, float* residual, int32_t* dev_status,
                                   void* stream);

typedef struct milo_lorc_params {
    int32_t rank;         /* r: 0..64 */
    int32_t rounds;       /* refinement rounds after the first: 0..16 (ignored when r = 0) */
    int32_t sketch;       /* l: columns of the random test matrix, r <= l <= 128 (r > 0) */
    int32_t power_iters;  /* subspace iterations q: 0..8 */
    int32_t hqq_iters;    /* 0..1000 */
    float hqq_beta;       /* initial shrinkage penalty, finite and > 0 */
    float hqq_kappa;      /* penalty growth per iteration, finite and > 0 */
} milo_lorc_params;

/* Workspace bytes of milo_quantize_lorc for a weight [N, K] (host size_t
 * *bytes); the same shape and parameter errors as milo_quantize_lorc. */
MILO_API milo_status milo_quantize_lorc_workspace(int32_t N, int32_t K, const milo_lorc_params* params,
                                                  size_t* bytes);

/*
 * milo_quantize_lorc -- the offline MiLo quantiser of one weight W fp16
 * [N, K] (K % 128 == 0).  Round 0: HQQ(W) (milo_hqq_pack), R = W - W_hat, and
 * the rank-r compensator of R.  Rounds 1..rounds: HQQ(W - U V) with the fp16
 * U, V of the round before, the new residual and its compensator.
 *
 * Compensator of R [N, K] (randomized subspace iteration, Halko, Martinsson
 * and Tropp 2011): Y = orth(R omega); q times Y = orth(R orth(R^T Y));
 * B = Y^T R; the eigenpairs of B B^T (descending lambda) give sigma_i =
 * sqrt(lambda_i), and, for the top r, U = Y P_r sigma^(1/2) [N, r],
 * V = sigma^(-1/2) P_r^T B [r, K] (a direction with sigma below 1e-12 sigma_0
 * gets zero U and V).  orth() is Cholesky QR (fp64 Gram and Cholesky, fp32
 * products; columns dependent on earlier ones are dropped), once between
 * power steps and twice for the final Y; eigenpairs by cyclic Jacobi in fp64.
 *   omega: f32 [K, sketch] row-major, the random test matrix (an input: the
 *   caller draws it, e.g. standard normal); NULL when r = 0.
 *   packed (milo_packed_bytes), U fp16 [N, r], V fp16 [r, K]: the round with
 *   the lowest error (the first on ties); U, V NULL when r = 0.
 *   err: NULL, or f32 [rounds + 1] (1 when r = 0) receiving each round's
 *   ||W - W_hat - U V||_F (fp16 U, V; accumulated in fp64).
 *   ws: milo_quantize_lorc_workspace bytes, 256-byte aligned, caller-owned;
 *   W must be 8-byte aligned.
 * Errors as milo_hqq_pack, plus: params NULL, rank outside 0..64, rounds,
 * sketch or power_iters out of range, omega / U / V NULL with r > 0, ws too
 * small or unaligned -> INVALID_ARG / WORKSPACE.  Stream-ordered, no host
 * synchronisation; deterministic for fixed inputs.
 */
MILO_API milo_status milo_quantize_lorc(const uint16_t* W, int32_t N, int32_t K,
                                        const milo_lorc_params* params, const float* omega,
                                        void* packed, uint16_t* U, uint16_t* V, float* err, void* ws,
                                        size_t ws_bytes, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------ */
/* Adaptive compensator ranks                                               */
/* ------------------------------------------------------------------------ */
/*
 * "MiLo Algorithm: Mixture of Low-Rank Compensators", adaptive rank
 * selection: a higher rank for weights with a higher kurtosis (strategy 3)
 * and for experts activated more often (strategy 2).
 */

/* Workspace bytes of milo_kurtosis (the same for every size; host size_t
 * *bytes, INVALID_ARG when NULL). */
MILO_API milo_status milo_kurtosis_workspace(size_t* bytes);

/*
 * milo_kurtosis -- Pearson kurtosis m4 / m2^2 (not the excess; a normal
 * distribution gives 3) of the `count` fp16 entries at W (device, 16-byte
 * aligned), from fp64 sums of w, w^2, w^3, w^4 over a fixed grid, written to
 * out[0] (device fp64).  A constant matrix gives 0.  Deterministic.  Device:
 * NONFINITE for NaN/Inf entries.  ws: milo_kurtosis_workspace bytes, 8-byte
 * aligned.
 */
MILO_API milo_status milo_kurtosis(const uint16_t* W, int64_t count, double* out, void* ws, size_t ws_bytes,
                                   int32_t* dev_status, void* stream);

/*
 * milo_assign_ranks -- split a rank budget over n matrices by score (host
 * arrays; a kurtosis, an activation frequency, ...).  Ranks are multiples of
 * 8 in 0..max_rank (max_rank a multiple of 8, at most 64) and add up to at most
 * n * avg_rank: the budget, in units of 8, is shared in proportion to the
 * scores (negative scores count as 0; when no remaining score is positive the
 * rest is shared equally); a share that reaches the cap is fixed there and the
 * rest re-shared among the others; each matrix then takes the floor of its
 * share and the leftover units go one at a time in decreasing order of the
 * fractional part (ties: higher score, then lower index), pass after pass
 * until the budget (capped at n * max_rank) is used.  A higher score never
 * gets a lower rank.  Errors: n <= 0,
 * NULL pointers, non-finite scores, max_rank not a multiple of 8 in 0..64,
 * avg_rank < 0 -> INVALID_ARG.
 */
MILO_API milo_status milo_assign_ranks(const double* score, int32_t n, int32_t avg_rank, int32_t max_rank,
                                       int32_t* ranks);

/* ------------------------------------------------------------------------ */
/* Routing                                                                  */
/* ------------------------------------------------------------------------ */
/*
 * milo_route -- top-k router and expert grouping (histogram, exclusive scan,
 * stable scatter).
 *   logits      fp16 [T, E] (ignored, may be NULL, with MILO_ROUTE_IDS_GIVEN)
 *   topk_ids    int32 [T, k]: output, slot j = j-th largest logit, ties to the
 *               lower expert id; input with MILO_ROUTE_IDS_GIVEN
 *   topk_w      f32 [T, k]: softmax weight exp(l_j - l_max) / sum, the sum over
 *               the k picked experts (MILO_ROUTE_RENORM) or over all E.
 *               Not written with MILO_ROUTE_IDS_GIVEN (may be NULL then).
 *   expert_offsets int32 [E+1]: exclusive scan of the per-expert slot counts
 *   perm        int32 [T*k]: the flat slots f = t*k + j of expert 0 in
 *               ascending order, then expert 1, ...
 *   inv_perm    int32 [T*k]: inv_perm[perm[p]] = p; -1 for a dropped slot
 * Limits: 1 <= E <= MILO_MAX_EXPERTS, 1 <= k <= min(E, MILO_MAX_TOPK), T >= 0,
 * T*k <= MILO_MAX_ROWS (else UNSUPPORTED_SHAPE).
 * Device: BAD_EXPERT_ID (given ids outside [0, E); the slot is dropped),
 * NONFINITE (NaN/Inf logits; ids then unspecified).
 */
MILO_API milo_status milo_route(const uint16_t* logits, int32_t T, int32_t E, int32_t k,
                       uint32_t flags, int32_t* topk_ids, float* topk_w,
                       int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm,
                       int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------ */
/* Quantised projections and layers                                         */
/* ------------------------------------------------------------------------ */

/* One quantised projection W [N, K] with its rank-r compensator (host struct
 * holding device pointers).  rank is a multiple of 8, at most MILO_MAX_RANK;
 * U and V may be NULL when rank == 0.  The compensator is stored in one of two
 * formats ("MiLo Algorithm": the compensators are quantised to 3 bits too):
 *   MILO_LORC_F16   U fp16 [N, r] and V fp16 [r, K], row-major;
 *   MILO_LORC_INT3  U points to the milo_pack blob of U^T [r, N] (groups of 64
 *                   along N; needs N % 128 == 0) and V to the blob of V [r, K]
 *                   (groups of 64 along K), both written by milo_pack. */
#define MILO_LORC_F16 0
#define MILO_LORC_INT3 1
typedef struct milo_qweight {
    const void* packed;     /* blob written by milo_pack */
    const void* U;
    const void* V;
    int32_t rank;
    int32_t lorc_format;    /* MILO_LORC_F16 or MILO_LORC_INT3 */
} milo_qweight;

/* One SwiGLU expert: w1, w3 [I, H] and w2 [H, I]. */
typedef struct milo_expert {
    milo_qweight w1, w3, w2;
} milo_expert;

/* A grouped projection: n_experts weights of the same shape [N, K]. */
typedef struct milo_linear {
    int32_t N, K, n_experts, group;
    int32_t max_rank;       /* set by milo_linear_prepare */
    const void* table;      /* device table written by milo_linear_prepare */
} milo_linear;

/* A SwiGLU MoE layer: experts 0..n_routed-1 are routed, the n_shared experts
 * after them see every token with weight 1. */
typedef struct milo_moe_layer {
    int32_t hidden, inter, n_routed, n_shared, top_k, group;
    int32_t max_rank;       /* set by milo_layer_prepare */
    const void* table;      /* device table written by milo_layer_prepare */
} milo_moe_layer;

/* Bytes of the device table for n projections (64-byte aligned buffer). */
MILO_API milo_status milo_table_bytes(int32_t n_projections, size_t* bytes);

/*
 * milo_linear_prepare / milo_layer_prepare -- validate the weights (host
 * array `weights` / `experts` of device pointers) and write the device table
 * (pointers, shapes and, for an fp16 V, a TMA tensor map of V) to
 * `device_table`, which the caller keeps alive and unmodified while the layer
 * is used; the weights, U and V must stay at the same addresses too (the
 * tensor map holds V's).  One-time set-up: the table is copied with a
 * synchronous cudaMemcpy.  lin/layer are host structs; the caller fills the
 * shape fields and the call sets max_rank and table.
 * Errors: UNSUPPORTED_SHAPE (K % 128, N % 16, K above 2^24, group != 64,
 * rank not a multiple of 8 or above MILO_MAX_RANK, n_experts outside 1..256,
 * top_k outside 1..min(n_routed, 16)), WORKSPACE (table too small or not 64-byte
 * aligned), INVALID_ARG (NULL or misaligned weight pointers, or a tensor map
 * the driver refuses to encode), CUDA (no tensor-map encoder in the driver).
 */
MILO_API milo_status milo_linear_prepare(milo_linear* lin, const milo_qweight* weights,
                                void* device_table, size_t table_bytes);
MILO_API milo_status milo_layer_prepare(milo_moe_layer* layer, const milo_expert* experts,
                               void* device_table, size_t table_bytes);

/* Workspace bytes for milo_grouped_linear / milo_moe_forward over T tokens,
 * for a prepared lin / layer (the size depends on the max_rank that the
 * preparation sets).  UNSUPPORTED_SHAPE for shape fields the preparation
 * would refuse or when the call's rows exceed MILO_MAX_ROWS; INVALID_ARG for
 * a max_rank outside 0..64 or not a multiple of 8.  The size is not monotone
 * in T (the split-K count and the GEMM kernel change with the rows), so a
 * caller reusing one workspace takes the largest size over the T it will
 * call with.  The size depends on which grouped GEMM the call takes (see
 * milo_set_gemm_path: the mma.sync kernel also keeps a plain fp16 copy of the
 * scaled rows and its counters in the workspace), so query it again after
 * changing that setting; a call given less returns MILO_ERR_WORKSPACE. */
MILO_API milo_status milo_linear_workspace_bytes(const milo_linear* lin, int32_t T, int32_t k,
                                        size_t* bytes);
MILO_API milo_status milo_moe_workspace_bytes(const milo_moe_layer* layer, int32_t T, size_t* bytes);

/*
 * Activations (milo_grouped_linear, milo_moe_forward): the GEMMs multiply the
 * int3 codes with FP16 activations (W3A16).  Each activation row (a token's
 * x, or a routed slot's SwiGLU output h) is first multiplied by a power of two
 * 2^a that brings its largest magnitude into [1, 2) and then rounded to fp16;
 * the result is multiplied by 2^-a.  So every fp16 activation, and every bf16
 * one within 2^17 of its row's largest magnitude, enters the product exactly,
 * whatever the row's scale: bf16 rows beyond the fp16 range are accepted too.
 */

/*
 * milo_grouped_linear -- per routed slot, y = x W_e^T + (x V_e^T) U_e^T.
 *   x        [T, K] fp16 or bf16 (x_dt), row-major
 *   expert_offsets, perm  from milo_route over n_experts experts and k slots
 *            per token (perm may be NULL: the identity, x already grouped, k = 1)
 *   y        [T*k, N] in y_dt (F32, F16 or BF16), row f = t*k + j; rows of
 *            dropped slots are written as zeros
 *   ws       >= milo_linear_workspace_bytes(lin, T, k), 256-byte aligned
 * Errors: INVALID_ARG (NULL or misaligned pointers, bad T, k or dtype),
 * UNSUPPORTED_SHAPE (T*k above MILO_MAX_ROWS, N not a multiple of 4),
 * WORKSPACE (ws too small or misaligned).
 * Device: NONFINITE (NaN/Inf in x), FP16_RANGE (an fp16 output or the
 * compensator's fp16 t = x V^T overflows), TIMEOUT.
 */
MILO_API milo_status milo_grouped_linear(const milo_linear* lin, const void* x, milo_dtype x_dt,
                                int32_t T, int32_t k, const int32_t* expert_offsets,
                                const int32_t* perm, void* y, milo_dtype y_dt,
                                void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * milo_moe_forward -- the SwiGLU MoE layer:
 *     h  = fp16( silu(x W1_e^T + LoRC1) * (x W3_e^T + LoRC3) )
 *     y_slot = h W2_e^T + LoRC2
 *     y[t] = sum_j topk_w[t, j] * y_slot[t*k + j]  +  sum_s shared_s(x_t)
 *   x        [T, hidden] fp16 or bf16, row-major
 *   topk_w, expert_offsets, perm, inv_perm  from milo_route (k = layer->top_k)
 *   y        [T, hidden] in y_dt (F32, F16, BF16); the fp16/bf16 outputs are the
 *            round-to-nearest of the f32 result
 *   ws       >= milo_moe_workspace_bytes(layer, T), 256-byte aligned.  The
 *            fp16 SwiGLU activations h [T*k + n_shared*T, inter] sit at byte
 *            offset milo_moe_h_offset(layer, T) of ws after the call, row p =
 *            expert-sorted slot p (shared-expert rows after the routed ones).
 * Errors: INVALID_ARG (NULL or misaligned pointers, T < 0, bad dtype),
 * UNSUPPORTED_SHAPE (T*(top_k + n_shared) above MILO_MAX_ROWS), WORKSPACE.
 * Device: NONFINITE, FP16_RANGE (h, t or an fp16 output overflows), TIMEOUT.
 */
MILO_API milo_status milo_moe_forward(const milo_moe_layer* layer, const void* x, milo_dtype x_dt,
                             int32_t T, const float* topk_w, const int32_t* expert_offsets,
                             const int32_t* perm, const int32_t* inv_perm, void* y,
                             milo_dtype y_dt, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream);

/*
 * milo_grouped_linear_noalloc -- milo_grouped_linear for callers that cannot
 * allocate device memory: code that is handed only its input and output
 * buffers (for example behind a plugin or custom-operator interface with no
 * allocator), or that must not call cudaMalloc on its path because the call
 * can synchronise the device.  This entry point has no counterpart in the
 * paper; it exists only for such callers.
 *
 * Same arguments and results as milo_grouped_linear, without ws / ws_bytes:
 * the scratch lives in a buffer of MILO_NOALLOC_SCRATCH_BYTES compiled into
 * the library, which every GPU that loads the library holds until the process
 * exits.  Nothing here allocates (no cudaMalloc, cudaFree or allocating
 * library routine).
 *   - A call whose scratch need (milo_linear_workspace_bytes for the same
 *     lin, T, k) exceeds MILO_NOALLOC_SCRATCH_BYTES returns MILO_ERR_WORKSPACE
 *     and enqueues nothing; decode-sized calls (tens of rows) fit.
 *   - The first call on each device looks up the buffer's device address
 *     with that device current (cudaGetSymbolAddress) and keeps it for the
 *     life of the process; make that first call before any stream capture,
 *     and do not reset the device (cudaDeviceReset) while the library is
 *     loaded, which would leave the kept address stale.  A failed lookup
 *     returns MILO_ERR_CUDA.
 *   - Every call on a device shares the one buffer and finds the previous
 *     call's contents in it; nothing in it needs to start at zero (each call
 *     writes what it reads).  Calls that overlap on the GPU (other streams,
 *     other threads) race on the buffer: order them on one stream.
 */
#define MILO_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
MILO_API milo_status milo_grouped_linear_noalloc(const milo_linear* lin, const void* x,
                                                 milo_dtype x_dt, int32_t T, int32_t k,
                                                 const int32_t* expert_offsets,
                                                 const int32_t* perm, void* y, milo_dtype y_dt,
                                                 int32_t* dev_status, void* stream);

/* Byte offset of h inside the forward workspace (see milo_moe_forward); 0
 * where milo_moe_workspace_bytes rejects the layer or T. */
MILO_API size_t milo_moe_h_offset(const milo_moe_layer* layer, int32_t T);

/*
 * milo_selftest_wait_timeout -- self-test of the bounded waits: one block
 * waits, with the same bounded wait the GEMM kernels use, on an mbarrier that
 * nothing completes; after the wait limit (about two seconds of SM clock) it
 * ORs MILO_DEV_TIMEOUT into dev_status (device memory, required) and returns.
 * The context stays usable.  Stream-ordered; no host synchronisation.
 */
MILO_API milo_status milo_selftest_wait_timeout(int32_t* dev_status, void* stream);

/*
 * milo_set_gemm_path -- measurement and test hook: which grouped GEMM kernel
 * milo_moe_forward and milo_grouped_linear use.  MILO_GEMM_AUTO: chosen per
 * call from the routed rows per expert (the tcgen05 kernel when they are many,
 * the mma.sync kernel when they are few); MILO_GEMM_MMA / MILO_GEMM_TC force
 * one (both compute the same results within fp32 rounding).  The initial
 * value comes from the environment variable MILO_GEMM ("mma" or "tc"), read
 * once, the first time a call needs it.  Process-wide; applies to calls made
 * after it returns.  Errors: an unknown mode -> INVALID_ARG.
 */
#define MILO_GEMM_AUTO 0
#define MILO_GEMM_MMA 1
#define MILO_GEMM_TC 2
MILO_API milo_status milo_set_gemm_path(int32_t mode);

/*
 * milo_set_profile_events -- measurement hook.  `events` is a host array of n
 * cudaEvent_t (n = 0 or events = NULL disables).  While set, every
 * milo_moe_forward records events[0] / events[1] on its stream right before /
 * after the launch of the w1|w3 grouped GEMM and events[2] / events[3] around
 * the w2 grouped GEMM; milo_grouped_linear records events[0] / events[1] around
 * its grouped GEMM.  The caller owns the events and reads them with
 * cudaEventElapsedTime after the stream completes.  Process-wide setting,
 * not synchronised: change it only while no other host thread is inside the
 * library.
 */
MILO_API milo_status milo_set_profile_events(void* const* events, int32_t n);

#ifdef __cplusplus
}
#endif

#endif /* MILO_H */
