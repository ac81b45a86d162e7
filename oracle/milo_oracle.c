/*
 * milo_oracle.c -- CPU oracle for the int3 + low-rank-compensator MoE forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or constant with the CUDA library, and neither side
 * includes or links the other.
 *
 * Plain, slow and meant to be checked by eye: scalar loops, bit-by-bit
 * packing, fp64 accumulation, one explicit top-k loop per token.  Build with
 * -O2 -ffp-contract=off so that the fp32 steps of the quantiser are the IEEE
 * operations written here (no fused multiply-add).
 *
 * Source: "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
 * Compensators" (MLSys 2025 talk write-up):
 *   - section "MiLo Algorithm: Mixture of Low-Rank Compensators": the output
 *     weight is W_quant + U*V with a rank-R pair (U, V); the rank may differ
 *     per expert ("mixture");
 *   - section "MiLo Kernel: Efficient Int3 Quantized GEMM Backend": int3
 *     weights x FP16 activations, 32 three-bit values held in three 32-bit
 *     words with no wasted bit, asymmetric dequantisation with a zero point;
 *   - sections "Background" / "Experimental Setup & Results": MoE layers route
 *     each token to a subset of experts; activations stay FP16 (W3A16).
 *
 * Readings taken where the pages are silent (each also listed with the
 * design notes of the repository):
 *   - quantiser: round-to-nearest asymmetric min/max per group of 64 along K
 *     (milo_ref_quantize; the paper's HQQ initialisation is milo_ref_hqq
 *     below); s = fp16(range / 7), z = fp16(-min / s), q = clamp(rint(w/s + z));
 *   - dequantisation: w_hat = (q - z) * s with fp16 s and z, z not rounded to
 *     an integer;
 *   - the packing layout (the page's description of the three-word packing is
 *     garbled) is the self-defined layout documented at milo_ref_code_bit();
 *   - compensator orientation: U [N_out, r], V [r, K], y += (x V^T) U^T;
 *   - int3 compensators (the pages quantise U and V to 3 bits too): V is
 *     quantised like a weight, groups of 64 along K; U is quantised
 *     transposed, as U^T [r, N_out] with groups of 64 along N_out (r is at
 *     most 64, and a group along r would not fill the 128-code blocks);
 *   - router: top-k largest logits (ties to the lower expert id), softmax
 *     weights renormalised over the top-k, or taken from the softmax over all
 *     experts when renormalisation is off;
 *   - SwiGLU experts, h = silu(x W1^T) * (x W3^T) rounded to fp16 because
 *     activations are FP16; shared experts have weight 1;
 *   - offline quantiser: HQQ with p = 1/2 shrinkage in fp32, each group keeping
 *     the zero point of lowest L1 error (see milo_ref_hqq()); the compensator
 *     and the refinement rounds are in oracle/__init__.py (numpy, fp64).
 */
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define REF_NONFINITE 2
#define REF_FP16_RANGE 4
#define REF_BAD_EXPERT 1

/* ------------------------------------------------------------------------ */
/* fp16 / bf16 conversion                                                   */
/* ------------------------------------------------------------------------ */

/* Exact value of an IEEE binary16 bit pattern. */
double milo_ref_h2d(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0x1F) {
        v = m ? NAN : INFINITY;
    } else if (e == 0) {
        v = ldexp((double)m, -24);            /* subnormal: m * 2^-24 */
    } else {
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Exact value of a bfloat16 bit pattern (the top half of an fp32). */
double milo_ref_bf2d(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest binary16, ties to even. */
uint16_t milo_ref_d2h(double d) {
    uint16_t sign = signbit(d) ? 0x8000 : 0;
    double a = fabs(d);
    if (isnan(d)) return 0x7E00;
    if (a >= 65520.0) return sign | 0x7C00;    /* rounds past 65504 -> inf */
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: integer multiple of 2^-24 (1024 -> min normal) */
        double m = nearbyint(ldexp(a, 24));
        return sign | (uint16_t)m;
    }
    int ex;
    frexp(a, &ex);                 /* a = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;                /* a in [2^e, 2^(e+1)) */
    double m = nearbyint(ldexp(a, 10 - e));   /* in [1024, 2048] */
    if (m == 2048.0) { m = 1024.0; e += 1; }
    if (e + 15 >= 31) return sign | 0x7C00;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)m - 1024));
}

uint16_t milo_ref_f2h(float f) { return milo_ref_d2h((double)f); }

static float h2f(uint16_t h) { return (float)milo_ref_h2d(h); }

/* ------------------------------------------------------------------------ */
/* quantiser                                                                */
/* ------------------------------------------------------------------------ */

/*
 * Asymmetric round-to-nearest int3 quantisation of W fp16 [N, K] in groups of
 * `group` along K.  Outputs codes q [N, K] (one byte each, 0..7), scale and
 * zero fp16 [K/group, N].  Returns REF_* status bits.
 */
int milo_ref_quantize(const uint16_t* W, int N, int K, int group,
                      uint8_t* q, uint16_t* scale, uint16_t* zero) {
    int status = 0;
    int G = K / group;
    for (int n = 0; n < N; ++n) {
        for (int j = 0; j < G; ++j) {
            const uint16_t* w = W + (size_t)n * K + (size_t)j * group;
            float mn = INFINITY, mx = -INFINITY;
            for (int i = 0; i < group; ++i) {
                float v = h2f(w[i]);
                if (!isfinite(v)) status |= REF_NONFINITE;
                if (v < mn) mn = v;
                if (v > mx) mx = v;
            }
            float range = mx - mn;          /* fp32 subtraction */
            float s_f = range / 7.0f;       /* IEEE fp32 division */
            uint16_t s_h = milo_ref_f2h(s_f);
            if ((s_h & 0x7FFF) == 0) s_h = 0x3C00;   /* degenerate group: s = 1 */
            float s = h2f(s_h);
            float z_f = -mn / s;
            uint16_t z_h = milo_ref_f2h(z_f);
            float z = h2f(z_h);
            if (!isfinite(s) || !isfinite(z)) status |= REF_FP16_RANGE;
            scale[(size_t)j * N + n] = s_h;
            zero[(size_t)j * N + n] = z_h;
            for (int i = 0; i < group; ++i) {
                float v = h2f(w[i]) / s;    /* two separate fp32 ops */
                v = v + z;
                float r = nearbyintf(v);    /* ties to even */
                if (!(r >= 0.0f)) r = 0.0f; /* also maps NaN to 0 */
                if (r > 7.0f) r = 7.0f;
                q[(size_t)n * K + (size_t)j * group + i] = (uint8_t)r;
            }
        }
    }
    return status;
}

/* ------------------------------------------------------------------------ */
/* packing: 32 int3 codes in three 32-bit words                             */
/* ------------------------------------------------------------------------ */

/*
 * Self-defined layout.  A row of K codes (K a multiple of 128) is cut into
 * super-blocks of 128 codes (two scale groups of 64).  Super-block b is held in
 * words 12b .. 12b+11 of the row, as four units of three words.  Unit c (0..3)
 * carries 32 codes u_0..u_31:
 *     u_m = q[128b + 16c + m]              for m = 0..15  (first group)
 *     u_m = q[128b + 64 + 16c + (m - 16)]   for m = 16..31 (second group)
 * Inside the unit, word t (0..2) holds, for i = 0..4,
 *     bits [3i, 3i+3)        = u_{10t + 2i}
 *     bits [16+3i, 16+3i+3)  = u_{10t + 2i + 1}
 * and bit 15 of word t is bit t of u_30, bit 31 of word t is bit t of u_31.
 * All 96 bits are used.
 *
 * milo_ref_code_bit() returns, for code index k of a row and bit beta of that
 * code, the word index within the row and the bit index within the word.
 */
void milo_ref_code_bit(int k, int beta, int* word, int* bit) {
    int b = k / 128, r = k % 128;
    int half = r / 64, rr = r % 64;   /* which group of the super-block */
    int c = rr / 16, m = rr % 16 + 16 * half;
    int t, pos;
    if (m < 30) {
        t = m / 10;
        int within = m % 10;
        pos = 16 * (within % 2) + 3 * (within / 2) + beta;
    } else {
        t = beta;
        pos = (m == 30) ? 15 : 31;
    }
    *word = 12 * b + 3 * c + t;
    *bit = pos;
}

/* Pack codes q [N, K] (values 0..7) into Q [N, 3K/32], bit by bit. */
void milo_ref_pack(const uint8_t* q, int N, int K, uint32_t* Q) {
    int W = 3 * K / 32;
    memset(Q, 0, sizeof(uint32_t) * (size_t)N * W);
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k)
            for (int beta = 0; beta < 3; ++beta) {
                int word, bit;
                milo_ref_code_bit(k, beta, &word, &bit);
                if ((q[(size_t)n * K + k] >> beta) & 1)
                    Q[(size_t)n * W + word] |= (uint32_t)1u << bit;
            }
}

/* Unpack Q [N, 3K/32] into codes q [N, K], bit by bit. */
void milo_ref_unpack(const uint32_t* Q, int N, int K, uint8_t* q) {
    int W = 3 * K / 32;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            int v = 0;
            for (int beta = 0; beta < 3; ++beta) {
                int word, bit;
                milo_ref_code_bit(k, beta, &word, &bit);
                v |= (int)((Q[(size_t)n * W + word] >> bit) & 1u) << beta;
            }
            q[(size_t)n * K + k] = (uint8_t)v;
        }
}

/*
 * Device layout of a packed weight: one byte blob.  Rows are grouped in tiles
 * of 64 (the last tile padded with zero rows); the block of (tile t,
 * super-block b) is contiguous, at byte (t * SB + b) * 3584, and holds
 *     the words of the tile's rows  [64 rows][12]               (3072 B)
 *     then for the super-block's groups 2b and 2b + 1, 256 bytes each: for
 *     each 16-row block m (0..3) and j (0..7) the fp16 quadruple
 *         s[16m + j], z[16m + j], s[16m + j + 8], z[16m + j + 8]
 * so the GPU kernels fetch one or two super-blocks of a tile -- codes, scales
 * and zeros -- with a single copy.  Word j of row n, super-block b, is
 * Q[n, 12 b + j]; s and z of row n, group g are scale[g, n] and zero[g, n].
 * This is a relayout only, used to compare with the device packer.
 */
void milo_ref_tile_pack(const uint32_t* Q, const uint16_t* scale, const uint16_t* zero,
                        int N, int K, uint8_t* blob) {
    int SB = K / 128, W = 3 * K / 32, NT = (N + 63) / 64;
    memset(blob, 0, (size_t)NT * SB * 3584);
    for (int t = 0; t < NT; ++t)
        for (int b = 0; b < SB; ++b) {
            uint8_t* base = blob + ((size_t)t * SB + b) * 3584;
            uint32_t* words = (uint32_t*)base;
            uint16_t* groups = (uint16_t*)(base + 3072);
            for (int r = 0; r < 64; ++r) {
                int n = 64 * t + r;
                if (n >= N) continue;
                for (int j = 0; j < 12; ++j) words[r * 12 + j] = Q[(size_t)n * W + 12 * b + j];
                for (int i = 0; i < 2; ++i) {
                    int g = 2 * b + i;
                    int q = i * 128 + ((r / 16) * 8 + r % 8) * 4 + ((r % 16) / 8) * 2;
                    groups[q] = scale[(size_t)g * N + n];
                    groups[q + 1] = zero[(size_t)g * N + n];
                }
            }
        }
}

/* w_hat[n, k] = (q - z) * s in fp64. */
void milo_ref_dequant(const uint8_t* q, const uint16_t* scale, const uint16_t* zero,
                      int N, int K, int group, double* w_hat) {
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            int j = k / group;
            double s = milo_ref_h2d(scale[(size_t)j * N + n]);
            double z = milo_ref_h2d(zero[(size_t)j * N + n]);
            w_hat[(size_t)n * K + k] = ((double)q[(size_t)n * K + k] - z) * s;
        }
}

/* ------------------------------------------------------------------------ */
/* HQQ: the initial quantisation of the offline MiLo quantiser              */
/* ------------------------------------------------------------------------ */

/*
 * "MiLo Algorithm: Mixture of Low-Rank Compensators", step 1 ("Initial
 * Quantization"): the weights are first quantised with HQQ (half-quadratic
 * quantisation), which needs no calibration data and treats quantisation as
 * an optimisation problem.  The pages give no more detail; HQQ as published
 * (Badri and Shaji, 2023) keeps the min/max scale and fits the zero point z of
 * each group by half-quadratic splitting of an lp error (p < 1):
 *     q      = clamp(rint(t * (1/s) + z), 0, 7)
 *     e      = t - (q - z) s                     the group's error
 *     w_e    = shrink(e)                          proximal step on |.|^p
 *     z_next = mean(q - (t - w_e) * (1/s))        least-squares zero given w_e
 *     beta   = kappa * beta
 * with shrink(e) = sign(e) max(|e| - |e|^(p-1) / beta, 0).
 *
 * Readings (listed with the design notes too):
 *   - p = 1/2, so |e|^(p-1) / beta = 1 / (sqrt(|e|) beta) uses only IEEE
 *     square root and division (HQQ's own default is p = 0.7);
 *   - every step is fp32, in the order written here (no fused multiply-add),
 *     sums run over the group's 64 values in index order; quantised codes are
 *     decided in fp32 on both sides; inside the iterations the target is
 *     multiplied by the fp32 inverse 1/s, as HQQ's quantisation step does;
 *   - HQQ stops when its error stops falling; here each group keeps the zero
 *     point whose L1 error sum_i |e_i| was lowest over the iterations (the
 *     error of a group depends only on its own zero point), first one on ties;
 *   - the kept zero point is rounded to fp16 (the storage format), and the
 *     codes are then re-derived from it exactly as the round-to-nearest
 *     quantiser does, so with one iteration HQQ equals round-to-nearest.
 *
 * hqq_group() quantises one group of 64 fp32 targets t.  z_trace (iters + 1)
 * and err_trace (iters), when not NULL, receive the zero point before each
 * iteration and after the last, and each iteration's L1 error.
 */
static int hqq_group(const float* t, int iters, float beta0, float kappa, uint8_t* q_out,
                     uint16_t* s_out, uint16_t* z_out, float* z_trace, float* err_trace) {
    int status = 0;
    float mn = INFINITY, mx = -INFINITY;
    for (int i = 0; i < 64; ++i) {
        float v = t[i];
        if (!isfinite(v)) status |= REF_NONFINITE;
        if (v < mn) mn = v;
        if (v > mx) mx = v;
    }
    float range = mx - mn;
    uint16_t s_h = milo_ref_f2h(range / 7.0f);
    if ((s_h & 0x7FFF) == 0) s_h = 0x3C00;
    float s = h2f(s_h);
    float z = -mn / s;
    float inv = 1.0f / s;                     /* HQQ quantises with the inverse scale */
    float beta = beta0;
    float best_err = INFINITY, best_z = z;
    if (z_trace) z_trace[0] = z;
    for (int it = 0; it < iters; ++it) {
        float err = 0.0f, acc = 0.0f;
        for (int i = 0; i < 64; ++i) {
            float v = t[i] * inv;
            v = v + z;
            float r = nearbyintf(v);
            if (!(r >= 0.0f)) r = 0.0f;
            if (r > 7.0f) r = 7.0f;
            float wr = r - z;
            wr = wr * s;
            float e = t[i] - wr;
            float a = fabsf(e);
            err = err + a;
            float w_e = 0.0f;                 /* shrink(e), p = 1/2 */
            if (a > 0.0f) {
                float d = sqrtf(a);
                d = d * beta;
                float m = a - 1.0f / d;
                if (m > 0.0f) w_e = e < 0.0f ? -m : m;
            }
            float u = t[i] - w_e;
            u = u * inv;
            acc = acc + (r - u);
        }
        if (err_trace) err_trace[it] = err;
        if (err < best_err) {
            best_err = err;
            best_z = z;
        }
        z = acc * 0.015625f;                  /* mean over 64 values */
        beta = beta * kappa;
        if (z_trace) z_trace[it + 1] = z;
    }
    uint16_t z_h = milo_ref_f2h(best_z);
    float zf = h2f(z_h);
    if (!isfinite(s) || !isfinite(zf)) status |= REF_FP16_RANGE;
    *s_out = s_h;
    *z_out = z_h;
    for (int i = 0; i < 64; ++i) {
        float v = t[i] / s;
        v = v + zf;
        float r = nearbyintf(v);
        if (!(r >= 0.0f)) r = 0.0f;
        if (r > 7.0f) r = 7.0f;
        q_out[i] = (uint8_t)r;
    }
    return status;
}

static int default_threads(int nthreads);

typedef struct {
    const float* T;
    int N, K, iters, n0, n1, status;
    float beta0, kappa;
    uint8_t* q;
    uint16_t* scale;
    uint16_t* zero;
} hqq_job;

static void* hqq_rows(void* arg) {
    hqq_job* J = arg;
    int G = J->K / 64;
    J->status = 0;
    for (int n = J->n0; n < J->n1; ++n)
        for (int j = 0; j < G; ++j) {
            size_t at = (size_t)n * J->K + (size_t)j * 64, sz = (size_t)j * J->N + n;
            J->status |= hqq_group(J->T + at, J->iters, J->beta0, J->kappa, J->q + at, J->scale + sz,
                                   J->zero + sz, NULL, NULL);
        }
    return NULL;
}

/*
 * HQQ quantisation of an fp32 target T [N, K] (K a multiple of 64) in groups
 * of 64 along K.  Outputs as milo_ref_quantize(): codes q [N, K], scale and
 * zero fp16 [K/64, N].  Rows are split over `nthreads` threads (<= 0: every
 * core this process may use); groups are independent, so the result does not depend on
 * the thread count.  Returns REF_* status bits.
 */
int milo_ref_hqq(const float* T, int N, int K, int iters, float beta0, float kappa,
                 uint8_t* q, uint16_t* scale, uint16_t* zero, int nthreads) {
    int nt = default_threads(nthreads);
    if (nt > N) nt = N > 0 ? N : 1;
    hqq_job* jobs = calloc((size_t)nt, sizeof(hqq_job));
    pthread_t* th = calloc((size_t)nt, sizeof(pthread_t));
    for (int t = 0; t < nt; ++t) {
        jobs[t] = (hqq_job){T, N, K, iters, (int)((long long)N * t / nt), (int)((long long)N * (t + 1) / nt), 0,
                            beta0, kappa, q, scale, zero};
        if (nt > 1) pthread_create(&th[t], NULL, hqq_rows, &jobs[t]);
    }
    if (nt == 1) hqq_rows(&jobs[0]);
    int status = 0;
    for (int t = 0; t < nt; ++t) {
        if (nt > 1) pthread_join(th[t], NULL);
        status |= jobs[t].status;
    }
    free(jobs);
    free(th);
    return status;
}

/* One group with its zero-point and error trajectory (for the pins). */
int milo_ref_hqq_trace(const float* t, int iters, float beta0, float kappa, uint8_t* q,
                       uint16_t* s, uint16_t* z, float* z_trace, float* err_trace) {
    return hqq_group(t, iters, beta0, kappa, q, s, z, z_trace, err_trace);
}

/* ------------------------------------------------------------------------ */
/* routing                                                                  */
/* ------------------------------------------------------------------------ */

/*
 * Group routed slots by expert.  ids [T*k] (flat slot f = t*k + j).  Writes
 * offsets [E+1] (exclusive scan of the per-expert counts), perm [T*k] (the
 * flat slots of expert 0 in ascending order, then expert 1, ...) and
 * inv_perm [T*k] (inv_perm[perm[p]] = p).  Returns REF_BAD_EXPERT when an id
 * is outside [0, E); such slots are left out of every group.
 */
int milo_ref_group(const int32_t* ids, int T, int k, int E,
                   int32_t* offsets, int32_t* perm, int32_t* inv_perm) {
    int status = 0, F = T * k;
    int32_t* count = calloc((size_t)E, sizeof(int32_t));
    for (int f = 0; f < F; ++f) {
        if (ids[f] < 0 || ids[f] >= E) { status |= REF_BAD_EXPERT; continue; }
        count[ids[f]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + count[e];
    for (int e = 0; e < E; ++e) count[e] = 0;
    for (int f = 0; f < F; ++f) inv_perm[f] = -1;
    for (int f = 0; f < F; ++f) {
        int e = ids[f];
        if (e < 0 || e >= E) continue;
        int p = offsets[e] + count[e]++;
        perm[p] = f;
        inv_perm[f] = p;
    }
    free(count);
    return status;
}

/*
 * Top-k softmax router over fp16 logits [T, E].  For each token the k largest
 * logits are picked one at a time (ties go to the lower expert id), so slot j
 * holds the j-th largest.  Weights: exp(l_j - l_max) divided by the sum over
 * the k picked experts (renorm != 0) or over all E experts (renorm == 0), in
 * fp64.  Then groups the slots as milo_ref_group().
 */
int milo_ref_route(const uint16_t* logits, int T, int E, int k, int renorm,
                   int32_t* ids, double* w, int32_t* offsets, int32_t* perm,
                   int32_t* inv_perm) {
    int status = 0;
    char* chosen = malloc((size_t)E);
    for (int t = 0; t < T; ++t) {
        const uint16_t* l = logits + (size_t)t * E;
        for (int e = 0; e < E; ++e)
            if (!isfinite(milo_ref_h2d(l[e]))) status |= REF_NONFINITE;
        memset(chosen, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (chosen[e]) continue;
                if (best < 0 || milo_ref_h2d(l[e]) > milo_ref_h2d(l[best])) best = e;
            }
            chosen[best] = 1;
            ids[(size_t)t * k + j] = best;
        }
        double lmax = milo_ref_h2d(l[ids[(size_t)t * k]]);
        double denom = 0.0;
        if (renorm) {
            for (int j = 0; j < k; ++j) denom += exp(milo_ref_h2d(l[ids[(size_t)t * k + j]]) - lmax);
        } else {
            for (int e = 0; e < E; ++e) denom += exp(milo_ref_h2d(l[e]) - lmax);
        }
        for (int j = 0; j < k; ++j)
            w[(size_t)t * k + j] = exp(milo_ref_h2d(l[ids[(size_t)t * k + j]]) - lmax) / denom;
    }
    free(chosen);
    return status | milo_ref_group(ids, T, k, E, offsets, perm, inv_perm);
}

/* ------------------------------------------------------------------------ */
/* linear: y = x * w_hat^T + (x * V^T) * U^T                                */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint32_t* Q;      /* packed codes [N, 3K/32] */
    const uint16_t* scale;  /* fp16 [K/group, N] */
    const uint16_t* zero;   /* fp16 [K/group, N] */
    const uint16_t* U;      /* fp16 [N, rank] (unused when Uq is set) */
    const uint16_t* V;      /* fp16 [rank, K] (unused when Uq is set) */
    int32_t rank;
    /* int3 compensator, optional: U^T packed [rank, 3N/32] with scale and zero
       [N/group, rank]; V packed [rank, 3K/32] with scale and zero [K/group, rank] */
    const uint32_t* Uq;
    const uint16_t* Us;
    const uint16_t* Uz;
    const uint32_t* Vq;
    const uint16_t* Vs;
    const uint16_t* Vz;
} milo_ref_proj;

/* Row p of a packed matrix [R, C] (groups of `group` along C), dequantised
   into out [C] in fp64 with the scalar unpack. */
static void dequant_row(const uint32_t* Qm, const uint16_t* sc, const uint16_t* ze, int R, int Cc, int group,
                        int p, double* out) {
    uint8_t* codes = malloc((size_t)Cc);
    milo_ref_unpack(Qm + (size_t)p * (3 * Cc / 32), 1, Cc, codes);
    for (int c = 0; c < Cc; ++c) {
        int j = c / group;
        double s = milo_ref_h2d(sc[(size_t)j * R + p]);
        double z = milo_ref_h2d(ze[(size_t)j * R + p]);
        out[c] = ((double)codes[c] - z) * s;
    }
    free(codes);
}

typedef struct {
    const double* X; int M, K, N, group;
    const milo_ref_proj* P;
    const double* t;         /* [M, rank] = X V^T */
    const double* Ud;        /* [N, rank] compensator U, fp64 */
    double* Y;               /* [M, N] */
    int n0, n1;
} linear_job;

static void* linear_rows(void* arg) {
    linear_job* J = arg;
    int K = J->K, W = 3 * K / 32, r = J->P->rank;
    uint8_t* codes = malloc((size_t)K);
    double* wrow = malloc(sizeof(double) * (size_t)K);
    for (int n = J->n0; n < J->n1; ++n) {
        /* scalar unpack and dequantisation of row n */
        milo_ref_unpack(J->P->Q + (size_t)n * W, 1, K, codes);
        for (int j = 0; j < K / J->group; ++j) {
            double s = milo_ref_h2d(J->P->scale[(size_t)j * J->N + n]);
            double z = milo_ref_h2d(J->P->zero[(size_t)j * J->N + n]);
            for (int k = j * J->group; k < (j + 1) * J->group; ++k)
                wrow[k] = ((double)codes[k] - z) * s;
        }
        for (int m = 0; m < J->M; ++m) {
            const double* x = J->X + (size_t)m * K;
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += x[k] * wrow[k];
            double lorc = 0.0;
            for (int p = 0; p < r; ++p)
                lorc += J->t[(size_t)m * r + p] * J->Ud[(size_t)n * r + p];
            J->Y[(size_t)m * J->N + n] = acc + lorc;
        }
    }
    free(codes);
    free(wrow);
    return NULL;
}

/* nthreads > 0 as given; else the cores this process may run on. */
static int default_threads(int nthreads) {
    if (nthreads > 0) return nthreads;
    cpu_set_t set;
    if (sched_getaffinity(0, sizeof(set), &set) == 0 && CPU_COUNT(&set) > 0) return CPU_COUNT(&set);
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    return c > 0 ? (int)c : 1;
}

/*
 * Y [M, N] = X [M, K] * w_hat^T + (X V^T) U^T, all in fp64, where w_hat is the
 * dequantised packed weight of P.  Rows n are split over `nthreads` threads
 * (<= 0: every core this process may use); each output is produced by one thread in a fixed
 * order, so the result does not depend on the thread count.
 */
void milo_ref_linear(const double* X, int M, int K, const milo_ref_proj* P, int N,
                     int group, double* Y, int nthreads) {
    int r = P->rank;
    /* the compensator in fp64: fp16 values, or the dequantised int3 codes */
    double* Vd = calloc((size_t)(r > 0 ? r : 1) * K, sizeof(double));
    double* Ud = calloc((size_t)N * (r > 0 ? r : 1), sizeof(double));
    double* urow = malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    for (int p = 0; p < r; ++p) {
        if (P->Uq) {
            dequant_row(P->Vq, P->Vs, P->Vz, r, K, group, p, Vd + (size_t)p * K);
            dequant_row(P->Uq, P->Us, P->Uz, r, N, group, p, urow);
            for (int n = 0; n < N; ++n) Ud[(size_t)n * r + p] = urow[n];
        } else {
            for (int k = 0; k < K; ++k) Vd[(size_t)p * K + k] = milo_ref_h2d(P->V[(size_t)p * K + k]);
            for (int n = 0; n < N; ++n) Ud[(size_t)n * r + p] = milo_ref_h2d(P->U[(size_t)n * r + p]);
        }
    }
    free(urow);
    double* t = calloc((size_t)M * (r > 0 ? r : 1), sizeof(double));
    for (int m = 0; m < M; ++m)
        for (int p = 0; p < r; ++p) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += X[(size_t)m * K + k] * Vd[(size_t)p * K + k];
            t[(size_t)m * r + p] = acc;
        }
    int nt = default_threads(nthreads);
    if (nt > N) nt = N > 0 ? N : 1;
    pthread_t* th = malloc(sizeof(pthread_t) * (size_t)nt);
    linear_job* jobs = malloc(sizeof(linear_job) * (size_t)nt);
    for (int i = 0; i < nt; ++i) {
        jobs[i] = (linear_job){X, M, K, N, group, P, t, Ud, Y,
                               (int)((long)N * i / nt), (int)((long)N * (i + 1) / nt)};
        pthread_create(&th[i], NULL, linear_rows, &jobs[i]);
    }
    for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
    free(th);
    free(jobs);
    free(t);
    free(Vd);
    free(Ud);
}

/* silu(a) = a / (1 + e^-a), in fp64. */
double milo_ref_silu(double a) { return a / (1.0 + exp(-a)); }

/* ------------------------------------------------------------------------ */
/* MoE layer                                                                */
/* ------------------------------------------------------------------------ */

/*
 * SwiGLU expert on the rows X [M, H]: a = X W1^T (+LoRC), b = X W3^T (+LoRC),
 * h = fp16(silu(a) * b), y = h W2^T (+LoRC).  h_bits [M, I] receives the fp16
 * activations, y [M, H] the fp64 outputs.  Returns NONFINITE when a product
 * silu(a) * b is not finite, FP16_RANGE when a finite one rounds to an fp16
 * infinity (h is an fp16 tensor).
 */
static int expert_forward(const double* X, int M, int H, int I, int group,
                          const milo_ref_proj* w1, const milo_ref_proj* w3,
                          const milo_ref_proj* w2, uint16_t* h_bits, double* y,
                          int nthreads) {
    int status = 0;
    double* a = malloc(sizeof(double) * (size_t)M * I);
    double* b = malloc(sizeof(double) * (size_t)M * I);
    double* h = malloc(sizeof(double) * (size_t)M * I);
    milo_ref_linear(X, M, H, w1, I, group, a, nthreads);
    milo_ref_linear(X, M, H, w3, I, group, b, nthreads);
    for (size_t i = 0; i < (size_t)M * I; ++i) {
        double v = milo_ref_silu(a[i]) * b[i];
        h_bits[i] = milo_ref_d2h(v);
        h[i] = milo_ref_h2d(h_bits[i]);
        if (!isfinite(v)) status |= REF_NONFINITE;
        else if (!isfinite(h[i])) status |= REF_FP16_RANGE;
    }
    milo_ref_linear(h, M, I, w2, H, group, y, nthreads);
    free(a);
    free(b);
    free(h);
    return status;
}

/*
 * Full layer.  x [T, H] raw 16-bit (bf16 when x_is_bf16, else fp16), routed
 * experts 0..E-1 with ids/w [T*k] from the router, shared experts E..E+S-1
 * applied to every token with weight 1.  w1/w3/w2 hold E+S projections each.
 *
 *   y[t] = sum_j w[t,j] * expert_{ids[t,j]}(x_t)   (slots in order j = 0..k-1)
 *        + sum_s expert_{E+s}(x_t)                  (shared experts in order)
 *
 * y [T, H] fp64.  h_bits (optional) receives the fp16 SwiGLU activations,
 * indexed by flat slot f = t*k + j for [0, T*k) and then T*k + s*T + t for the
 * shared experts; it must hold (T*k + S*T) * I entries.
 */
int milo_ref_moe_forward(const uint16_t* x, int x_is_bf16, int T, int H, int I,
                         int E, int S, int k, int group,
                         const int32_t* ids, const double* w,
                         const milo_ref_proj* w1, const milo_ref_proj* w3,
                         const milo_ref_proj* w2, double* y, uint16_t* h_bits,
                         int nthreads) {
    int status = 0, F = T * k;
    double* X = malloc(sizeof(double) * (size_t)T * H);
    for (size_t i = 0; i < (size_t)T * H; ++i) {
        X[i] = x_is_bf16 ? milo_ref_bf2d(x[i]) : milo_ref_h2d(x[i]);
        if (!isfinite(X[i])) status |= REF_NONFINITE;
    }
    double* y_slot = calloc((size_t)(F > 0 ? F : 1) * H, sizeof(double));
    double* y_sh = calloc((size_t)(S > 0 ? S : 1) * T * H, sizeof(double));
    size_t rows_max = (size_t)(F > T ? F : T) + 1;
    uint16_t* h_tmp = malloc(sizeof(uint16_t) * rows_max * I);
    double* Xe = malloc(sizeof(double) * rows_max * H);
    double* ye = malloc(sizeof(double) * rows_max * H);
    int* rows = malloc(sizeof(int) * (size_t)(F > 0 ? F : 1));
    for (int e = 0; e < E; ++e) {
        /* the slots routed to expert e, in ascending flat order */
        int M = 0;
        for (int f = 0; f < F; ++f) {
            if (ids[f] < 0 || ids[f] >= E) { status |= REF_BAD_EXPERT; continue; }
            if (ids[f] == e) rows[M++] = f;
        }
        if (M == 0) continue;
        for (int m = 0; m < M; ++m)
            memcpy(Xe + (size_t)m * H, X + (size_t)(rows[m] / k) * H, sizeof(double) * H);
        status |= expert_forward(Xe, M, H, I, group, &w1[e], &w3[e], &w2[e], h_tmp, ye, nthreads);
        for (int m = 0; m < M; ++m) {
            memcpy(y_slot + (size_t)rows[m] * H, ye + (size_t)m * H, sizeof(double) * H);
            if (h_bits)
                memcpy(h_bits + (size_t)rows[m] * I, h_tmp + (size_t)m * I, sizeof(uint16_t) * I);
        }
    }
    for (int s = 0; s < S; ++s) {
        status |= expert_forward(X, T, H, I, group, &w1[E + s], &w3[E + s], &w2[E + s], h_tmp,
                                 y_sh + (size_t)s * T * H, nthreads);
        if (h_bits)
            memcpy(h_bits + ((size_t)F + (size_t)s * T) * I, h_tmp, sizeof(uint16_t) * T * I);
    }
    for (int t = 0; t < T; ++t)
        for (int n = 0; n < H; ++n) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                int f = t * k + j;
                if (ids[f] < 0 || ids[f] >= E) continue;
                acc += w[f] * y_slot[(size_t)f * H + n];
            }
            for (int s = 0; s < S; ++s) acc += y_sh[((size_t)s * T + t) * H + n];
            y[(size_t)t * H + n] = acc;
        }
    free(X); free(y_slot); free(y_sh); free(h_tmp); free(Xe); free(ye); free(rows);
    return status;
}
