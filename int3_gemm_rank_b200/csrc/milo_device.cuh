// milo_device.cuh -- device helpers shared by the sm_100a kernels of libmilo.
//
// PTX wrappers (mbarrier, 1-D bulk copies, mma.sync), the int3 field
// extraction of the packing format and its register schedule, and small
// conversions.  Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/milo.h"

namespace milo {

// ---------------------------------------------------------------------------
// status
// ---------------------------------------------------------------------------

__device__ __forceinline__ void flag(int32_t* st, int32_t bits) {
    if (st != nullptr && bits) atomicOr(st, bits);
}

// Range checks of the checked build (MILO_CHECKED): in_range(st, cond) is
// true when cond holds; otherwise it flags MILO_DEV_BOUNDS and returns false,
// and the caller skips the access.  In the normal build it is always true and
// costs nothing.
#ifdef MILO_CHECKED
__device__ __forceinline__ bool in_range(int32_t* st, bool cond) {
    if (!cond) flag(st, MILO_DEV_BOUNDS);
    return cond;
}
#else
__device__ __forceinline__ constexpr bool in_range(int32_t*, bool) { return true; }
#endif

// ---------------------------------------------------------------------------
// programmatic dependent launch
// ---------------------------------------------------------------------------

// The kernels of a forward are launched with programmatic stream
// serialization: a kernel may be scheduled while the previous one drains.
// grid_dep_wait() returns once the grids it depends on have completed and
// their writes are visible (at once for a normal launch); every kernel calls
// it before touching what earlier kernels wrote, so completion stays
// transitive along the stream.  grid_dep_launch() lets the next kernel start
// launching.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// conversions
// ---------------------------------------------------------------------------

// Activation element (fp16 or bf16 bits) as f32, exactly.
__device__ __forceinline__ float act_f32(uint16_t bits, bool is_bf16) {
    return is_bf16 ? __uint_as_float(static_cast<uint32_t>(bits) << 16) : __half2float(__ushort_as_half(bits));
}

// Activation element times its row's scale 2^a, rounded to fp16 (nearest
// even).  The product is exact in f32; the rounding keeps every bit of an
// fp16 or bf16 element down to 2^-17 of the row's largest magnitude, and the
// scaled values are below 2 (FP16_RANGE guards a scale that does not match).
__device__ __forceinline__ __half to_half_scaled(uint16_t bits, bool is_bf16, float scale, int32_t& st) {
    const float f = act_f32(bits, is_bf16) * scale;
    if (!isfinite(f)) st |= MILO_DEV_NONFINITE;
    else if (fabsf(f) > 65504.0f) st |= MILO_DEV_FP16_RANGE;
    return __float2half_rn(f);
}

// The row scale 2^a for a row whose largest magnitude is `mx` (f32 bits of a
// non-negative value): max * 2^a in [1, 2), a clamped to [-126, 126] so that
// 2^a and 2^-a are normal floats; 1 for a zero or non-finite maximum.
__device__ __forceinline__ float row_scale_for(uint32_t mx_bits) {
    if (mx_bits == 0u || mx_bits >= 0x7F800000u) return 1.0f;
    int a = 127 - static_cast<int>(mx_bits >> 23);     // a subnormal maximum (exponent field 0) clamps
    a = a < -126 ? -126 : (a > 126 ? 126 : a);
    return __uint_as_float(static_cast<uint32_t>(127 + a) << 23);
}

// 2^-a from 2^a (both normal powers of two): exact.
__device__ __forceinline__ float inv_pow2(float s) {
    return __uint_as_float(0x7F000000u - __float_as_uint(s));
}

// Four packed activation pairs times their row's scale, as fp16 pairs.
__device__ __forceinline__ uint4 scaled_pairs(uint4 v, bool bf16, float scale, int32_t& st) {
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __half lo = to_half_scaled(static_cast<uint16_t>(w[q] & 0xFFFFu), bf16, scale, st);
        const __half hi = to_half_scaled(static_cast<uint16_t>(w[q] >> 16), bf16, scale, st);
        w[q] = static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// A compensator value t rounded to fp16 (FP16_RANGE if it overflows).
__device__ __forceinline__ uint16_t t_half(float v, int32_t& st) {
    const __half h = __float2half_rn(v);
    if (__hisinf(h)) st |= MILO_DEV_FP16_RANGE;
    return __half_as_ushort(h);
}

// ---------------------------------------------------------------------------
// int3 format: field extraction
// ---------------------------------------------------------------------------
//
// A word holds five 3-bit fields in each 16-bit half (bits 3i..3i+2 and
// 16+3i..16+3i+2, i = 0..4) plus one spare bit per half (bits 15 and 31).
// Masking a field that lies in bits 0..8 of a half leaves an fp16 whose value
// is code * 8^i * 2^-24 (fields 0, 1, 2: the pattern is an integer below 2^11,
// and fp16 patterns below 2^11 are that integer times 2^-24).  Fields 3 and 4
// and the spare bit of word t are brought down by one shift of 9 - t, so they
// land t bits higher than fields 0 and 1 do.  Each pair of codes costs one
// LOP3 (plus one shift per word) and the power-of-2 factor left in the value
// is undone on the activation side, where it costs nothing per weight.  The
// six spare bits of a unit (bit t of u_30 in bit 15 of word t, bit t of u_31
// in bit 31) arrive at bits 6 + t / 22 + t of the shifted words, so three
// LOP3s gather them into one more register: u_30 * 64 and u_31 * 64 in the
// fp16 halves.
constexpr uint32_t kField0 = 0x00070007u;   // bits 0-2   -> code * 1
constexpr uint32_t kField1 = 0x00380038u;   // bits 3-5   -> code * 8
constexpr uint32_t kField2 = 0x01C001C0u;   // bits 6-8   -> code * 64
constexpr uint32_t kSpare = 0x00400040u;    // bit 15 >> 9 -> bit 6 (bit 31 >> 9 -> bit 22)

// Shift that brings fields 3, 4 and the spare bit of word t down.
__host__ __device__ constexpr int word_shift(int t) { return 9 - t; }

// Register f (0..5) of a unit; w[] are its three words, hw[t] = w[t] >>
// word_shift(t).  Fields 0..4 come from word t; register 5 gathers the spare
// bits.
template <int T, int F>
__device__ __forceinline__ uint32_t unit_reg(const uint32_t (&w)[3], const uint32_t (&hw)[3]) {
    if constexpr (F == 0) return w[T] & kField0;
    else if constexpr (F == 1) return w[T] & kField1;
    else if constexpr (F == 2) return w[T] & kField2;
    else if constexpr (F == 3) return hw[T] & (kField0 << T);
    else if constexpr (F == 4) return hw[T] & (kField1 << T);
    else return (hw[0] & kSpare) | (hw[1] & (kSpare << 1)) | (hw[2] & (kSpare << 2));
}

// Register schedule of one 3-word unit over the eight k16 MMA steps of a
// 128-code super-block.  Step s uses register (sched_word, sched_field)[s][0]
// for A-fragment slots (2c, 2c+1) and [s][1] for slots (2c+8, 2c+9).  Steps
// 0..3 cover the first scale group (unit codes u_0..u_15), steps 4..7 the
// second (u_16..u_31).  Field 5 is the gathered spare register (word unused).
__host__ __device__ constexpr int sched_word(int s, int h) {
    constexpr int w[8][2] = {{0, 0}, {0, 0}, {0, 1}, {1, 1}, {1, 1}, {2, 2}, {2, 2}, {2, 0}};
    return w[s][h];
}
__host__ __device__ constexpr int sched_field(int s, int h) {
    constexpr int f[8][2] = {{0, 1}, {2, 3}, {4, 0}, {1, 2}, {3, 4}, {0, 1}, {2, 3}, {4, 5}};
    return f[s][h];
}
constexpr int kSteps = 8;
// Unit code index of the low half of register (word t, field f); the high
// half holds the next code.  The spare register holds u_30 (low), u_31 (high).
__host__ __device__ constexpr int reg_code(int t, int f) { return f < 5 ? 10 * t + 2 * f : 30; }
// Offset inside the 128-code super-block of unit code m of unit c.
__host__ __device__ constexpr int unit_k(int c, int m) {
    return m < 16 ? 16 * c + m : 64 + 16 * c + (m - 16);
}
// Power of 2 left in the extracted value of register (word t, field f), 2^e
// with e <= 6, and the factor 2^(6 - e) >= 1 that multiplies the activation
// paired with it, so that every product carries the same 2^6 (undone with
// the 2^-24 of the fp16 pattern by kFoldScale = 2^18).  Scaling up keeps
// fp16 activations exact, subnormal ones included.
__host__ __device__ constexpr int field_shift(int t, int f) {
    return f == 0 ? 0 : f == 1 ? 3 : f == 2 ? 6 : f == 3 ? t : f == 4 ? 3 + t : 6;
}
__host__ __device__ constexpr float act_scale(int t, int f) {
    return static_cast<float>(1 << (6 - field_shift(t, f)));
}

// ---------------------------------------------------------------------------
// int3 compensator blobs (one 64-row tile: U^T [r][N] or V [r][K], r <= 64)
// ---------------------------------------------------------------------------

// A blob block (one 64-row tile, one 128-code super-block): the rows' words
// [64][12] u32, then the two groups' (s, z) pairs, 256 bytes each.
constexpr int kBlobBlockBytes = 64 * 12 * 4 + 2 * 256;
constexpr int kBlobWordBytes = 64 * 12 * 4;
constexpr int kBlobGroupBytes = 256;

// Byte offset of row j's three words of unit u of super-block b.  Unit u
// holds the 16 codes at positions 16u..16u+15 of the super-block's first
// group (codes 0..15 of the unit) and the 16 at 64+16u.. of its second
// (codes 16..31).
__device__ __forceinline__ int lorc_words_off(int j, int b, int u) { return b * kBlobBlockBytes + j * 48 + 12 * u; }

// Unit and code index of position k (0..127) of a super-block.
__device__ __forceinline__ int blob_unit(int k) { return (k & 63) >> 4; }
__device__ __forceinline__ int blob_code(int k) { return (k & 15) + 16 * (k >> 6); }

// Byte offset of row j's (s, z) fp16 pair for group g (64 codes along the row).
__device__ __forceinline__ int lorc_sz_off(int j, int g) {
    return (g >> 1) * kBlobBlockBytes + kBlobWordBytes + (g & 1) * kBlobGroupBytes +
           (((j >> 4) * 8 + (j & 7)) * 4 + ((j >> 3) & 1) * 2) * 2;
}

// Code i (0..31) of a unit's three words: pair p = i / 2 < 15 sits in bits
// 3 (p % 5) (+16 for the odd code) of word p / 5; codes 30 and 31 take bit t
// from bits 15 and 31 of word t.
__device__ __forceinline__ uint32_t unit_code(const uint32_t (&w)[3], int i) {
    if (i < 30) {
        const int p = i >> 1;
        const uint32_t word = p < 5 ? w[0] : p < 10 ? w[1] : w[2];
        return (word >> (3 * (p % 5) + 16 * (i & 1))) & 7u;
    }
    const int sh = i == 30 ? 15 : 31;
    return ((w[0] >> sh) & 1u) | (((w[1] >> sh) & 1u) << 1) | (((w[2] >> sh) & 1u) << 2);
}

// The 16 values (q - z) * s of one group's half of a unit (codes 16 h ..
// 16 h + 15, h = which group) as 8 fp16 pairs, in position order.
__device__ __forceinline__ void unit_half_dequant(const uint32_t (&w)[3], int h, float s, float z,
                                                  uint32_t (&out)[8]) {
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const float lo = (static_cast<float>(unit_code(w, 16 * h + 2 * m)) - z) * s;
        const float hi = (static_cast<float>(unit_code(w, 16 * h + 2 * m + 1)) - z) * s;
        out[m] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(lo))) |
                 (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(hi))) << 16);
    }
}

__device__ __forceinline__ float sz_scale(uint32_t sz) { return __half2float(__ushort_as_half(static_cast<uint16_t>(sz & 0xFFFFu))); }
__device__ __forceinline__ float sz_zero(uint32_t sz) { return __half2float(__ushort_as_half(static_cast<uint16_t>(sz >> 16))); }

// ---------------------------------------------------------------------------
// PTX: mbarrier
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait: gives up after about two seconds of SM clock (the caller then
// flags MILO_DEV_TIMEOUT and unwinds), however long each try_wait suspends.
constexpr long long kWaitCycles = 4000000000LL;

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

// True in one lane of a converged warp (the same lane every time).
__device__ __forceinline__ bool elect_one() {
    uint32_t e;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(e));
    return e != 0;
}

// The same, decided for the whole warp: every lane returns the same answer,
// so the warp never splits on a timeout ahead of a warp-collective step.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity));
}

// ---------------------------------------------------------------------------
// PTX: bulk copies (TMA engine, 1-D; no multicast anywhere in this library)
// ---------------------------------------------------------------------------

// L2 policy for data read once per launch (packed weights): evict first, so
// that activations and partial sums stay resident.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Copy `bytes` contiguous bytes global -> this CTA's shared memory; the
// mbarrier's transaction count receives them.  Both addresses 16-byte
// aligned, `bytes` a positive multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// 2-D tiled TMA load (no multicast): box of the tensor map at (x, y).  The
// innermost coordinate x times the element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                            int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void bulk_load_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                               uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy) : "memory");
}

// Four 8x8 b16 matrices from shared memory: lane l gives the address of row
// l % 8 of matrix l / 8; lane t receives, of each matrix, row t / 4, elements
// 2 (t % 4) and 2 (t % 4) + 1.
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_u32(p)));
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a tile of
// 128-byte rows written by TMA with the 128-byte swizzle (tile base 1024-byte
// aligned): the chunk index is XORed with the row index modulo 8.
__device__ __forceinline__ uint32_t swz128(int row, int chunk) {
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------------------
// PTX: warp-level MMA  D[16x8] (+)= A[16x16] * B[16x8], fp16 in, fp32 accumulate
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma16816_zc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
    float z = 0.0f;
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

}  // namespace milo
