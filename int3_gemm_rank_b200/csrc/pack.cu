// pack.cu -- int3 quantise + pack, and the field-extraction unpack.
//
// "MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
// Compensators", section "MiLo Kernel: Efficient Int3 Quantized GEMM Backend":
// 32 three-bit values per three 32-bit words, no wasted bit, asymmetric
// dequantisation with a zero point.  The quantiser here is round-to-nearest
// asymmetric min/max; the paper's HQQ initialisation is in quant.cu.
#include <cuda_runtime.h>

#include "milo_blob.cuh"
#include "milo_device.cuh"
#include "milo_host.h"
#include "milo_kernels.h"

namespace milo {

// One thread per (row, 128-code super-block): two scale groups.  Rows N..
// of the last tile get zero words, scales and zeros.
__global__ void __launch_bounds__(128) pack_kernel(const uint16_t* __restrict__ W, int N, int K,
                                                   uint8_t* __restrict__ blob,
                                                   int32_t* __restrict__ dev_status) {
    const int SB = K / 128;
    const int Npad = (N + 63) / 64 * 64;
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid >= static_cast<long long>(Npad) * SB) return;
    const int n = static_cast<int>(gid / SB);
    const int b = static_cast<int>(gid % SB);
    if (n >= N) {
        blob_zero_row(blob, n, b, SB);
        return;
    }
    const uint16_t* w = W + static_cast<size_t>(n) * K + static_cast<size_t>(b) * 128;

    int32_t st = 0;
    uint8_t q[128];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        float mn = INFINITY, mx = -INFINITY;
        for (int i = 0; i < 64; ++i) {
            const float v = __half2float(__ushort_as_half(w[64 * g + i]));
            if (!isfinite(v)) st |= MILO_DEV_NONFINITE;
            if (v < mn) mn = v;
            if (v > mx) mx = v;
        }
        const float range = __fsub_rn(mx, mn);
        __half sh = __float2half_rn(__fdiv_rn(range, 7.0f));
        if ((__half_as_ushort(sh) & 0x7FFF) == 0) sh = __ushort_as_half(0x3C00);   // s := 1
        const float s = __half2float(sh);
        const __half zh = __float2half_rn(__fdiv_rn(-mn, s));
        const float z = __half2float(zh);
        if (!isfinite(s) || !isfinite(z)) st |= MILO_DEV_FP16_RANGE;
        blob_store_sz(blob, n, 2 * b + g, SB, __half_as_ushort(sh), __half_as_ushort(zh));
        for (int i = 0; i < 64; ++i) {
            const float v = __fadd_rn(__fdiv_rn(__half2float(__ushort_as_half(w[64 * g + i])), s), z);
            float r = rintf(v);
            if (!(r >= 0.0f)) r = 0.0f;
            if (r > 7.0f) r = 7.0f;
            q[64 * g + i] = static_cast<uint8_t>(r);
        }
    }

    uint32_t words[12];
    place_codes(q, words);
    blob_store_words(blob, n, b, SB, words);
    flag(dev_status, st);
}

// One thread per (row, super-block, unit): recover the 32 codes of a unit with
// the register-level extraction of the GEMM (field masks, one shift per word,
// the gathered spare register, the eight-step schedule), so that its bit-exact
// parity covers that logic.
template <int S, int H>
__device__ __forceinline__ void unpack_reg(const uint32_t (&w)[3], const uint32_t (&hw)[3],
                                           uint8_t (&u)[32]) {
    constexpr int t = sched_word(S, H), f = sched_field(S, H);
    constexpr int m = reg_code(t, f), sh = field_shift(t, f);
    const uint32_t r = unit_reg<t, f>(w, hw);
    u[m] = static_cast<uint8_t>((r & 0xFFFFu) >> sh);
    u[m + 1] = static_cast<uint8_t>((r >> 16) >> sh);
}

template <int S>
__device__ __forceinline__ void unpack_step(const uint32_t (&w)[3], const uint32_t (&hw)[3],
                                            uint8_t (&u)[32]) {
    unpack_reg<S, 0>(w, hw, u);
    unpack_reg<S, 1>(w, hw, u);
}

__global__ void __launch_bounds__(128) unpack_kernel(const uint8_t* __restrict__ blob, int N, int K,
                                                     uint8_t* __restrict__ codes) {
    const int SB = K / 128;
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid >= static_cast<long long>(N) * SB * 4) return;
    const int c = static_cast<int>(gid % 4);
    const long long nb = gid / 4;
    const int n = static_cast<int>(nb / SB), b = static_cast<int>(nb % SB);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(blob + blob_words(n, b, SB)) + 3 * c;
    const uint32_t w[3] = {src[0], src[1], src[2]};
    const uint32_t hw[3] = {w[0] >> word_shift(0), w[1] >> word_shift(1), w[2] >> word_shift(2)};
    uint8_t u[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) u[i] = 0xFF;   // a code the schedule misses stays 0xFF
    unpack_step<0>(w, hw, u);
    unpack_step<1>(w, hw, u);
    unpack_step<2>(w, hw, u);
    unpack_step<3>(w, hw, u);
    unpack_step<4>(w, hw, u);
    unpack_step<5>(w, hw, u);
    unpack_step<6>(w, hw, u);
    unpack_step<7>(w, hw, u);
    uint8_t* out = codes + static_cast<size_t>(n) * K + 128 * b;
#pragma unroll
    for (int m = 0; m < 32; ++m) out[unit_k(c, m)] = u[m];
}

// fp64 value -> fp16 bits, rounded once to nearest even: to fp32 rounding
// towards zero with a sticky last bit (round to odd keeps the information a
// second rounding needs), then fp32 -> fp16 to nearest even.
__device__ __forceinline__ uint16_t d2h_rn(double d) {
    float f = __double2float_rz(d);
    if (static_cast<double>(f) != d) f = __uint_as_float(__float_as_uint(f) | 1u);
    return __half_as_ushort(__float2half_rn(f));
}

// Dequantisation of one 32-code unit of one row: w_hat = (q - z) s for the
// unit's two groups, written as fp16 (the unfused baseline's weights).  The
// product is exact in fp64, so each value is rounded once.
__global__ void __launch_bounds__(128) dequant_kernel(const uint8_t* __restrict__ blob, int N, int K,
                                                       uint16_t* __restrict__ out) {
    const int SB = K / 128;
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid >= static_cast<long long>(N) * SB * 4) return;
    const int c = static_cast<int>(gid & 3);
    const long long nb = gid / 4;
    const int n = static_cast<int>(nb / SB), b = static_cast<int>(nb % SB);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(blob + blob_words(n, b, SB)) + 3 * c;
    const uint32_t w[3] = {src[0], src[1], src[2]};
    uint16_t v[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint16_t* sz = reinterpret_cast<const uint16_t*>(blob + blob_group(n, 2 * b + h, SB));
        const double s = static_cast<double>(__half2float(__ushort_as_half(sz[0])));
        const double z = static_cast<double>(__half2float(__ushort_as_half(sz[1])));
#pragma unroll
        for (int m = 0; m < 16; ++m)
            v[16 * h + m] = d2h_rn((static_cast<double>(unit_code(w, 16 * h + m)) - z) * s);
    }
    uint16_t* row = out + static_cast<size_t>(n) * K + 128 * b;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint4* o = reinterpret_cast<uint4*>(row + 64 * h + 16 * c);
        uint32_t p[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            p[i] = static_cast<uint32_t>(v[16 * h + 2 * i]) | (static_cast<uint32_t>(v[16 * h + 2 * i + 1]) << 16);
        o[0] = make_uint4(p[0], p[1], p[2], p[3]);
        o[1] = make_uint4(p[4], p[5], p[6], p[7]);
    }
}

}  // namespace milo

using namespace milo;

extern "C" milo_status milo_pack(const uint16_t* W, int32_t N, int32_t K, int32_t group, void* packed,
                                 int32_t* dev_status, void* stream) {
    clear_error();
    if (N <= 0 || K <= 0) return fail(MILO_ERR_INVALID_ARG, "milo_pack: N and K must be positive");
    if (N > kMaxWeightRows) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_pack: N above 2^31 - 64");
    if (group != MILO_GROUP) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_pack: group must be 64");
    if (K % 128) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_pack: K must be a multiple of 128");
    if (!W || !packed) return fail(MILO_ERR_INVALID_ARG, "milo_pack: NULL pointer");
    if (!aligned(packed, 16) || !aligned(W, 2))
        return fail(MILO_ERR_INVALID_ARG, "milo_pack: the packed buffer must be 16-byte aligned");
    const long long threads = static_cast<long long>((N + 63) / 64 * 64) * (K / 128);
    const int block = 128;
    const long long grid = (threads + block - 1) / block;
    if (grid > 0x7FFFFFFFLL) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_pack: too large");
    pack_kernel<<<static_cast<unsigned>(grid), block, 0, static_cast<cudaStream_t>(stream)>>>(
        W, N, K, static_cast<uint8_t*>(packed), dev_status);
    return check_launch("milo_pack");
}

extern "C" milo_status milo_unpack(const void* packed, int32_t N, int32_t K, uint8_t* codes, void* stream) {
    clear_error();
    if (!packed || !codes) return fail(MILO_ERR_INVALID_ARG, "milo_unpack: NULL pointer");
    if (N <= 0 || K <= 0) return fail(MILO_ERR_INVALID_ARG, "milo_unpack: N and K must be positive");
    if (N > kMaxWeightRows) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_unpack: N above 2^31 - 64");
    if (K % 128) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_unpack: K must be a multiple of 128");
    if (!aligned(packed, 4)) return fail(MILO_ERR_INVALID_ARG, "milo_unpack: the packed buffer must be 4-byte aligned");
    const long long threads = static_cast<long long>(N) * (K / 128) * 4;
    const int block = 128;
    const long long grid = (threads + block - 1) / block;
    if (grid > 0x7FFFFFFFLL) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_unpack: too large");
    unpack_kernel<<<static_cast<unsigned>(grid), block, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(packed), N, K, codes);
    return check_launch("milo_unpack");
}

extern "C" milo_status milo_packed_bytes(int32_t N, int32_t K, size_t* bytes) {
    clear_error();
    if (N <= 0 || K <= 0 || !bytes) return fail(MILO_ERR_INVALID_ARG, "milo_packed_bytes: bad argument");
    if (N > kMaxWeightRows) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_packed_bytes: N above 2^31 - 64");
    if (K % 128) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_packed_bytes: K must be a multiple of 128");
    *bytes = static_cast<size_t>((N + 63) / 64) * (K / 128) * kBlockSB;
    return MILO_OK;
}

extern "C" milo_status milo_dequantize(const void* packed, int32_t N, int32_t K, uint16_t* W_hat, void* stream) {
    clear_error();
    if (!packed || !W_hat) return fail(MILO_ERR_INVALID_ARG, "milo_dequantize: NULL pointer");
    if (N <= 0 || K <= 0) return fail(MILO_ERR_INVALID_ARG, "milo_dequantize: N and K must be positive");
    if (N > kMaxWeightRows) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_dequantize: N above 2^31 - 64");
    if (K % 128) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_dequantize: K must be a multiple of 128");
    if (!aligned(packed, 16) || !aligned(W_hat, 16))
        return fail(MILO_ERR_INVALID_ARG, "milo_dequantize: pointers must be 16-byte aligned");
    const long long threads = static_cast<long long>(N) * (K / 128) * 4;
    const int block = 128;
    const long long grid = (threads + block - 1) / block;
    if (grid > 0x7FFFFFFFLL) return fail(MILO_ERR_UNSUPPORTED_SHAPE, "milo_dequantize: too large");
    dequant_kernel<<<static_cast<unsigned>(grid), block, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(packed), N, K, W_hat);
    return check_launch("milo_dequantize");
}
