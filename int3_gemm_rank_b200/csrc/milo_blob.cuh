// milo_blob.cuh -- writing the packed blob (milo.h): where a row's words and
// its groups' scales and zeros go, and how 128 codes become 12 words.  Used by
// the quantise-and-pack kernels.
#pragma once

#include <stdint.h>

#include "milo_device.cuh"
#include "milo_kernels.h"

namespace milo {

// Byte offsets of row n's words for super-block b and of its scale for group j
// (its zero follows 2 bytes later).  Blocks are (64-row tile, super-block):
// the tile's words [64 rows][12], then the two groups' (s, z) pairs of rows r
// and r + 8 of each 16-row block.
__device__ __forceinline__ size_t blob_words(int n, int b, int SB) {
    return (static_cast<size_t>(n / 64) * SB + b) * kBlockSB + (n % 64) * 48;
}
__device__ __forceinline__ size_t blob_group(int n, int j, int SB) {
    const int r = n % 64;
    return (static_cast<size_t>(n / 64) * SB + (j >> 1)) * kBlockSB + kQTileSBWords * 4 + (j & 1) * kGroupBytes +
           (((r >> 4) * 8 + (r & 7)) * 4 + ((r >> 3) & 1) * 2) * 2;
}

// The 12 words of one row's 128-code super-block: unit c holds unit codes m
// (unit_k), word t of the unit holds codes 10t..10t+9 as five pairs (bits 3i
// and 16 + 3i), and bits 15 / 31 of word t are bit t of codes 30 / 31.
__device__ __forceinline__ void place_codes(const uint8_t (&q)[128], uint32_t (&words)[12]) {
#pragma unroll
    for (int i = 0; i < 12; ++i) words[i] = 0u;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int m = 0; m < 30; ++m) {
            const int t = m / 10, r = m % 10;
            const int pos = 16 * (r & 1) + 3 * (r >> 1);
            words[3 * c + t] |= static_cast<uint32_t>(q[unit_k(c, m)]) << pos;
        }
        const uint32_t u30 = q[unit_k(c, 30)], u31 = q[unit_k(c, 31)];
#pragma unroll
        for (int t = 0; t < 3; ++t)
            words[3 * c + t] |= (((u30 >> t) & 1u) << 15) | (((u31 >> t) & 1u) << 31);
    }
}

// The same placement one code at a time: code q at super-block position k
// (0..127) ORed into the zero-initialised words (k a compile-time constant
// after unrolling keeps the words in registers).
__device__ __forceinline__ void place_code(uint32_t (&words)[12], int k, uint32_t q) {
    const int c = (k & 63) >> 4, m = (k & 15) + ((k >> 6) << 4);   // unit, unit code (unit_k inverted)
    if (m < 30) {
        const int t = m / 10, r = m % 10;
        words[3 * c + t] |= q << (16 * (r & 1) + 3 * (r >> 1));
    } else {
        const int bit = m == 30 ? 15 : 31;
#pragma unroll
        for (int t = 0; t < 3; ++t) words[3 * c + t] |= ((q >> t) & 1u) << bit;
    }
}

// Zero words, scales and zeros for a padding row n >= N of the last tile.
__device__ __forceinline__ void blob_zero_row(uint8_t* blob, int n, int b, int SB) {
    uint4* dst = reinterpret_cast<uint4*>(blob + blob_words(n, b, SB));
    dst[0] = dst[1] = dst[2] = make_uint4(0u, 0u, 0u, 0u);
    uint16_t* sz = reinterpret_cast<uint16_t*>(blob);
    for (int g = 0; g < 2; ++g) {
        const size_t o = blob_group(n, 2 * b + g, SB) / 2;
        sz[o] = 0;
        sz[o + 1] = 0;
    }
}

__device__ __forceinline__ void blob_store_words(uint8_t* blob, int n, int b, int SB, const uint32_t (&words)[12]) {
    uint4* dst = reinterpret_cast<uint4*>(blob + blob_words(n, b, SB));
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    dst[2] = make_uint4(words[8], words[9], words[10], words[11]);
}

__device__ __forceinline__ void blob_store_sz(uint8_t* blob, int n, int j, int SB, uint16_t s, uint16_t z) {
    uint16_t* sz = reinterpret_cast<uint16_t*>(blob);
    const size_t o = blob_group(n, j, SB) / 2;
    sz[o] = s;
    sz[o + 1] = z;
}

}  // namespace milo
