// kvq4.cuh -- the 4-bit full cache of the retrieval heads: quantizing a row,
// storing it in the cache layouts, and widening codes to fp16 MMA operands.
//
// Scheme (the paper review's "Quantization combination" pairs 8-bit weights
// with a 4-bit KV cache and gives no scheme): per cached row of d = 128
// values, amax = max |x|, code = x * (7 / amax) rounded to nearest even,
// scale = amax / 7, each one IEEE fp32 operation; codes -7..7 are stored as
// the nibble code + 8; a zero row has scale 0 and codes 0.  Attention reads
// code * scale.
//
// Layouts (slot z = b * R + r, 64-token tiles; a byte holds two nibbles,
// the first in its low half):
//   K codes  [z][capacity][64 bytes]: a row per token.  Byte 16 q + 4 j + c
//            of a row holds, for lane group q (features 32 q ..) and word j,
//            with e = 32 q + 8 j:  c = 0: (e, e + 2)   c = 1: (e + 4, e + 6)
//                                  c = 2: (e + 1, e + 3)  c = 3: (e + 5, e + 7)
//            so that the word's nibble pairs (0, 4), (1, 5), (2, 6), (3, 7)
//            -- what one mask-and-or splits into two fp16 values -- are the
//            features (e, e+1), (e+2, e+3), (e+4, e+5), (e+6, e+7): the q . K
//            MMA operands of two k-steps of the group's permuted feature order.
//   V codes  [z][capacity / 64][4096 bytes]: per tile, for each 16-token
//            group g, feature block m (features 16 m .. 16 m + 15), row r
//            (0..7) and key quad k (0..3) one word at
//            1024 g + 128 m + 16 r + 4 k whose bytes are the tokens
//            2k, 2k + 8, 2k + 1, 2k + 9 of the group, each byte holding
//            features 16 m + r (low nibble) and 16 m + 8 + r (high nibble):
//            one byte per token, so appends never share a byte, and the
//            word's nibble pairs are the P V operands of two feature rows.
//   scales   fp32 [z][capacity] for K and for V.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

namespace duo {

constexpr int kQ4RowBytes = 64;     // K codes of one token
constexpr int kQ4TileBytes = 4096;  // K or V codes of a 64-token tile

// Lane l of a warp holds x[4l .. 4l+3] of one 128-value row: returns the four
// codes (-7..7) and the row's scale.
__device__ __forceinline__ void q4_quantize(const float (&x)[4], int (&code)[4], float& scale) {
    float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (amax == 0.f) {
        scale = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) code[i] = 0;
        return;
    }
    const float inv = __fdiv_rn(7.f, amax);
#pragma unroll
    for (int i = 0; i < 4; ++i) code[i] = max(-7, min(7, __float2int_rn(__fmul_rn(x[i], inv))));
    scale = __fdiv_rn(amax, 7.f);
}

__device__ __forceinline__ uint8_t q4_byte(int lo, int hi) {
    return (uint8_t)((lo + 8) | ((hi + 8) << 4));
}

// Stores the quantized row (codes from q4_quantize, whole warp) of retrieval
// slot `slot` of sequence b at position p: K (kv = 0) the token's 64-byte
// row, V (kv = 1) one byte in each of the tile's 64 feature-pair words;
// lane 0 stores the scale.
__device__ __forceinline__ void q4_store_row(const LayerArgs& a, const CacheArgs& c, int kv, int b, int slot, int p,
                                             const int (&code)[4], float scale, int lane) {
    if (!bounds_ok(slot >= 0 && slot < a.R && p >= 0 && p < a.capacity, c.status)) return;  // warp-uniform
    const size_t z = (size_t)b * a.R + slot;
    if (kv == 0) {
        // lane l: features 4l + i = 32 q + 4 kb + i with q = l / 8, kb = l % 8;
        // word j = kb / 2, s = kb % 2: byte s holds (i = 0, i = 2), byte
        // s + 2 holds (i = 1, i = 3)
        uint8_t* row = static_cast<uint8_t*>(c.k_full) + (z * a.capacity + p) * kQ4RowBytes;
        const int q = lane >> 3, kb = lane & 7, j = kb >> 1, s = kb & 1;
        row[16 * q + 4 * j + s] = q4_byte(code[0], code[2]);
        row[16 * q + 4 * j + 2 + s] = q4_byte(code[1], code[3]);
        if (lane == 0) c.k_scale[z * a.capacity + p] = scale;
    } else {
        // a byte pairs features f and f + 8: lanes whose features have bit 3
        // clear (l / 2 even) take the partner codes from lane l + 2
        int partner[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) partner[i] = __shfl_down_sync(0xffffffffu, code[i], 2);
        if (((lane >> 1) & 1) == 0) {
            uint8_t* tile = static_cast<uint8_t*>(c.v_full) + (z * (a.capacity / 64) + p / 64) * kQ4TileBytes;
            const int t = p & 63, g = t >> 4, tt = t & 15;
            const int k = (tt & 7) >> 1, byte_in_word = (tt & 1) * 2 + (tt >> 3);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int f = 4 * lane + i, m = f >> 4, r = f & 7;
                tile[1024 * g + 128 * m + 16 * r + 4 * k + byte_in_word] = q4_byte(code[i], partner[i]);
            }
        }
        if (lane == 0) c.v_scale[z * a.capacity + p] = scale;
    }
}

// Nibbles at bits 0-3 and 16-19 of w -> the fp16 pair (1024 + n0, 1024 + n1).
__device__ __forceinline__ uint32_t u4_lo_f16x2(uint32_t w) { return (w & 0x000F000Fu) | 0x64006400u; }
// Nibbles at bits 4-7 and 20-23 of w -> the fp16 pair (1024 + 16 n0, 1024 + 16 n1).
__device__ __forceinline__ uint32_t u4_hi_f16x2(uint32_t w) { return (w & 0x00F000F0u) | 0x64006400u; }

// Nibbles at bits 0-3 / 16-19 of w as fp16 subnormals n * 2^-24, and those
// at bits 4-7 / 20-23 as 16 n * 2^-24, exactly (zero exponent).
__device__ __forceinline__ uint32_t u4_lo_sub(uint32_t w) { return w & 0x000F000Fu; }
__device__ __forceinline__ uint32_t u4_hi_sub(uint32_t w) { return w & 0x00F000F0u; }

// Nibbles 0 and 4 of w (bits 0-3 and 16-19) -> two fp16 values nibble - 8,
// exactly: a nibble n under the fp16 exponent of 1024 is the number 1024 + n,
// and subtracting 1032 leaves n - 8.
__device__ __forceinline__ uint32_t u4x2_to_f16x2(uint32_t w) {
    const uint32_t t = (w & 0x000F000Fu) | 0x64006400u;
    const __half2 bias = __halves2half2(__ushort_as_half((unsigned short)0x6408),
                                        __ushort_as_half((unsigned short)0x6408));
    const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&t), bias);
    return *reinterpret_cast<const uint32_t*>(&r);
}

}  // namespace duo
