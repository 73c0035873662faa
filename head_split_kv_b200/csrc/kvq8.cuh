// kvq8.cuh -- the 8-bit full cache of the retrieval heads: quantizing a row,
// storing it in the cache layouts, and widening codes to fp16 MMA operands.
//
// Scheme (the pages pair the method with a quantized KV cache -- review S5
// "Decoding performance" -- without giving one): per cached row of d = 128
// values, amax = max |x|, code = x * (127 / amax) rounded to nearest even,
// scale = amax / 127, each one IEEE fp32 operation; a zero row has scale 0
// and codes 0.  Attention reads code * scale.
//
// Layouts (slot z = b * R + r):
//   K codes  int8 [z][capacity][128]        a row per token;
//   V codes  int8 [z][capacity / 64][128][64]  per 64-token tile, transposed
//            (one 64-byte row per feature), the 16 tokens of each 16-token
//            group in the order 0 1 8 9 2 3 10 11 4 5 12 13 6 7 14 15, so that
//            the four bytes a lane needs for one PV fragment are adjacent;
//   scales   fp32 [z][capacity] for K and for V.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

namespace duo {

// Position of token k (0..15) of a 16-token group in the V layout's order.
__device__ __forceinline__ int q8_group_pos(int k) {
    return k < 8 ? (k >> 1) * 4 + (k & 1) : ((k - 8) >> 1) * 4 + 2 + (k & 1);
}

// Lane l of a warp holds x[4l .. 4l+3] of one 128-value row: returns the four
// codes packed in a word (byte i = code of x[4l + i]) and the row's scale.
__device__ __forceinline__ uint32_t q8_quantize(const float (&x)[4], float& scale) {
    float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (amax == 0.f) {
        scale = 0.f;
        return 0u;
    }
    const float inv = __fdiv_rn(127.f, amax);
    uint32_t packed = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int c = __float2int_rn(__fmul_rn(x[i], inv));
        c = max(-127, min(127, c));
        packed |= (uint32_t)(c & 0xff) << (8 * i);
    }
    scale = __fdiv_rn(amax, 127.f);
    return packed;
}

// Stores the quantized row (codes from q8_quantize) of retrieval slot `slot`
// of sequence b at position p: K (kv = 0) one row of codes, V (kv = 1) one
// byte in each of the tile's feature rows; lane 0 stores the scale.
__device__ __forceinline__ void q8_store_row(const LayerArgs& a, const CacheArgs& c, int kv, int b, int slot, int p,
                                             uint32_t codes, float scale, int lane) {
    if (!bounds_ok(slot >= 0 && slot < a.R && p >= 0 && p < a.capacity, c.status)) return;  // warp-uniform
    const size_t z = (size_t)b * a.R + slot;
    if (kv == 0) {
        reinterpret_cast<uint32_t*>(static_cast<int8_t*>(c.k_full) + (z * a.capacity + p) * 128)[lane] = codes;
        if (lane == 0) c.k_scale[z * a.capacity + p] = scale;
    } else {
        int8_t* tile = static_cast<int8_t*>(c.v_full) + (z * (a.capacity / 64) + p / 64) * (128 * 64);
        const int col = ((p & 63) >> 4) * 16 + q8_group_pos(p & 15);
#pragma unroll
        for (int i = 0; i < 4; ++i) tile[(4 * lane + i) * 64 + col] = (int8_t)(codes >> (8 * i));
        if (lane == 0) c.v_scale[z * a.capacity + p] = scale;
    }
}

// Four int8 codes -> two fp16 pairs, exactly: the biased byte x + 128 under
// the fp16 exponent of 1024 is the number 1024 + x + 128, and subtracting
// 1152 leaves x.  lo = (code 0, code 1), hi = (code 2, code 3).
__device__ __forceinline__ void i8x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t t0 = __byte_perm(u, 0x64646464u, 0x4140);
    const uint32_t t1 = __byte_perm(u, 0x64646464u, 0x4342);
    const __half2 bias = __halves2half2(__ushort_as_half((unsigned short)0x6480),
                                        __ushort_as_half((unsigned short)0x6480));
    const __half2 r0 = __hsub2(*reinterpret_cast<const __half2*>(&t0), bias);
    const __half2 r1 = __hsub2(*reinterpret_cast<const __half2*>(&t1), bias);
    lo = *reinterpret_cast<const uint32_t*>(&r0);
    hi = *reinterpret_cast<const uint32_t*>(&r1);
}

// The same without the subtraction: (1152 + code 0, 1152 + code 1) and
// (1152 + code 2, 1152 + code 3), for products whose bias is removed later.
__device__ __forceinline__ void i8x4_to_f16x2_biased(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    lo = __byte_perm(u, 0x64646464u, 0x4140);
    hi = __byte_perm(u, 0x64646464u, 0x4342);
}

// Codes 0..3 of w as fp16 subnormals: (code + 128) * 2^-24 in each half,
// exactly (the offset code fills bits 0-7 of the half under a zero
// exponent).  For products whose bias, 128 times the sum of the partners,
// is removed once at the end.
__device__ __forceinline__ void i8x4_to_f16x2_sub(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    lo = __byte_perm(u, 0u, 0x4140);
    hi = __byte_perm(u, 0u, 0x4342);
}

__device__ __forceinline__ uint32_t f16x2_pack(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace duo
