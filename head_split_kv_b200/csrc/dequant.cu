// dequant.cu -- the rows an 8- or 4-bit full cache holds, staged for the
// tensor-core pre-fill in a contiguous [B][R][capacity][128] K area and V
// area: the K codes as bf16 values and the V codes times 16 as fp16 values
// (both exact: |16 code| <= 2032), and each row's (k scale, v scale / 16,
// 0, 0) in a [B][R][capacity][4] fp32 area, which the pre-fill loads with
// each prior K tile and applies to the scores and to p.  Staging
// code * scale itself in bf16 would round every cached value once more than
// the oracle's code * scale; keeping the scales apart keeps that product
// out of bf16, and the fp16 PV operands keep the rounding of p times the
// scale at 2^-11.
//
// One warp per cached row (slot z = b * R + r, position p < seq_len[b]);
// lane l writes features 4l .. 4l+3 of the K row and of the V row, reading
// the codes from the layouts kvq8.cuh and kvq4.cuh describe.  Rows at or
// past seq_len[b] are not read or written: the pre-fill only reads prior
// rows below the chunk start.
#include "common.cuh"
#include "internal.h"
#include "kvq4.cuh"
#include "kvq8.cuh"

namespace duo {
namespace {

__device__ __forceinline__ void store4_bf16(__nv_bfloat16* dst, const float (&v)[4]) { store_row<__nv_bfloat16, 4>(dst, v); }

__device__ __forceinline__ void store4_f16(__half* dst, const float (&v)[4]) {
    const __half2 a = __floats2half2_rn(v[0], v[1]), b = __floats2half2_rn(v[2], v[3]);
    uint2 w;
    w.x = *reinterpret_cast<const uint32_t*>(&a);
    w.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(dst) = w;
}

template <int BITS>
__global__ void __launch_bounds__(256) dequant_kernel(const LayerArgs a, const CacheArgs c, __nv_bfloat16* kd,
                                                      __half* vd, float4* sd) {
    const int lane = threadIdx.x & 31;
    const long rows = (long)a.B * a.R * a.capacity;
    const long warps = (long)gridDim.x * (blockDim.x >> 5);
    for (long x = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); x < rows; x += warps) {
        const long z = x / a.capacity;
        const int p = (int)(x - z * a.capacity);
        const int b = (int)(z / a.R);
        if (p >= c.seq_len[b]) continue;
        if (lane == 0) sd[x] = make_float4(c.k_scale[x], c.v_scale[x] * 0.0625f, 0.f, 0.f);
        float kv[4], vv[4];
        if constexpr (BITS == 8) {
            const uint32_t w = reinterpret_cast<const uint32_t*>(static_cast<const int8_t*>(c.k_full) + x * 128)[lane];
            const int8_t* tile = static_cast<const int8_t*>(c.v_full) + (z * (a.capacity / 64) + p / 64) * (128 * 64);
            const int col = ((p & 63) >> 4) * 16 + q8_group_pos(p & 15);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                kv[i] = (float)(int8_t)(w >> (8 * i));
                vv[i] = 16.f * (float)tile[(4 * lane + i) * 64 + col];
            }
        } else {
            // K: lane l holds features 32 q + 4 kb + i (q = l / 8, kb = l % 8):
            // byte s of word kb / 2 has (i = 0, i = 2), byte s + 2 has (1, 3)
            const uint8_t* row = static_cast<const uint8_t*>(c.k_full) + x * kQ4RowBytes;
            const int q = lane >> 3, kb = lane & 7, j = kb >> 1, s = kb & 1;
            const uint8_t b02 = row[16 * q + 4 * j + s], b13 = row[16 * q + 4 * j + 2 + s];
            kv[0] = (float)((int)(b02 & 15) - 8);
            kv[2] = (float)((int)(b02 >> 4) - 8);
            kv[1] = (float)((int)(b13 & 15) - 8);
            kv[3] = (float)((int)(b13 >> 4) - 8);
            // V: feature f = 16 m + r (+ 8 in the high nibble) of token t at
            // 1024 g + 128 m + 16 r + 4 k + byte-in-word
            const uint8_t* tile = static_cast<const uint8_t*>(c.v_full) + (z * (a.capacity / 64) + p / 64) * kQ4TileBytes;
            const int t = p & 63, g = t >> 4, tt = t & 15;
            const int k = (tt & 7) >> 1, bw = (tt & 1) * 2 + (tt >> 3);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int f = 4 * lane + i, m = f >> 4, r = f & 7, high = (f >> 3) & 1;
                const uint8_t byte = tile[1024 * g + 128 * m + 16 * r + 4 * k + bw];
                vv[i] = 16.f * (float)((int)(high ? byte >> 4 : byte & 15) - 8);
            }
        }
        store4_bf16(kd + x * 128 + 4 * lane, kv);
        store4_f16(vd + x * 128 + 4 * lane, vv);
    }
}

}  // namespace

size_t dequant_staging_bytes(const LayerArgs& a) {
    const size_t rows = (size_t)a.B * a.R * a.capacity;
    return rows * (2 * 128 * sizeof(__nv_bfloat16) + 4 * sizeof(float));
}

cudaError_t launch_dequant(const LayerArgs& a, const CacheArgs& c, void* staging, cudaStream_t s) {
    const long rows = (long)a.B * a.R * a.capacity;
    if (rows == 0) return cudaSuccess;
    long blocks = (rows + 7) / 8;
    if (blocks > 148L * 16) blocks = 148L * 16;
    auto* kd = static_cast<__nv_bfloat16*>(staging);
    auto* vd = reinterpret_cast<__half*>(kd + (size_t)rows * 128);
    auto* sd = reinterpret_cast<float4*>(vd + (size_t)rows * 128);
    if (a.kv_bits == 8)
        dequant_kernel<8><<<(unsigned)blocks, 256, 0, s>>>(a, c, kd, vd, sd);
    else
        dequant_kernel<4><<<(unsigned)blocks, 256, 0, s>>>(a, c, kd, vd, sd);
    return cudaGetLastError();
}

}  // namespace duo
