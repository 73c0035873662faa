// dequant.cu -- the rows an 8- or 4-bit full cache holds, staged for the
// tensor-core pre-fill in a contiguous [B][R][capacity][128] K area and V
// area: the K codes as bf16 values and the V codes times 16 as fp16 values
// (both exact: |16 code| <= 2032); then, per (sequence, retrieval head), a
// row of the k scales and a row of the v scales / 16, each capacity + 4
// floats long: [B][R][2][capacity + 4].  The pre-fill loads a prior tile's
// 128 scales of each row with its K tile and applies them to the scores and
// to p.  Staging code * scale itself in bf16 would round every cached value
// once more than the oracle's code * scale; keeping the scales apart keeps
// that product out of bf16, and the fp16 PV operands keep the rounding of p
// times the scale at 2^-11.
//
// The scale of position p sits at index p + delta of its row, delta =
// (4 - c0 % 4) % 4 with c0 = seq_len[b], the start of the chunk the pre-fill
// runs next: a prior tile starts at c0 - 128 k, so every tile's first scale
// lands on a multiple of four floats -- the 16-byte alignment a tensor copy's
// x coordinate needs -- and the softmax reads the scales four at a time.
//
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

// One CTA per (sequence, retrieval head, 64-token tile) below seq_len: the
// tile's V codes (4 or 8 KB) come into shared memory with coalesced 16-byte
// loads, then each warp writes 8 of the tile's rows -- lane l features 4l ..
// 4l + 3 of the K row (read straight from its contiguous row) and of the V
// row (gathered from the shared copy of the tile) -- and the rows' scales.
template <int BITS>
__global__ void __launch_bounds__(256) dequant_kernel(const LayerArgs a, const CacheArgs c, __nv_bfloat16* kd,
                                                      __half* vd, float* sd) {
    constexpr int kVTileBytes = BITS == 8 ? 128 * 64 : kQ4TileBytes;
    __shared__ __align__(16) uint8_t sv[kVTileBytes];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tiles = a.capacity / 64;
    const long n_tiles = (long)a.B * a.R * tiles;
    for (long tz = blockIdx.x; tz < n_tiles; tz += gridDim.x) {
        const long z = tz / tiles;
        const int p0 = (int)(tz - z * tiles) * 64;
        const int b = (int)(z / a.R);
        const int c0 = c.seq_len[b];
        if (p0 >= c0) continue;                          // the same for the whole CTA
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(c.v_full) + tz * kVTileBytes);
        for (int i = threadIdx.x; i < kVTileBytes / 16; i += blockDim.x) reinterpret_cast<uint4*>(sv)[i] = src[i];
        __syncthreads();
        const size_t srow = (size_t)(a.capacity + 4);
        const int shift = (4 - (c0 & 3)) & 3;
        for (int tt = warp; tt < 64; tt += 8) {
            const int p = p0 + tt;
            if (p >= c0) break;                          // rows past the length: not read
            const long x = z * a.capacity + p;
            if (lane == 0) {
                sd[(2 * z) * srow + p + shift] = c.k_scale[x];
                sd[(2 * z + 1) * srow + p + shift] = c.v_scale[x] * 0.0625f;
            }
            float kv[4], vv[4];
            if constexpr (BITS == 8) {
                const uint32_t w = reinterpret_cast<const uint32_t*>(static_cast<const int8_t*>(c.k_full) + x * 128)[lane];
                const int col = (tt >> 4) * 16 + q8_group_pos(tt & 15);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    kv[i] = (float)(int8_t)(w >> (8 * i));
                    vv[i] = 16.f * (float)(int8_t)sv[(4 * lane + i) * 64 + col];
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
                // 1024 g + 128 m + 16 r + 4 k + byte-in-word of the tile
                const int g = tt >> 4, t16 = tt & 15;
                const int k = (t16 & 7) >> 1, bw = (t16 & 1) * 2 + (t16 >> 3);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int f = 4 * lane + i, m = f >> 4, r = f & 7, high = (f >> 3) & 1;
                    const uint8_t byte = sv[1024 * g + 128 * m + 16 * r + 4 * k + bw];
                    vv[i] = 16.f * (float)((int)(high ? byte >> 4 : byte & 15) - 8);
                }
            }
            store4_bf16(kd + x * 128 + 4 * lane, kv);
            store4_f16(vd + x * 128 + 4 * lane, vv);
        }
        __syncthreads();                                 // the tile buffer is reused
    }
}

}  // namespace

size_t dequant_staging_bytes(const LayerArgs& a) {
    const size_t rows = (size_t)a.B * a.R * a.capacity;
    return rows * 2 * 128 * sizeof(__nv_bfloat16) + (size_t)a.B * a.R * 2 * (a.capacity + 4) * sizeof(float);
}

cudaError_t launch_dequant(const LayerArgs& a, const CacheArgs& c, void* staging, cudaStream_t s) {
    const long rows = (long)a.B * a.R * a.capacity;
    if (rows == 0) return cudaSuccess;
    long blocks = rows / 64;                          // one CTA per 64-token tile, grid-stride
    if (blocks > 148L * 8) blocks = 148L * 8;
    auto* kd = static_cast<__nv_bfloat16*>(staging);
    auto* vd = reinterpret_cast<__half*>(kd + (size_t)rows * 128);
    auto* sd = reinterpret_cast<float*>(vd + (size_t)rows * 128);
    if (a.kv_bits == 8)
        dequant_kernel<8><<<(unsigned)blocks, 256, 0, s>>>(a, c, kd, vd, sd);
    else
        dequant_kernel<4><<<(unsigned)blocks, 256, 0, s>>>(a, c, kd, vd, sd);
    return cudaGetLastError();
}

}  // namespace duo
