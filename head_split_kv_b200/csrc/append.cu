// append.cu -- duo_append_kv: T new tokens per sequence into the two caches.
//
// [Review S3 "Inference flow"] each layer keeps a full KV cache for the
// retrieval heads and a constant-size sink + recent cache for the streaming
// heads; [Summary S2 "Chunked Pre-filling"] pre-fill fills both.
//
// A pure copy: every thread moves 16-byte pieces of K/V rows, reading the
// input rows in order (coalesced) and writing each row to its cache slot.
// Streaming heads write only the tokens that survive the chunk (p < sink or
// among the last `recent`).  seq_len is advanced by the last CTA to finish
// (an atomic ticket, no waiting), after every CTA has read the old value.
#include "common.cuh"
#include "internal.h"
#include "kvq4.cuh"
#include "kvq8.cuh"

namespace duo {
namespace {

__global__ void __launch_bounds__(256) append_kernel(const LayerArgs a, const CacheArgs c, const uint4* __restrict__ k_new,
                                                     const uint4* __restrict__ v_new, const int T) {
    const int row_bytes = a.D * (a.dtype == DUO_BF16 ? 2 : 4);
    const int cpr = row_bytes / 16;                     // 16-byte pieces per row
    const long rows = (long)a.B * T * a.Hkv;            // input rows per tensor
    const long per_tensor = rows * cpr;
    const long total = 2 * per_tensor;
    for (long x = (long)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += (long)gridDim.x * blockDim.x) {
        const int tensor = x >= per_tensor;              // 0: K, 1: V
        const long xr = x - tensor * per_tensor;
        const long r = xr / cpr;
        const int piece = (int)(xr - r * cpr);
        const int h_in = (int)(r % a.Hkv);
        const long bt = r / a.Hkv;
        const int t = (int)(bt % T);
        const int b = (int)(bt / T);
        const int slot = a.slot_of[h_in];
        if (!bounds_ok(slot >= 0 && slot < a.R + a.S, c.status)) continue;
        const int L = c.seq_len[b];
        const int p = L + t;
        const uint4 val = (tensor ? v_new : k_new)[xr];
        if (slot < a.R) {
            long dst_row;
            if (p >= a.capacity || p < 0) {
                if (piece == 0 && tensor == 0) atomicOr(c.status, DUO_DEV_FULL_CACHE_OVERFLOW);
                continue;
            }
            if (a.page_size == 0) {
                dst_row = ((long)b * a.R + slot) * a.capacity + p;
            } else {
                const int pg = c.page_table[(long)b * a.max_pages + p / a.page_size];
                if (pg < 0 || pg >= a.n_pages) {
                    if (piece == 0 && tensor == 0) atomicOr(c.status, DUO_DEV_BAD_PAGE);
                    continue;
                }
                dst_row = ((long)pg * a.R + slot) * a.page_size + (p % a.page_size);
            }
            uint4* dst = reinterpret_cast<uint4*>(tensor ? c.v_full : c.k_full);
            dst[dst_row * cpr + piece] = val;
        } else {
            // keep only the tokens that survive this append: sinks and the last `recent`
            if (p < 0) {
                if (piece == 0 && tensor == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
                continue;
            }
            if (!(p < a.sink || p >= L + T - a.recent)) continue;
            const int s = slot - a.R;
            const int rs = ring_slot(p, a.sink, a.recent);
            if (!bounds_ok(rs >= 0 && rs < a.W, c.status)) continue;
            const long dst_row = ((long)b * a.S + s) * a.W + rs;
            uint4* dst = reinterpret_cast<uint4*>(tensor ? c.v_ring : c.k_ring);
            dst[dst_row * cpr + piece] = val;
            if (s == 0 && piece == 0 && tensor == 0) c.ring_pos[(long)b * a.W + rs] = p;
        }
    }
    // The last CTA to finish advances the lengths.  Every CTA read seq_len
    // before its ticket, so none can see the new value.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned ticket = atomicAdd(&c.counters[0], 1u);
        if (ticket == gridDim.x - 1) {
            __threadfence();
            for (int b = 0; b < a.B; ++b) c.seq_len[b] += T;
            c.counters[0] = 0u;
            __threadfence();
        }
    }
}

// ------------------------------------------------------------------------
// 8- and 4-bit full caches: one warp per (token, KV head, K|V) row.  A
// retrieval row is quantized and stored in the BITS-bit layouts (kvq8.cuh,
// kvq4.cuh); a streaming row is copied into the ring as in the plain kernel.

template <int BITS>
__global__ void __launch_bounds__(256) append_q_kernel(const LayerArgs a, const CacheArgs c,
                                                       const __nv_bfloat16* __restrict__ k_new,
                                                       const __nv_bfloat16* __restrict__ v_new, const int T) {
    const int lane = threadIdx.x & 31;
    const long rows = (long)a.B * T * a.Hkv;             // input rows per tensor
    const long warps = (long)gridDim.x * (blockDim.x >> 5);
    for (long x = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); x < 2 * rows; x += warps) {
        const int kv = x >= rows;                         // 0: K, 1: V
        const long r = x - kv * rows;
        const int h_in = (int)(r % a.Hkv);
        const long bt = r / a.Hkv;
        const int t = (int)(bt % T);
        const int b = (int)(bt / T);
        const int slot = a.slot_of[h_in];
        if (!bounds_ok(slot >= 0 && slot < a.R + a.S, c.status)) continue;
        const int L = c.seq_len[b];
        const int p = L + t;
        const __nv_bfloat16* src = (kv ? v_new : k_new) + r * 128;
        if (slot < a.R) {
            if (p >= a.capacity || p < 0) {
                if (lane == 0 && kv == 0) atomicOr(c.status, DUO_DEV_FULL_CACHE_OVERFLOW);
                continue;
            }
            const uint2 w = reinterpret_cast<const uint2*>(src)[lane];
            const float xv[4] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y)};
            float scale;
            if constexpr (BITS == 8) {
                const uint32_t codes = q8_quantize(xv, scale);
                q8_store_row(a, c, kv, b, slot, p, codes, scale, lane);
            } else {
                int codes[4];
                q4_quantize(xv, codes, scale);
                q4_store_row(a, c, kv, b, slot, p, codes, scale, lane);
            }
        } else {
            if (p < 0) {
                if (lane == 0 && kv == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
                continue;
            }
            if (!(p < a.sink || p >= L + T - a.recent)) continue;
            const int s = slot - a.R;
            const int rs = ring_slot(p, a.sink, a.recent);
            if (!bounds_ok(rs >= 0 && rs < a.W, c.status)) continue;
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(kv ? c.v_ring : c.k_ring) + (((long)b * a.S + s) * a.W + rs) * 128;
            reinterpret_cast<uint2*>(dst)[lane] = reinterpret_cast<const uint2*>(src)[lane];
            if (s == 0 && lane == 0 && kv == 0) c.ring_pos[(long)b * a.W + rs] = p;
        }
    }
    // the last CTA to finish advances the lengths (every CTA read them first)
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned ticket = atomicAdd(&c.counters[0], 1u);
        if (ticket == gridDim.x - 1) {
            __threadfence();
            for (int b = 0; b < a.B; ++b) c.seq_len[b] += T;
            c.counters[0] = 0u;
            __threadfence();
        }
    }
}

}  // namespace

cudaError_t launch_append(const LayerArgs& a, const CacheArgs& c, const void* k_new, const void* v_new, int T,
                          cudaStream_t s) {
    if (a.kv_bits) {
        const long warps = 2L * a.B * T * a.Hkv;
        long blocks = (warps + 7) / 8;
        if (blocks > 148L * 8) blocks = 148L * 8;
        if (blocks < 1) blocks = 1;
        const auto* kn = static_cast<const __nv_bfloat16*>(k_new);
        const auto* vn = static_cast<const __nv_bfloat16*>(v_new);
        if (a.kv_bits == 8)
            append_q_kernel<8><<<(unsigned)blocks, 256, 0, s>>>(a, c, kn, vn, T);
        else
            append_q_kernel<4><<<(unsigned)blocks, 256, 0, s>>>(a, c, kn, vn, T);
        return cudaGetLastError();
    }
    const int row_bytes = a.D * (a.dtype == DUO_BF16 ? 2 : 4);
    const long total = 2L * a.B * T * a.Hkv * (row_bytes / 16);
    const int threads = 256;
    long blocks = (total + threads - 1) / threads;
    if (blocks > 148L * 8) blocks = 148L * 8;
    if (blocks < 1) blocks = 1;
    append_kernel<<<(unsigned)blocks, threads, 0, s>>>(a, c, static_cast<const uint4*>(k_new),
                                                       static_cast<const uint4*>(v_new), T);
    return cudaGetLastError();
}

}  // namespace duo
