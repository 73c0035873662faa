// mix.cu -- the gated mix's second pass for bf16, head_dim 128: streaming
// (Lambda-mask) attention of every query head, mixed with the causal
// attention the tensor-core pre-fill kernel has already written to `out`:
//   out = alpha * causal + (1 - alpha) * streaming.
//
// [Review S3 "Core formula": attn = alpha * full_attn + (1 - alpha) *
//  streaming_attn, the streaming mask allowing only the initial (sink) tokens
//  and the recent tokens; Summary S2 "Optimization-based Identification": one
//  gate per KV head, shared by its query heads.]
//
// One warp per (sequence, token i, KV head) handles the G query heads of the
// group, so each key and value row is loaded once for all of them.  Lane l
// holds features 4l .. 4l+3.  Keys are visited in increasing position: the
// sinks j < min(sink, i + 1), then the recent band max(sink, i - recent + 1)
// .. i -- at most sink + recent keys, so the pass is linear in the sequence
// length.  Per key and head: a 4-element partial dot, a butterfly sum over
// the warp, and an online-softmax update in fp32.
#include "common.cuh"
#include "internal.h"

namespace duo {
namespace {

constexpr int kD = 128;
constexpr int kWarps = 8;   // warps per CTA

__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    x[0] = bf16_lo(u.x);
    x[1] = bf16_hi(u.x);
    x[2] = bf16_lo(u.y);
    x[3] = bf16_hi(u.y);
}

template <int G>
__global__ void __launch_bounds__(kWarps * 32)
    lambda_mix_kernel(const LayerArgs a, const float* __restrict__ alpha, const __nv_bfloat16* __restrict__ q,
                      const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, int N,
                      __nv_bfloat16* out) {
    const int lane = threadIdx.x & 31;
    const long unit = (long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (unit >= (long)a.B * N * a.Hkv) return;
    const int kv = (int)(unit % a.Hkv);
    const int i = (int)((unit / a.Hkv) % N);
    const int b = (int)(unit / ((long)a.Hkv * N));
    const float sl = a.scale * kLog2e;

    float qf[G][4], acc[G][4], m[G], l[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        load4(q + (((size_t)b * N + i) * a.Hq + kv * G + g) * kD + 4 * lane, qf[g]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            qf[g][e] *= sl;
            acc[g][e] = 0.f;
        }
        m[g] = -INFINITY;
        l[g] = 0.f;
    }
    auto visit = [&](int j) {
        float kf[4], vf[4];
        const size_t row = (((size_t)b * N + j) * a.Hkv + kv) * kD + 4 * lane;
        load4(k + row, kf);
        load4(v + row, vf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float s = qf[g][0] * kf[0] + qf[g][1] * kf[1] + qf[g][2] * kf[2] + qf[g][3] * kf[3];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const float m_new = fmaxf(m[g], s);
            const float corr = exp2f(m[g] - m_new);   // 0 on the first key (m = -inf)
            const float p = exp2f(s - m_new);
            l[g] = l[g] * corr + p;
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[g][e] = acc[g][e] * corr + p * vf[e];
            m[g] = m_new;
        }
    };
    const int n_sink = min(a.sink, i + 1);
    for (int j = 0; j < n_sink; ++j) visit(j);
    for (int j = max(a.sink, i - a.recent + 1); j <= i; ++j) visit(j);

    const float al = alpha[kv];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        __nv_bfloat16* op = out + (((size_t)b * N + i) * a.Hq + kv * G + g) * kD + 4 * lane;
        float c[4];
        load4(op, c);
        const float inv = 1.f / l[g];   // the token itself is always visible: l >= 1
        float r[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) r[e] = al * c[e] + (1.f - al) * acc[g][e] * inv;
        store_row<__nv_bfloat16, 4>(op, r);
    }
}

template <int G>
cudaError_t launch_g(const LayerArgs& a, const float* alpha, const void* q, const void* k, const void* v, int N,
                     void* out, cudaStream_t s) {
    const long units = (long)a.B * N * a.Hkv;
    const long grid = (units + kWarps - 1) / kWarps;
    if (grid > 0x7fffffffL) return cudaErrorInvalidConfiguration;
    lambda_mix_kernel<G><<<(unsigned)grid, kWarps * 32, 0, s>>>(
        a, alpha, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), N, static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError();
}

}  // namespace

bool lambda_mix_supported(const LayerArgs& a) {
    return a.dtype == DUO_BF16 && a.D == kD && (a.G == 1 || a.G == 2 || a.G == 4 || a.G == 8);
}

cudaError_t launch_lambda_mix(const LayerArgs& a, const float* alpha, const void* q, const void* k, const void* v,
                              int N, void* out, cudaStream_t s) {
    if (N <= 0 || a.B <= 0) return cudaSuccess;
    switch (a.G) {
        case 1: return launch_g<1>(a, alpha, q, k, v, N, out, s);
        case 2: return launch_g<2>(a, alpha, q, k, v, N, out, s);
        case 4: return launch_g<4>(a, alpha, q, k, v, N, out, s);
        case 8: return launch_g<8>(a, alpha, q, k, v, N, out, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace duo
