// simt_attn.cu -- attention on the CUDA cores for the cases the tensor-core
// path does not take: fp32 data (tf32 would miss a 1e-4 bound) and head_dim
// 64.  Two modes:
//
//   mode 0, chunked pre-fill [Summary S2 "Chunked Pre-filling"]: the queries
//     of a chunk attend to the caches as they stand plus the chunk's own keys;
//     retrieval heads causally over the full cache, streaming heads under the
//     Lambda mask over the ring (positions from ring_pos) and the chunk, or in
//     whole-chunk mode over the ring and the chunk causally.
//   mode 1, gated mix [Review S3 "Core formula"]: every head over the whole
//     sequence, alpha * causal + (1 - alpha) * Lambda; one score per (query,
//     key) feeds both online-softmax states.
//   mode 2, gate gradient of the gated mix [Review S3 "Core formula",
//     "Retrieval-head identification": the gates are what training updates]:
//     the same two attentions per row, then dout . (causal - Lambda) summed
//     over the CTA's rows and added atomically into dalpha[kv].
//
// A CTA holds 32 query rows of one query head; four threads share a row, each
// with a quarter of the head dimension, and reduce the dot product with two
// shuffles.  Keys stream through shared memory 32 at a time, widened to fp32.
#include "common.cuh"
#include "internal.h"

namespace duo {
namespace {

constexpr int kRows = 32;
constexpr int kKeys = 32;
constexpr int kThreadsSimt = kRows * 4;

struct SimtArgs {
    const void* q;
    const void* k;        // chunk (mode 0) or whole sequence (mode 1)
    const void* v;
    void* out;
    const float* alpha;   // mode 1
    int n_tokens;         // C (mode 0) or N (modes 1, 2)
    int mode;
    const void* dout;     // mode 2: [B][N][Hq][D]
    float* dalpha;        // mode 2: [Hkv], accumulated
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreadsSimt) simt_attention_kernel(const LayerArgs a, const CacheArgs c,
                                                                      const SimtArgs s) {
    constexpr int QD = D / 4;  // elements per thread
    __shared__ float sK[kKeys][D];
    __shared__ float sV[kKeys][D];
    __shared__ int sPos[kKeys];

    const int b = blockIdx.z;
    const int qh_blk = blockIdx.y;                 // query head in block order: slot * G + g
    const int slot = qh_blk / a.G, g = qh_blk % a.G;
    const int q_idx = a.q_head0[slot] + g;         // caller's query-head index
    const int kv_idx = a.kv_head[slot];            // caller's KV-head index
    if (!bounds_ok(b < a.B && q_idx >= 0 && q_idx < a.Hq && kv_idx >= 0 && kv_idx < a.Hkv, c.status))
        return;                                    // debug build only; the same for the whole CTA
    const int r0 = blockIdx.x * kRows;
    const int row = r0 + (threadIdx.x >> 2);
    const int quarter = threadIdx.x & 3;
    const int N = s.n_tokens;
    const bool mix = s.mode >= 1;       // modes 1 and 2 run both attentions over the whole sequence
    const bool retrieval = slot < a.R;

    int c0 = 0;
    if (!mix) {
        c0 = c.seq_len[b];
        if (retrieval && c0 > a.capacity) c0 = a.capacity;
        if (c0 < 0) c0 = 0;
    }
    const int qpos = c0 + row;
    const bool row_ok = row < N;

    float q[QD];
    {
        const T* qp = static_cast<const T*>(s.q) + (((size_t)b * N + (row_ok ? row : 0)) * a.Hq + q_idx) * D + quarter * QD;
#pragma unroll
        for (int e = 0; e < QD; ++e) q[e] = Elem<T>::to_f32(qp[e]) * a.scale * kLog2e;
    }
    // two online-softmax states: 0 = the head's mask (mode 0) or causal
    // (mode 1); 1 = Lambda (mode 1 only)
    float m0 = kNegBig, l0 = 0.f, m1 = kNegBig, l1 = 0.f;
    float o0[QD], o1[QD];
#pragma unroll
    for (int e = 0; e < QD; ++e) o0[e] = o1[e] = 0.f;

    const int last_row = min(N, r0 + kRows);      // chunk rows visible to this CTA: [0, last_row)
    // key segments: 0 = prior keys from the caches (mode 0), 1..2 = chunk / sequence rows
    int seg_begin[3], seg_end[3];
    if (mix) {
        seg_begin[0] = seg_end[0] = 0;
        seg_begin[1] = 0; seg_end[1] = last_row;
        seg_begin[2] = seg_end[2] = 0;
    } else if (retrieval) {
        seg_begin[0] = 0; seg_end[0] = c0;
        seg_begin[1] = 0; seg_end[1] = last_row;
        seg_begin[2] = seg_end[2] = 0;
    } else if (a.stream_chunk) {
        seg_begin[0] = 0; seg_end[0] = a.W;                                    // ring slots
        seg_begin[1] = 0; seg_end[1] = last_row;                               // the whole chunk
        seg_begin[2] = seg_end[2] = 0;
    } else {
        seg_begin[0] = 0; seg_end[0] = a.W;                                    // ring slots
        const int sink_end = max(0, min(last_row, a.sink - c0));               // chunk sinks
        seg_begin[1] = 0; seg_end[1] = sink_end;
        seg_begin[2] = max(sink_end, r0 - a.recent + 1); seg_end[2] = last_row;  // recent band
        if (seg_begin[2] > seg_end[2]) seg_begin[2] = seg_end[2];
    }

    for (int seg = 0; seg < 3; ++seg) {
        for (int k0 = seg_begin[seg]; k0 < seg_end[seg]; k0 += kKeys) {
            const int nk = min(kKeys, seg_end[seg] - k0);
            __syncthreads();
            for (int i = threadIdx.x; i < kKeys * D; i += kThreadsSimt) {
                const int j = i / D, e = i % D;
                float kv = 0.f, vv = 0.f;
                int pos = -1;
                if (j < nk) {
                    const int kr = k0 + j;
                    const T* kp;
                    const T* vp;
                    if (seg == 0 && retrieval) {
                        const size_t off = (((size_t)b * a.R + slot) * a.capacity + kr) * D + e;
                        kp = static_cast<const T*>(c.k_full) + off;
                        vp = static_cast<const T*>(c.v_full) + off;
                        pos = kr;
                    } else if (seg == 0) {
                        const size_t off = (((size_t)b * a.S + (slot - a.R)) * a.W + kr) * D + e;
                        kp = static_cast<const T*>(c.k_ring) + off;
                        vp = static_cast<const T*>(c.v_ring) + off;
                        pos = c.ring_pos[(size_t)b * a.W + kr];
                        if (pos >= c0) pos = -1;   // only tokens before the chunk come from the ring
                    } else {
                        const size_t off = (((size_t)b * N + kr) * a.Hkv + kv_idx) * D + e;
                        kp = static_cast<const T*>(s.k) + off;
                        vp = static_cast<const T*>(s.v) + off;
                        pos = c0 + kr;
                    }
                    if (pos >= 0) {
                        kv = Elem<T>::to_f32(*kp);
                        vv = Elem<T>::to_f32(*vp);
                    }
                }
                sK[j][e] = kv;
                sV[j][e] = vv;
                if (e == 0) sPos[j] = pos;
            }
            __syncthreads();
            for (int j = 0; j < nk; ++j) {
                float part = 0.f;
#pragma unroll
                for (int e = 0; e < QD; ++e) part = fmaf(q[e], sK[j][quarter * QD + e], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                const int kp = sPos[j];
                const bool causal = kp >= 0 && kp <= qpos;
                const bool lam = causal && (kp < a.sink || (a.stream_chunk && !mix ? kp >= c0 - a.recent
                                                                                   : qpos - kp < a.recent));
                const bool vis0 = mix ? causal : (retrieval ? causal : lam);
                if (vis0) {
                    const float mn = fmaxf(m0, part);
                    const float cr = exp2f(m0 - mn), p = exp2f(part - mn);
                    l0 = l0 * cr + p;
#pragma unroll
                    for (int e = 0; e < QD; ++e) o0[e] = fmaf(p, sV[j][quarter * QD + e], o0[e] * cr);
                    m0 = mn;
                }
                if (mix && lam) {
                    const float mn = fmaxf(m1, part);
                    const float cr = exp2f(m1 - mn), p = exp2f(part - mn);
                    l1 = l1 * cr + p;
#pragma unroll
                    for (int e = 0; e < QD; ++e) o1[e] = fmaf(p, sV[j][quarter * QD + e], o1[e] * cr);
                    m1 = mn;
                }
            }
        }
    }
    if (s.mode == 2) {
        // this row's dout . (causal - Lambda), then the CTA's sum, once per CTA
        __shared__ float sPart[kThreadsSimt / 32];
        float part = 0.f;
        if (row_ok) {
            const T* dp = static_cast<const T*>(s.dout) + (((size_t)b * N + row) * a.Hq + q_idx) * D + quarter * QD;
#pragma unroll
            for (int e = 0; e < QD; ++e)
                part = fmaf(Elem<T>::to_f32(dp[e]), (l0 > 0.f ? o0[e] / l0 : 0.f) - (l1 > 0.f ? o1[e] / l1 : 0.f), part);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if ((threadIdx.x & 31) == 0) sPart[threadIdx.x >> 5] = part;
        __syncthreads();
        if (threadIdx.x == 0) {
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kThreadsSimt / 32; ++w) sum += sPart[w];
            atomicAdd(&s.dalpha[kv_idx], sum);
        }
        return;
    }
    if (!row_ok) return;
    float res[QD];
    if (mix) {
        const float al = s.alpha[kv_idx];
#pragma unroll
        for (int e = 0; e < QD; ++e)
            res[e] = al * (l0 > 0.f ? o0[e] / l0 : 0.f) + (1.f - al) * (l1 > 0.f ? o1[e] / l1 : 0.f);
    } else {
#pragma unroll
        for (int e = 0; e < QD; ++e) res[e] = l0 > 0.f ? o0[e] / l0 : 0.f;
    }
    T* op = static_cast<T*>(s.out) + (((size_t)b * N + row) * a.Hq + q_idx) * D + quarter * QD;
#pragma unroll
    for (int e = 0; e < QD; ++e) op[e] = Elem<T>::from_f32(res[e]);
}

template <typename T, int D>
cudaError_t launch_simt_t(const LayerArgs& a, const CacheArgs& c, const SimtArgs& s, cudaStream_t st) {
    dim3 grid((s.n_tokens + kRows - 1) / kRows, a.Hq, a.B);
    simt_attention_kernel<T, D><<<grid, kThreadsSimt, 0, st>>>(a, c, s);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_attention(const LayerArgs& a, const CacheArgs* c, const float* alpha, const void* q,
                                  const void* k, const void* v, int n_tokens, void* out, int mode, cudaStream_t st,
                                  const void* dout, float* dalpha) {
    SimtArgs s{q, k, v, out, alpha, n_tokens, mode, dout, dalpha};
    CacheArgs cc{};
    if (c) cc = *c;
    if (a.B > 65535 || a.Hq > 65535) return cudaErrorInvalidConfiguration;
    if (a.dtype == DUO_BF16) {
        if (a.D == 128) return launch_simt_t<__nv_bfloat16, 128>(a, cc, s, st);
        return launch_simt_t<__nv_bfloat16, 64>(a, cc, s, st);
    }
    if (a.D == 128) return launch_simt_t<float, 128>(a, cc, s, st);
    return launch_simt_t<float, 64>(a, cc, s, st);
}

}  // namespace duo
