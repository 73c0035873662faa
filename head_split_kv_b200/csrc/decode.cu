// decode.cu -- duo_decode_attn: one new token per sequence attends over its
// caches, retrieval and streaming heads in a single launch.
//
// [Review S3 "Inference flow", decode: the new token's Q/K/V are split along
// the head dimension, each part is attended against its own cache, and the
// per-head results are concatenated before the output projection.]
//
// Work units (one CTA each, one 1-D grid):
//   retrieval: (sequence b, retrieval slot r, split s) -- rows
//              [s*chunk, (s+1)*chunk) of the full cache, chunk derived on the
//              device from seq_len[b], so the launch shape does not depend on
//              the length;
//   streaming: (sequence b, streaming slot) -- the min(seq_len, W) ring rows.
// The G query heads of the KV head share every K/V tile.
//
// Per CTA: warp 4 is the producer -- one lane issues cp.async.bulk copies
// (the TMA engine, no tensor map needed: K/V rows of one head are contiguous,
// or one 64-token page) into a STAGES-deep ring of 64-key shared-memory tiles,
// signalled through mbarriers.  Warps 0-3 consume: warp w takes keys
// [16w, 16w+16) of each tile, half-warp h keys 16w + 8h + (0..7); each lane
// holds D/16 elements of q (pre-scaled by scale*log2 e) and of the output
// accumulator for every query head of the group.  Dot products are reduced
// across the 16 lanes by a transposed butterfly (8 keys in 8 shuffles instead
// of 32), each warp keeps its own online-softmax state, and the four states
// are merged at the end.  With several splits, each CTA stores (m, l, o) to
// the workspace and the last CTA of the (b, r) pair -- found with an atomic
// ticket, never a wait -- combines them and writes the output.
#include "common.cuh"
#include "internal.h"

namespace duo {
namespace {

constexpr int kTile = 64;            // keys per pipeline stage
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

struct DecodeArgs {
    const void* q;
    void* out;
    float* partial;      // [B*R][nsplit][G][D + 2]: m, l, o[D]
    uint32_t* ticket;    // [B*R]
    int nsplit;
    int n_ret_units;     // B * R * nsplit
};

template <typename T, int D>
struct Cfg {
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kTileBytes = kTile * kRowBytes;
    static constexpr int kStagesRaw = 98304 / (2 * kTileBytes);
    static constexpr int kStages = kStagesRaw < 2 ? 2 : (kStagesRaw > 6 ? 6 : kStagesRaw);
    static constexpr int kEPL = D / 16;  // elements per lane
};

template <typename T, int D, int G>
constexpr size_t decode_smem_bytes() {
    using C = Cfg<T, D>;
    size_t s = 2 * (size_t)C::kStages * C::kTileBytes;     // K and V stages
    s += (size_t)kConsumerWarps * 16 * G * sizeof(float);   // probabilities
    s += 2 * C::kStages * sizeof(uint64_t) + 64;            // barriers, flag, rows per stage
    return s + 1024;                                        // alignment slack
}

// Transposed butterfly over the 16 lanes of a half-warp: on entry v[j] is this
// lane's partial dot for key j (j < 8); on exit v[0] is the full dot of key
// ((lane & 15) >> 1), held by lanes 2k and 2k+1.
__device__ __forceinline__ float reduce8_transposed(float (&v)[8], int lane) {
    const bool b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b3 ? v[i] : v[i + 4];
        const float keep = b3 ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b2 ? v[i] : v[i + 2];
        const float keep = b2 ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    {
        const float send = b1 ? v[0] : v[1];
        const float keep = b1 ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    return v[0];
}

template <typename T, int D, int G, bool PAGED>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const LayerArgs a, const CacheArgs c, const DecodeArgs d) {
    using C = Cfg<T, D>;
    constexpr int EPL = C::kEPL;
    constexpr int STAGES = C::kStages;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    T* sK = reinterpret_cast<T*>(smem);
    T* sV = reinterpret_cast<T*>(smem + (size_t)STAGES * C::kTileBytes);
    float* sP = reinterpret_cast<float*>(smem + 2 * (size_t)STAGES * C::kTileBytes);  // [warp][16 keys][G]
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sP + kConsumerWarps * 16 * G);
    uint64_t* empty_bar = full_bar + STAGES;
    int* s_flag = reinterpret_cast<int*>(empty_bar + STAGES);
    int* s_tile_n = s_flag + 1;  // valid rows of each stage, written by the producer before its arrive

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---------------------------------------------------------- work unit
    const bool retrieval = (int)blockIdx.x < d.n_ret_units;
    int b, slot, split = 0;
    if (retrieval) {
        split = blockIdx.x % d.nsplit;
        const int pair = blockIdx.x / d.nsplit;
        slot = pair % a.R;
        b = pair / a.R;
    } else {
        const int u = blockIdx.x - d.n_ret_units;
        slot = a.R + u % a.S;
        b = u / a.S;
    }
    int len = c.seq_len[b];
    int row_begin = 0, row_end = 0;
    const T* k_base;
    const T* v_base;
    if (retrieval) {
        if (len > a.capacity || len < 0) {
            if (threadIdx.x == 0 && split == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
            len = len < 0 ? 0 : a.capacity;
        }
        const int per = (len + d.nsplit - 1) / d.nsplit;
        const int chunk = (per + kTile - 1) / kTile * kTile;
        row_begin = min(len, split * chunk);
        row_end = min(len, row_begin + chunk);
        if (PAGED) {
            k_base = static_cast<const T*>(c.k_full);
            v_base = static_cast<const T*>(c.v_full);
        } else {
            const size_t off = ((size_t)b * a.R + slot) * a.capacity * D;
            k_base = static_cast<const T*>(c.k_full) + off;
            v_base = static_cast<const T*>(c.v_full) + off;
        }
    } else {
        row_end = len < 0 ? 0 : min(len, a.W);
        const size_t off = ((size_t)b * a.S + (slot - a.R)) * a.W * D;
        k_base = static_cast<const T*>(c.k_ring) + off;
        v_base = static_cast<const T*>(c.v_ring) + off;
    }
    const int n_tiles = (row_end - row_begin + kTile - 1) / kTile;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kConsumerWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            for (int t = 0; t < n_tiles; ++t) {
                const int st = t % STAGES, round = t / STAGES;
                if (round > 0 && !mbar_wait(&empty_bar[st], (round - 1) & 1, c.status)) break;
                const int r0 = row_begin + t * kTile;
                const int n = min(kTile, row_end - r0);
                const uint32_t bytes = (uint32_t)n * C::kRowBytes;
                const T* ks;
                const T* vs;
                bool ok = true;
                if (PAGED && retrieval) {
                    const int pg = c.page_table[(size_t)b * a.max_pages + r0 / kTile];
                    if (pg < 0 || pg >= a.n_pages) {
                        atomicOr(c.status, DUO_DEV_BAD_PAGE);
                        ok = false;
                    }
                    const size_t off = ((size_t)(ok ? pg : 0) * a.R + slot) * (size_t)kTile * D;
                    ks = k_base + off;
                    vs = v_base + off;
                } else {
                    ks = k_base + (size_t)r0 * D;
                    vs = v_base + (size_t)r0 * D;
                }
                s_tile_n[st] = ok ? n : 0;
                if (ok) {
                    mbar_arrive_expect_tx(&full_bar[st], 2 * bytes);
                    bulk_g2s(sK + (size_t)st * kTile * D, ks, bytes, &full_bar[st]);
                    bulk_g2s(sV + (size_t)st * kTile * D, vs, bytes, &full_bar[st]);
                } else {
                    mbar_arrive(&full_bar[st]);  // an empty tile: every key of it is masked
                }
            }
        }
        // the producer warp joins the merge below only through __syncthreads
    }

    // ------------------------------------------------------ consumers
    float o[G][EPL];
    float m_run[G], l_run[G];
    const int hw = lane >> 4;        // half-warp
    const int dl = lane & 15;        // lane within the half-warp: owns d-slice [dl*EPL, dl*EPL+EPL)
    if (warp < kConsumerWarps) {
        float q[G][EPL];
        const T* qp = static_cast<const T*>(d.q) + ((size_t)b * a.Hq + a.q_head0[slot]) * D + dl * EPL;
        const float qs = a.scale * kLog2e;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            load_row_f32<T, EPL>(qp + (size_t)g * D, q[g]);
#pragma unroll
            for (int e = 0; e < EPL; ++e) q[g][e] *= qs;
            m_run[g] = kNegBig;
            l_run[g] = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[g][e] = 0.f;
        }
        float* myP = sP + warp * 16 * G;
        const int kidx = (lane & 15) >> 1;  // key this lane scores after the butterfly

        for (int t = 0; t < n_tiles; ++t) {
            const int st = t % STAGES, round = t / STAGES;
            if (!mbar_wait(&full_bar[st], round & 1, c.status)) break;
            const int n = s_tile_n[st];
            const T* tK = sK + (size_t)st * kTile * D;
            const T* tV = sV + (size_t)st * kTile * D;
            const int key0 = warp * 16 + hw * 8;    // first key of this half-warp in the tile

            // scores: s[g] of key key0 + kidx
            float s[G];
#pragma unroll
            for (int g = 0; g < G; ++g) s[g] = 0.f;
            {
                float part[G][8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float kf[EPL];
                    load_row_f32<T, EPL>(tK + (size_t)(key0 + j) * D + dl * EPL, kf);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < EPL; ++e) acc = fmaf(q[g][e], kf[e], acc);
                        part[g][j] = acc;
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) s[g] = reduce8_transposed(part[g], lane);
            }
            const bool valid = key0 + kidx < n;
            float m_new[G], corr[G], p[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float sv = valid ? s[g] : kNegBig;
                float mt = sv;
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                m_new[g] = fmaxf(m_run[g], mt);
                corr[g] = exp2f(m_run[g] - m_new[g]);
                p[g] = valid ? exp2f(sv - m_new[g]) : 0.f;
                m_run[g] = m_new[g];
                l_run[g] = l_run[g] * corr[g] + ((lane & 1) ? 0.f : p[g]);
#pragma unroll
                for (int e = 0; e < EPL; ++e) o[g][e] *= corr[g];
            }
            if ((lane & 1) == 0) {
#pragma unroll
                for (int g = 0; g < G; ++g) myP[(hw * 8 + kidx) * G + g] = p[g];
            }
            __syncwarp();
            // o += p v over this half-warp's keys
            const int nh = min(8, n - key0);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j < nh) {
                    float vf[EPL];
                    load_row_f32<T, EPL>(tV + (size_t)(key0 + j) * D + dl * EPL, vf);
                    const float* pj = myP + (hw * 8 + j) * G;
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float pg = pj[g];
#pragma unroll
                        for (int e = 0; e < EPL; ++e) o[g][e] = fmaf(pg, vf[e], o[g][e]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }
        // merge the two half-warps (same running max within a warp)
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[g][e] += __shfl_xor_sync(0xffffffffu, o[g][e], 16);
            float l = l_run[g];
            l += __shfl_xor_sync(0xffffffffu, l, 1);
            l += __shfl_xor_sync(0xffffffffu, l, 2);
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            l_run[g] = l;
        }
    }
    __syncthreads();  // all tiles consumed: the stage buffers are free

    // ---------------------------------------------- merge the 4 warp states
    // layout in the (now free) K stages: [warp][G][D + 2]
    float* sM = reinterpret_cast<float*>(sK);
    constexpr int STRIDE = D + 2;
    if (warp < kConsumerWarps) {
        float* dst = sM + (size_t)warp * G * STRIDE;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (lane < 16) {
#pragma unroll
                for (int e = 0; e < EPL; ++e) dst[g * STRIDE + 2 + dl * EPL + e] = o[g][e];
            }
            if (lane == 0) {
                dst[g * STRIDE + 0] = m_run[g];
                dst[g * STRIDE + 1] = l_run[g];
            }
        }
    }
    __syncthreads();
    // the CTA's combined state, one (g, element) per thread step; stored in
    // slot [kConsumerWarps] of sM
    float* cta = sM + (size_t)kConsumerWarps * G * STRIDE;
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
        const int g = i / D, e = i % D;
        float M = kNegBig;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sM[(w * G + g) * STRIDE]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float sc = exp2f(sM[(w * G + g) * STRIDE] - M);
            L += sc * sM[(w * G + g) * STRIDE + 1];
            O += sc * sM[(w * G + g) * STRIDE + 2 + e];
        }
        cta[g * STRIDE + 2 + e] = O;
        if (e == 0) {
            cta[g * STRIDE + 0] = M;
            cta[g * STRIDE + 1] = L;
        }
    }
    __syncthreads();

    T* outp = static_cast<T*>(d.out) + ((size_t)b * a.Hq + a.q_head0[slot]) * D;
    if (!retrieval || d.nsplit == 1) {
        for (int i = threadIdx.x; i < G * D; i += kThreads) {
            const int g = i / D, e = i % D;
            const float L = cta[g * STRIDE + 1];
            const float v = L > 0.f ? cta[g * STRIDE + 2 + e] / L : 0.f;
            outp[(size_t)g * D + e] = Elem<T>::from_f32(v);
        }
        return;
    }

    // ------------------------------------------------ split-K combine
    const size_t pair = (size_t)b * a.R + slot;
    float* mine = d.partial + (pair * d.nsplit + split) * (size_t)G * STRIDE;
    for (int i = threadIdx.x; i < G * STRIDE; i += kThreads) mine[i] = cta[i];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned tk = atomicAdd(&d.ticket[pair], 1u);
        *s_flag = (tk == (unsigned)d.nsplit - 1);
    }
    __syncthreads();
    if (!*s_flag) return;
    __threadfence();
    const float* all = d.partial + pair * d.nsplit * (size_t)G * STRIDE;
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
        const int g = i / D, e = i % D;
        float M = kNegBig;
        for (int sp = 0; sp < d.nsplit; ++sp) M = fmaxf(M, __ldcg(all + ((size_t)sp * G + g) * STRIDE));
        float L = 0.f, O = 0.f;
        for (int sp = 0; sp < d.nsplit; ++sp) {
            const float* ps = all + ((size_t)sp * G + g) * STRIDE;
            const float sc = exp2f(__ldcg(ps) - M);
            L += sc * __ldcg(ps + 1);
            O += sc * __ldcg(ps + 2 + e);
        }
        outp[(size_t)g * D + e] = Elem<T>::from_f32(L > 0.f ? O / L : 0.f);
    }
    if (threadIdx.x == 0) d.ticket[pair] = 0u;  // leave the workspace ready for the next call
}

template <typename T, int D, int G, bool PAGED>
cudaError_t launch_t(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d, int grid, cudaStream_t s) {
    constexpr size_t smem = decode_smem_bytes<T, D, G>();
    auto kern = decode_kernel<T, D, G, PAGED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, s>>>(a, c, d);
    return cudaGetLastError();
}

template <typename T, int D, int G>
cudaError_t launch_g(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d, int grid, cudaStream_t s) {
    if (a.page_size) return launch_t<T, D, G, true>(a, c, d, grid, s);
    return launch_t<T, D, G, false>(a, c, d, grid, s);
}

template <typename T, int D>
cudaError_t launch_d(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d, int grid, cudaStream_t s) {
    switch (a.G) {
        case 1: return launch_g<T, D, 1>(a, c, d, grid, s);
        case 2: return launch_g<T, D, 2>(a, c, d, grid, s);
        case 4: return launch_g<T, D, 4>(a, c, d, grid, s);
        case 8: return launch_g<T, D, 8>(a, c, d, grid, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const LayerArgs& a, const CacheArgs& c, const DecodePlan& plan, const void* q, void* out,
                          void* workspace, cudaStream_t s) {
    DecodeArgs d;
    d.q = q;
    d.out = out;
    d.partial = static_cast<float*>(workspace);
    d.ticket = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + plan.ticket_offset);
    d.nsplit = plan.nsplit;
    d.n_ret_units = a.B * a.R * plan.nsplit;
    const long grid = (long)d.n_ret_units + (long)a.B * a.S;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffffL) return cudaErrorInvalidConfiguration;
    if (a.dtype == DUO_BF16) {
        if (a.D == 128) return launch_d<__nv_bfloat16, 128>(a, c, d, (int)grid, s);
        return launch_d<__nv_bfloat16, 64>(a, c, d, (int)grid, s);
    }
    if (a.D == 128) return launch_d<float, 128>(a, c, d, (int)grid, s);
    return launch_d<float, 64>(a, c, d, (int)grid, s);
}

}  // namespace duo
