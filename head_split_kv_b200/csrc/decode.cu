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
// signalled through mbarriers.  NW consumer warps (8 for query groups of 1
// or 2, 4 for larger groups, whose accumulators need more registers) split
// each tile: warp w takes keys [KW*w, KW*w + KW) with KW = 64 / NW, half-warp
// h the KH = KW / 2 keys after KW*w + KH*h; each lane holds D/16 elements of
// q (pre-scaled by scale*log2 e) and of the output accumulator for every
// query head of the group.  Dot products are reduced across the 16 lanes by a
// transposed butterfly (KH keys in KH + log2(16/KH) - 1 shuffles instead of
// 4*KH), each warp keeps its own online-softmax state, and the warp states
// are merged at the end.  With several splits, each CTA stores (m, l, o) to
// the workspace and the last CTA of the (b, r) pair -- found with an atomic
// ticket, never a wait -- combines them and writes the output.
//
// duo_decode_step runs the same kernel with the append fused in: the CTA
// whose rows include the new token's position splices the token into its
// shared-memory tile straight from the call's k/v inputs and stores it into
// the cache (full-cache row or ring slot), and the last CTA of the grid
// advances seq_len, so one launch does duo_append_kv(T = 1) + decode.
#include <utility>

#include "common.cuh"
#include "internal.h"
#include "kvq4.cuh"
#include "kvq8.cuh"

namespace duo {
namespace {

constexpr int kTile = 64;            // keys per pipeline stage

// consumer warps per CTA for a query group of G heads
__host__ __device__ constexpr int consumer_warps(int G) { return G <= 2 ? 8 : 4; }

struct DecodeArgs {
    const void* q;
    void* out;
    float* partial;      // [B*R][nsplit][G][D + 4]: m, l, -, -, o[D]
    uint32_t* ticket;    // [B*R]
    int nsplit;
    int n_ret_units;     // B * R * nsplit
    // Fused append (duo_decode_step): the new token's K/V rows [B][Hkv][D];
    // NULL for plain decode.
    const void* k_new;
    const void* v_new;
    uint32_t* grid_ticket;  // one state counter word: the last CTA advances seq_len
    uint32_t* tile_ctr;     // [B*R]: tiles handed out past the static ones (tensor-core bf16 kernel)
    int draw;               // draw tiles from tile_ctr: only when the whole grid is resident at once
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
    s += (size_t)kTile * G * sizeof(float);                  // probabilities of one tile
    s += (2 * C::kStages + 1) * sizeof(uint64_t) + 64;      // barriers, flag, rows per stage
    return s + 1024;                                        // alignment slack
}

// Transposed butterfly over the 16 lanes of a half-warp: on entry v[j] is this
// lane's partial dot for key j (j < K, K = 8 or 4); on exit the return value
// is the full dot of key ((lane & 15) >> (4 - log2 K)), held by the 16/K
// lanes that share those high bits.
template <int K>
__device__ __forceinline__ float reduce_transposed(float (&v)[K], int lane) {
    static_assert(K == 8 || K == 4, "4 or 8 keys per half-warp");
    const bool b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int i = 0; i < K / 2; ++i) {
        const float send = b3 ? v[i] : v[i + K / 2];
        const float keep = b3 ? v[i + K / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < K / 4; ++i) {
        const float send = b2 ? v[i] : v[i + K / 4];
        const float keep = b2 ? v[i + K / 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    if (K == 8) {
        const float send = b1 ? v[0] : v[1];
        const float keep = b1 ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    return v[0];
}

// Registers per thread that let two CTAs share an SM: 65536 / (2 * threads),
// rounded down to the allocation granularity of 8.
__host__ __device__ constexpr int decode_max_regs(int G) {
    return (65536 / (2 * (consumer_warps(G) + 1) * 32)) / 8 * 8;
}

// With a fused append every CTA reads its sequence's length once (thread 0,
// broadcast through shared memory) and then takes a grid-wide ticket; the
// CTA that takes the last ticket knows every CTA has read the old lengths and
// advances them.  Taken at the start, this stays off the kernel's tail.
// Atomic add at GPU scope with acquire-release semantics.  The release half
// orders the calling thread's earlier memory accesses -- and, after a CTA
// barrier, those of the whole CTA (release is cumulative) -- before the add;
// the acquire half orders its later accesses after it.  A chain of such adds
// on one counter therefore hands every earlier adder's writes to the last
// one, with one round trip to L2 instead of a full fence plus the atomic.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Called by the thread that read seq_len, after it read it: the CTA that
// takes the last ticket of the grid advances every sequence's length.  The
// release half of each add orders that CTA's read of seq_len before its
// ticket; the acquire half of the last add orders the increments after every
// CTA's read.  The counter is reset for the next launch, which waits for this
// grid to complete before it reads the counter.
__device__ __forceinline__ void length_ticket(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d) {
    const unsigned tk = atom_add_acq_rel_gpu(d.grid_ticket, 1u);
    if (tk == gridDim.x - 1) {
        for (int bb = 0; bb < a.B; ++bb) atomicAdd(&c.seq_len[bb], 1);
        *d.grid_ticket = 0u;
    }
}

// The end of a decode CTA, shared by both decode kernels.  On entry every
// consumer warp w has stored its online-softmax state for each query head g
// of the group into sM[w][g][D + 4] (m, l, -, -, o[D]) and the CTA has
// synchronised; the K/V stage buffers (kStageBytes from sM) are free.  Merges
// the warp states, then writes the output (streaming heads, single split) or
// stores the split-K record and, in the last CTA of the (sequence, head)
// pair, combines all splits.
template <typename T, int D, int G, int NW, int kThreads, size_t kStageBytes>
__device__ __forceinline__ void decode_finish(float* sM, uint64_t* comb_bar, int* s_flag, const LayerArgs& a,
                                              const CacheArgs& c, const DecodeArgs& d, int b, int slot, int split,
                                              bool retrieval, bool fused) {
    constexpr int STRIDE = D + 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the CTA's combined state, in slot [NW] of sM
    float* cta = sM + (size_t)NW * G * STRIDE;
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
        const int g = i / D, e = i % D;
        float M = kNegBig;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, sM[(w * G + g) * STRIDE]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float sc = exp2f(sM[(w * G + g) * STRIDE] - M);
            L += sc * sM[(w * G + g) * STRIDE + 1];
            O += sc * sM[(w * G + g) * STRIDE + 4 + e];
        }
        cta[g * STRIDE + 4 + e] = O;
        if (e == 0) {
            cta[g * STRIDE + 0] = M;
            cta[g * STRIDE + 1] = L;
        }
    }
    __syncthreads();

    T* outp = static_cast<T*>(d.out) + ((size_t)b * a.Hq + a.q_head0[slot]) * D;
    if (!bounds_ok(b < a.B && a.q_head0[slot] >= 0 && a.q_head0[slot] + G <= a.Hq, c.status)) return;
    if (!retrieval || d.nsplit == 1) {
        for (int i = threadIdx.x; i < G * D; i += kThreads) {
            const int g = i / D, e = i % D;
            const float L = cta[g * STRIDE + 1];
            const float v = L > 0.f ? cta[g * STRIDE + 4 + e] / L : 0.f;
            outp[(size_t)g * D + e] = Elem<T>::from_f32(v);
        }
        return;
    }

    // ------------------------------------------------ split-K combine
    const size_t pair = (size_t)b * a.R + slot;
    // the record, the ticket and the combine's weights ([128][G] in shared memory)
    if (!bounds_ok(pair < (size_t)a.B * a.R && split < d.nsplit && d.nsplit <= 128, c.status)) return;
    float* mine = d.partial + (pair * d.nsplit + split) * (size_t)G * STRIDE;
    for (int i = threadIdx.x; i < G * STRIDE; i += kThreads) mine[i] = cta[i];
    // The barrier orders every thread's record stores before thread 0's
    // acquire-release ticket; the CTA that takes the last ticket thus sees
    // every split's record, and its second barrier passes them on to its
    // other threads.
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned tk = atom_add_acq_rel_gpu(&d.ticket[pair], 1u);
        *s_flag = (tk == (unsigned)d.nsplit - 1);
    }
    __syncthreads();
    if (!*s_flag) {
        return;
    }
    // This CTA is the last of its (b, r) pair: every split's record is in
    // global memory (L2).  (1) The first batch of records starts streaming
    // into the free stage buffers with a bulk copy (the TMA engine moves
    // them at L2 bandwidth) while (2) the splits' m and l, read from L2, give
    // the per-head maximum, each split's weight and 1 / L.  (3) Each thread
    // accumulates float4 quads of outputs over its share of the splits, a
    // batch of records at a time; where a group has fewer quads than there
    // are threads (MHA: 32 quads), the splits are dealt out to TP threads
    // per quad and their partial sums added at the end.
    const float* all = d.partial + pair * d.nsplit * (size_t)G * STRIDE;
    const int ns = d.nsplit;
    float* s_w = sM;                            // [ns][G] weights (the stage buffers are free)
    float* s_inv = s_w + 128 * G;               // [G] 1 / L (ns <= 128)
    constexpr int kRecFloats = G * STRIDE;      // one split's record
    constexpr size_t kHead = ((128 * G + G) * sizeof(float) + 1023) / 1024 * 1024;
    constexpr int kBatch = (int)((kStageBytes - kHead) / (kRecFloats * sizeof(float)));
    static_assert(kBatch >= 1, "a split-K record must fit in the stage buffers");
    float* stage = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sM) + kHead);
    constexpr int kQuads = G * D / 4;                            // float4 outputs of the group
    constexpr int TP = kQuads >= kThreads ? 1 : kThreads / kQuads;  // threads per quad
    auto issue_batch = [&](int b0) {
        const int nb = min(kBatch, ns - b0);
        const uint32_t bytes = (uint32_t)(nb * kRecFloats * sizeof(float));
        fence_proxy_async_smem();  // earlier thread accesses of this space before the async-proxy writes
        // the records were written through the generic proxy; the bulk copy reads them through the async one
        asm volatile("fence.proxy.async.global;" ::: "memory");
        mbar_arrive_expect_tx(comb_bar, bytes);
        bulk_g2s(stage, all + (size_t)b0 * kRecFloats, bytes, comb_bar);
    };
    if (threadIdx.x == 0) issue_batch(0);
    // one warp per query head of the group (two for the first warps when G
    // exceeds the warp count), a lane per split and per split + 32, + 64,
    // + 96: every (m, l) pair the warp needs is loaded at once, so the pass
    // costs one round trip to L2; the maximum and the sum are warp reductions
    constexpr int kWarps = kThreads / 32;
    constexpr int kHPW = (G + kWarps - 1) / kWarps;             // query heads per warp
    float2 ml[kHPW][4];
#pragma unroll
    for (int h = 0; h < kHPW; ++h) {
        const int g = warp + h * kWarps;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int sp = lane + 32 * j;
            ml[h][j] = (g < G && sp < ns)
                           ? __ldcg(reinterpret_cast<const float2*>(all + (size_t)sp * kRecFloats + g * STRIDE))
                           : make_float2(kNegBig, 0.f);
        }
    }
#pragma unroll
    for (int h = 0; h < kHPW; ++h) {
        const int g = warp + h * kWarps;
        if (g >= G) break;                                      // warp-uniform
        float M = fmaxf(fmaxf(ml[h][0].x, ml[h][1].x), fmaxf(ml[h][2].x, ml[h][3].x));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int sp = lane + 32 * j;
            if (sp < ns) {
                const float w = exp2f(ml[h][j].x - M);
                s_w[sp * G + g] = w;
                L += w * ml[h][j].y;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (lane == 0) s_inv[g] = L > 0.f ? 1.f / L : 0.f;
    }
    __syncthreads();
    constexpr int kQPer = (kQuads + kThreads - 1) / kThreads;     // quads per thread (TP == 1)
    float4 acc[kQPer];
#pragma unroll
    for (int k = 0; k < kQPer; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int sub = (int)threadIdx.x / kQuads;                    // this thread's share of the splits (TP > 1)
    uint32_t phase = 0;
    for (int b0 = 0; b0 < ns; b0 += kBatch) {
        const int nb = min(kBatch, ns - b0);
        // a CTA-uniform decision: no thread may leave while others wait at a barrier
        if (!__syncthreads_and(mbar_wait(comb_bar, phase, c.status))) return;
        phase ^= 1;
#pragma unroll
        for (int k = 0; k < kQPer; ++k) {
            const int qd = TP > 1 ? (int)threadIdx.x % kQuads : (int)threadIdx.x + k * kThreads;
            if (qd < kQuads && (TP == 1 || sub < TP)) {
                const int g = (4 * qd) / D, e = (4 * qd) % D;
                float4 v = acc[k];
                for (int sp = TP > 1 ? sub : 0; sp < nb; sp += TP) {
                    const float w = s_w[(b0 + sp) * G + g];
                    const float4 x = *reinterpret_cast<const float4*>(stage + sp * kRecFloats + g * STRIDE + 4 + e);
                    v.x = fmaf(w, x.x, v.x);
                    v.y = fmaf(w, x.y, v.y);
                    v.z = fmaf(w, x.z, v.z);
                    v.w = fmaf(w, x.w, v.w);
                }
                acc[k] = v;
            }
        }
        __syncthreads();  // the next batch overwrites the staging area
        if (threadIdx.x == 0 && b0 + kBatch < ns) issue_batch(b0 + kBatch);
    }
    if constexpr (TP > 1) {
        // add the TP partial sums of each quad (the staging area is free)
        float4* part = reinterpret_cast<float4*>(stage);
        if (sub < TP) part[sub * kQuads + (int)threadIdx.x % kQuads] = acc[0];
        __syncthreads();
        if ((int)threadIdx.x < kQuads) {
            float4 v = part[threadIdx.x];
            for (int t = 1; t < TP; ++t) {
                const float4 x = part[t * kQuads + threadIdx.x];
                v.x += x.x;
                v.y += x.y;
                v.z += x.z;
                v.w += x.w;
            }
            acc[0] = v;
        }
    }
#pragma unroll
    for (int k = 0; k < kQPer; ++k) {
        const int qd = (int)threadIdx.x + k * kThreads;
        if (qd < kQuads) {
            const float inv = s_inv[(4 * qd) / D];
            const float v[4] = {acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv};
            store_row<T, 4>(outp + 4 * qd, v);
        }
    }
    if (threadIdx.x == 0) {                     // leave the workspace ready for the next call
        d.ticket[pair] = 0u;
        if (d.tile_ctr) d.tile_ctr[pair] = 0u;
    }
}

template <typename T, int D, int G, bool PAGED>
__global__ void __maxnreg__(decode_max_regs(G))
    decode_kernel(const LayerArgs a, const CacheArgs c, const DecodeArgs d) {
    using C = Cfg<T, D>;
    constexpr int EPL = C::kEPL;
    constexpr int STAGES = C::kStages;
    constexpr int NW = consumer_warps(G);     // consumer warps
    constexpr int kThreads = (NW + 1) * 32;
    constexpr int KW = kTile / NW;            // keys per warp and tile
    constexpr int KH = KW / 2;                // keys per half-warp
    constexpr int DUP = 16 / KH;              // lanes holding the same key after the butterfly

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    T* sK = reinterpret_cast<T*>(smem);
    T* sV = reinterpret_cast<T*>(smem + (size_t)STAGES * C::kTileBytes);
    float* sP = reinterpret_cast<float*>(smem + 2 * (size_t)STAGES * C::kTileBytes);  // [warp][KW keys][G]
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sP + kTile * G);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* comb_bar = empty_bar + STAGES;     // bulk loads of the split-K records
    int* s_flag = reinterpret_cast<int*>(comb_bar + 1);
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
    // With a fused append the new token (position L0 = seq_len[b]) goes to
    // full-cache row L0 or ring slot ring_slot(L0) -- `new_row` -- and is read
    // from k_new / v_new; every other row comes from the caches.
    const bool fused = d.k_new != nullptr;
    // launched with programmatic stream serialization: let the next launch's
    // CTAs take SM slots as ours free, and wait for the previous grid before
    // the first read of anything it may have written
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) *s_flag = c.seq_len[b];
    __syncthreads();
    const int L0 = *s_flag;
    if (fused && threadIdx.x == 0) length_ticket(a, c, d);
    int len = L0;
    int new_row = -1;
    const T* kn = nullptr;
    const T* vn = nullptr;
    if (fused) {
        kn = static_cast<const T*>(d.k_new) + ((size_t)b * a.Hkv + a.kv_head[slot]) * D;
        vn = static_cast<const T*>(d.v_new) + ((size_t)b * a.Hkv + a.kv_head[slot]) * D;
        if (L0 < 0) {
            if (threadIdx.x == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
            len = 0;
        } else if (retrieval && L0 >= a.capacity) {
            if (threadIdx.x == 0 && split == 0) atomicOr(c.status, DUO_DEV_FULL_CACHE_OVERFLOW);
        } else {
            new_row = retrieval ? L0 : ring_slot(L0, a.sink, a.recent);
            len = L0 + 1;
        }
    }
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
            mbar_init(&empty_bar[s], NW);
        }
        mbar_init(comb_bar, 1);
        fence_barrier_init();
    }
    __syncthreads();

    // the CTA that covers the new token's row stores it into its cache
    const bool owns_new = new_row >= 0 && (!retrieval || (new_row >= row_begin && new_row < row_end));
    if (warp == NW && owns_new && bounds_ok(new_row < (retrieval ? a.capacity : a.W), c.status)) {
        T* dk = nullptr;
        T* dv = nullptr;
        if (!retrieval) {
            const size_t off = (((size_t)b * a.S + (slot - a.R)) * a.W + new_row) * D;
            dk = static_cast<T*>(c.k_ring) + off;
            dv = static_cast<T*>(c.v_ring) + off;
            if (slot == a.R && lane == 0) c.ring_pos[(size_t)b * a.W + new_row] = L0;
        } else if (!PAGED) {
            const size_t off = (((size_t)b * a.R + slot) * a.capacity + new_row) * D;
            dk = static_cast<T*>(c.k_full) + off;
            dv = static_cast<T*>(c.v_full) + off;
        } else {
            const int pg = c.page_table[(size_t)b * a.max_pages + new_row / kTile];
            if (pg >= 0 && pg < a.n_pages) {
                const size_t off = (((size_t)pg * a.R + slot) * kTile + new_row % kTile) * D;
                dk = static_cast<T*>(c.k_full) + off;
                dv = static_cast<T*>(c.v_full) + off;
            } else if (lane == 0) {
                atomicOr(c.status, DUO_DEV_BAD_PAGE);
            }
        }
        if (dk) {
            constexpr int kPieces = C::kRowBytes / 16;
            for (int i = lane; i < 2 * kPieces; i += 32) {
                if (i < kPieces)
                    reinterpret_cast<uint4*>(dk)[i] = reinterpret_cast<const uint4*>(kn)[i];
                else
                    reinterpret_cast<uint4*>(dv)[i - kPieces] = reinterpret_cast<const uint4*>(vn)[i - kPieces];
            }
        }
    }

    if (warp == NW) {
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
                    ok = bounds_ok(r0 >= 0 && r0 + n <= (retrieval ? a.capacity : a.W), c.status);
                }
                s_tile_n[st] = ok ? n : 0;
                T* dK = sK + (size_t)st * kTile * D;
                T* dV = sV + (size_t)st * kTile * D;
                if (ok && new_row >= r0 && new_row < r0 + n) {
                    // splice: cached rows before, the new row from k_new / v_new, cached rows after
                    const int nb = new_row - r0, na = n - nb - 1;
                    mbar_arrive_expect_tx(&full_bar[st], 2 * bytes);
                    if (nb > 0) {
                        bulk_g2s(dK, ks, (uint32_t)nb * C::kRowBytes, &full_bar[st]);
                        bulk_g2s(dV, vs, (uint32_t)nb * C::kRowBytes, &full_bar[st]);
                    }
                    bulk_g2s(dK + (size_t)nb * D, kn, C::kRowBytes, &full_bar[st]);
                    bulk_g2s(dV + (size_t)nb * D, vn, C::kRowBytes, &full_bar[st]);
                    if (na > 0) {
                        bulk_g2s(dK + (size_t)(nb + 1) * D, ks + (size_t)(nb + 1) * D, (uint32_t)na * C::kRowBytes,
                                 &full_bar[st]);
                        bulk_g2s(dV + (size_t)(nb + 1) * D, vs + (size_t)(nb + 1) * D, (uint32_t)na * C::kRowBytes,
                                 &full_bar[st]);
                    }
                } else if (ok) {
                    mbar_arrive_expect_tx(&full_bar[st], 2 * bytes);
                    bulk_g2s(dK, ks, bytes, &full_bar[st]);
                    bulk_g2s(dV, vs, bytes, &full_bar[st]);
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
    if (warp < NW) {
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
        float* myP = sP + warp * KW * G;
        const int kidx = (lane & 15) / DUP;  // key this lane scores after the butterfly

        for (int t = 0; t < n_tiles; ++t) {
            const int st = t % STAGES, round = t / STAGES;
            if (!mbar_wait(&full_bar[st], round & 1, c.status)) break;
            const int n = s_tile_n[st];
            const T* tK = sK + (size_t)st * kTile * D;
            const T* tV = sV + (size_t)st * kTile * D;
            const int key0 = warp * KW + hw * KH;   // first key of this half-warp in the tile

            // scores: s[g] of key key0 + kidx
            float s[G];
#pragma unroll
            for (int g = 0; g < G; ++g) s[g] = 0.f;
            {
                float part[G][KH];
#pragma unroll
                for (int j = 0; j < KH; ++j) {
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
                for (int g = 0; g < G; ++g) s[g] = reduce_transposed<KH>(part[g], lane);
            }
            const bool valid = key0 + kidx < n;
            float m_new[G], corr[G], p[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float sv = valid ? s[g] : kNegBig;
                float mt = sv;
                if (DUP == 2) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                m_new[g] = fmaxf(m_run[g], mt);
                corr[g] = exp2f(m_run[g] - m_new[g]);
                p[g] = valid ? exp2f(sv - m_new[g]) : 0.f;
                m_run[g] = m_new[g];
                l_run[g] = l_run[g] * corr[g] + ((lane & (DUP - 1)) ? 0.f : p[g]);
#pragma unroll
                for (int e = 0; e < EPL; ++e) o[g][e] *= corr[g];
            }
            if ((lane & (DUP - 1)) == 0) {
#pragma unroll
                for (int g = 0; g < G; ++g) myP[(hw * KH + kidx) * G + g] = p[g];
            }
            __syncwarp();
            // o += p v over this half-warp's keys
            const int nh = min(KH, n - key0);
#pragma unroll
            for (int j = 0; j < KH; ++j) {
                if (j < nh) {
                    float vf[EPL];
                    load_row_f32<T, EPL>(tV + (size_t)(key0 + j) * D + dl * EPL, vf);
                    const float* pj = myP + (hw * KH + j) * G;
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

    // ---------------------------------------------- merge the warp states
    // layout in the (now free) K stages: [warp][G][STRIDE] with m, l, -, -, o[D]
    float* sM = reinterpret_cast<float*>(sK);
    constexpr int STRIDE = D + 4;
    if (warp < NW) {
        float* dst = sM + (size_t)warp * G * STRIDE;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (lane < 16) {
#pragma unroll
                for (int e = 0; e < EPL; ++e) dst[g * STRIDE + 4 + dl * EPL + e] = o[g][e];
            }
            if (lane == 0) {
                dst[g * STRIDE + 0] = m_run[g];
                dst[g * STRIDE + 1] = l_run[g];
            }
        }
    }
    __syncthreads();
    decode_finish<T, D, G, NW, kThreads, 2 * (size_t)STAGES * C::kTileBytes>(sM, comb_bar, s_flag, a, c, d, b, slot,
                                                                         split, retrieval, fused);
}

// ===========================================================================
// Tensor-core decode consumer (bf16, head_dim 128).
//
// The same work units, pipeline and epilogue as decode_kernel, but the K/V
// tiles arrive through TMA tensor copies with the 128-byte swizzle (two
// 64-column boxes per tile), so warps read them conflict-free with ldmatrix,
// and the contraction runs on mma.sync m16n8k16 (bf16 in, fp32 accumulate):
// the G query heads of the group are the rows of the A operand, padded to 16.
// Four consumer warps each take 16 keys of a 64-key tile:
//   S (16 x 16) = Q K^T  -- 8 k-steps x 2 key blocks, K fragments by ldmatrix
//   softmax on the lane's 4 scores (2 shuffles per row for the maximum)
//   O (16 x 128) += P V  -- P reused in registers as the A fragment, V
//                           fragments by ldmatrix.trans
// For a group of 4 heads this is about a tenth of the instructions of the
// CUDA-core loop, which makes the kernel bound by HBM instead of by issue.
// With a fused append the new token's row is stored into its cache first and
// the tile that holds it is then loaded from there (after a proxy fence).
// ===========================================================================

constexpr int kMmaWarps = 4;
constexpr int kMmaThreads = (kMmaWarps + 1) * 32;
constexpr int kMmaStages = 3;
constexpr uint32_t kMmaTileBytes = kTile * 128 * 2;   // one K or V tile: two 8 KB swizzled halves

constexpr size_t decode_mma_smem_bytes() {
    return 2 * (size_t)kMmaStages * kMmaTileBytes + (2 * kMmaStages + 1) * sizeof(uint64_t) + 64;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

// D = A (16 x 16, rows 8..15 zero) * B (16 x 8) + C, in place in all four
// accumulator registers: rows 8..15 of C stay zero (their rows of A are
// zero), so c[2], c[3] are carried, never re-materialised before an MMA.
__device__ __forceinline__ void mma_rows8(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// byte offset of (row, 16-byte chunk c16 of the 256-byte row) in a tile made
// of two [64 rows][128 B] boxes written by TMA with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw_off(int row, int c16) {
    return (uint32_t)((c16 >> 3) * (kMmaTileBytes / 2) + row * 128 + (((c16 & 7) ^ (row & 7)) << 4));
}

// Tiles each split of decode_mma_kernel takes by its index before it draws
// further tiles from its head's counter: split s takes tiles s, s + nsplit,
// ..., then nsplit * kStaticTiles + (counter draws).
constexpr int kStaticTiles = 2;
constexpr int kWarmTiles = 3;  // tiles per split asked of L2 (or loaded) before the dependency wait
// Rows below (a relaxed read of seq_len) - kSpecMargin are loaded before the
// dependency wait: two earlier decode launches of the same layer may still be
// writing their new rows just below that length.
constexpr int kSpecMargin = 2 * kTile;

// The k-th tile split `split` takes when the tiles are not drawn from a
// counter (one split: all of them in order; otherwise the static ones).
__device__ __forceinline__ int static_tile(int split, int nsplit, int k) { return split + k * nsplit; }

// Runs before griddepcontrol.wait, while the previous grid on the stream may
// still be streaming its own caches: asks L2 for the first kWarmTiles K and V
// tiles of this CTA's split, so the first TMA loads after the wait hit L2.
// The rows come from a relaxed read of seq_len and (paged) of the page table
// and are clamped to the cache, so a stale value only wastes a prefetch.
template <bool PAGED>
__device__ __forceinline__ void warm_l2_split(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d, int b,
                                              int slot, int split, int n_spec) {
    constexpr int kRowBytes = 128 * 2;
    int len = ld_relaxed_gpu(&c.seq_len[b]) + (d.k_new != nullptr ? 1 : 0);
    len = max(0, min(len, a.capacity));
    const uint8_t* kf = static_cast<const uint8_t*>(c.k_full);
    const uint8_t* vf = static_cast<const uint8_t*>(c.v_full);
    for (int k = n_spec; k < kWarmTiles; ++k) {
        // the static tiles not already loading, then (drawn splits) the
        // first tile of the counter's range that this split's index points at
        const int r0 = (k < kStaticTiles ? static_tile(split, d.nsplit, k) : kStaticTiles * d.nsplit + split) * kTile;
        if (r0 >= len) break;
        const uint32_t bytes = (uint32_t)min(kTile, len - r0) * kRowBytes;
        size_t off;
        if (PAGED) {
            const int pg = ld_relaxed_gpu(&c.page_table[(size_t)b * a.max_pages + r0 / kTile]);
            if (pg < 0 || pg >= a.n_pages) continue;
            off = ((size_t)pg * a.R + slot) * kTile * kRowBytes;
        } else {
            off = (((size_t)b * a.R + slot) * a.capacity + r0) * kRowBytes;
        }
        bulk_prefetch_l2(kf + off, bytes);
        bulk_prefetch_l2(vf + off, bytes);
    }
}

template <int G, bool PAGED>
__global__ void __maxnreg__(200)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tmKf, const __grid_constant__ CUtensorMap tmVf,
                      const __grid_constant__ CUtensorMap tmKr, const __grid_constant__ CUtensorMap tmVr,
                      const LayerArgs a, const CacheArgs c, const DecodeArgs d) {
    using T = __nv_bfloat16;
    constexpr int D = 128;
    constexpr int STAGES = kMmaStages;
    constexpr int NW = kMmaWarps;
    constexpr int kThreads = kMmaThreads;
    static_assert(G <= 8, "the group must fit the 8 live rows of an m16 tile");

    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sKb = smem;
    uint8_t* sVb = smem + (size_t)STAGES * kMmaTileBytes;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + 2 * (size_t)STAGES * kMmaTileBytes);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* comb_bar = empty_bar + STAGES;
    int* s_flag = reinterpret_cast<int*>(comb_bar + 1);
    int* s_tile_n = s_flag + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
        if (threadIdx.x == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
        return;
    }

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
    const bool fused = d.k_new != nullptr;
    // Work that reads nothing the previous grid writes: barriers, the tensor
    // maps (kernel parameters), and -- contiguous full cache -- the split's
    // static tiles that lie at least kSpecMargin rows below the length a
    // relaxed read of seq_len gives.  The only grid that can still run
    // before this one's dependency wait is an earlier decode launch (no
    // other kernel of the library triggers its dependents early); it writes
    // one new row per sequence, at or past the length it read, and the
    // lengths only grow, so those rows are final already.  The producer
    // loads them into the first stages now; past the wait it continues from
    // there.
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NW);
        }
        mbar_init(comb_bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    int n_spec = 0;   // producer lane: static tiles already loading
    if (warp == NW && lane == 0) {
        prefetch_map(retrieval ? &tmKf : &tmKr);
        prefetch_map(retrieval ? &tmVf : &tmVr);
        if (retrieval && !PAGED) {
            const int safe = min(ld_relaxed_gpu(&c.seq_len[b]), a.capacity) - kSpecMargin;
            const int z = b * a.R + slot;
            for (int k = 0; k < kStaticTiles; ++k) {
                const int t = static_tile(split, d.nsplit, k);
                if ((t + 1) * kTile > safe) break;
                s_tile_n[k] = kTile;
                mbar_arrive_expect_tx(&full_bar[k], 2 * kMmaTileBytes);
                const uint32_t dk = smem_u32(sKb + (size_t)k * kMmaTileBytes);
                const uint32_t dv = smem_u32(sVb + (size_t)k * kMmaTileBytes);
                for (int h = 0; h < 2; ++h) {
                    tma_load_3d(dk + h * (kMmaTileBytes / 2), &tmKf, 64 * h, t * kTile, z, &full_bar[k]);
                    tma_load_3d(dv + h * (kMmaTileBytes / 2), &tmVf, 64 * h, t * kTile, z, &full_bar[k]);
                }
                ++n_spec;
            }
        }
        if (retrieval) warm_l2_split<PAGED>(a, c, d, b, slot, split, n_spec);
    }
    // launched with programmatic stream serialization: let the next launch's
    // CTAs take SM slots as ours free, and wait for the previous grid before
    // the first read of anything it may have written
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) *s_flag = c.seq_len[b];
    __syncthreads();
    const int L0 = *s_flag;
    if (fused && d.grid_ticket && threadIdx.x == 0) length_ticket(a, c, d);
    int len = L0;
    int new_row = -1;
    if (fused) {
        if (L0 < 0) {
            if (threadIdx.x == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
            len = 0;
        } else if (retrieval && L0 >= a.capacity) {
            if (threadIdx.x == 0 && split == 0) atomicOr(c.status, DUO_DEV_FULL_CACHE_OVERFLOW);
        } else {
            new_row = retrieval ? L0 : ring_slot(L0, a.sink, a.recent);
            len = L0 + 1;
        }
    }
    // Retrieval: the cache rows [0, len) of the (sequence, head) in 64-row
    // tiles, shared out to the head's splits -- each takes kStaticTiles by
    // its index, then draws the rest from the head's counter, so that splits
    // on SMs that stream faster take more tiles and all end together.
    // Streaming: the min(len, W) ring rows.
    int rows;
    if (retrieval) {
        if (len > a.capacity || len < 0) {
            if (threadIdx.x == 0 && split == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
            len = len < 0 ? 0 : a.capacity;
        }
        rows = len;
    } else {
        rows = len < 0 ? 0 : min(len, a.W);
    }
    const int total_tiles = (rows + kTile - 1) / kTile;
    const size_t pair = (size_t)b * a.R + slot;

    if (warp == NW) {
        // ------------------------------------------------------ producer
        // the new token goes into its cache (whole warp) before the tile
        // that holds it is read back through TMA
        auto store_new_row = [&]() {
            if (!bounds_ok(new_row < (retrieval ? a.capacity : a.W), c.status)) return;
            const T* kn = static_cast<const T*>(d.k_new) + ((size_t)b * a.Hkv + a.kv_head[slot]) * D;
            const T* vn = static_cast<const T*>(d.v_new) + ((size_t)b * a.Hkv + a.kv_head[slot]) * D;
            T* dk = nullptr;
            T* dv = nullptr;
            if (!retrieval) {
                const size_t off = (((size_t)b * a.S + (slot - a.R)) * a.W + new_row) * D;
                dk = static_cast<T*>(c.k_ring) + off;
                dv = static_cast<T*>(c.v_ring) + off;
                if (slot == a.R && lane == 0) c.ring_pos[(size_t)b * a.W + new_row] = L0;
            } else if (!PAGED) {
                const size_t off = (((size_t)b * a.R + slot) * a.capacity + new_row) * D;
                dk = static_cast<T*>(c.k_full) + off;
                dv = static_cast<T*>(c.v_full) + off;
            } else {
                const int pg = c.page_table[(size_t)b * a.max_pages + new_row / kTile];
                if (pg >= 0 && pg < a.n_pages) {
                    const size_t off = (((size_t)pg * a.R + slot) * kTile + new_row % kTile) * D;
                    dk = static_cast<T*>(c.k_full) + off;
                    dv = static_cast<T*>(c.v_full) + off;
                } else if (lane == 0) {
                    atomicOr(c.status, DUO_DEV_BAD_PAGE);
                }
            }
            if (dk) {
                if (lane < 16)
                    reinterpret_cast<uint4*>(dk)[lane] = reinterpret_cast<const uint4*>(kn)[lane];
                else
                    reinterpret_cast<uint4*>(dv)[lane - 16] = reinterpret_cast<const uint4*>(vn)[lane - 16];
                asm volatile("fence.proxy.async.global;" ::: "memory");
            }
            __syncwarp();
        };
        if (!retrieval && new_row >= 0) store_new_row();   // the ring's one tile holds every slot
        const CUtensorMap* mk = retrieval ? &tmKf : &tmKr;
        const CUtensorMap* mv = retrieval ? &tmVf : &tmVr;
        const int z = retrieval ? b * a.R + slot : b * a.S + (slot - a.R);
        const bool draw = retrieval && d.draw && d.nsplit > 1;
        const int i0 = __shfl_sync(0xffffffffu, n_spec, 0);   // tiles loaded before the wait
        uint32_t drawn = 0;   // lane 0: the counter draw for the next tile, made while this one loads
        if (lane == 0 && draw && i0 >= kStaticTiles) drawn = atomicAdd(&d.tile_ctr[pair], 1u);
        for (int i = i0;; ++i) {
            const int st = i % STAGES, round = i / STAGES;
            int ok = 1;
            if (lane == 0 && round > 0) ok = mbar_wait(&empty_bar[st], (round - 1) & 1, c.status) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const int t = (draw && i >= kStaticTiles)
                              ? kStaticTiles * d.nsplit + (int)__shfl_sync(0xffffffffu, drawn, 0)
                              : (retrieval ? static_tile(split, d.nsplit, i) : i);
            if (t >= total_tiles) {
                if (lane == 0) {             // no more tiles: tell the consumers
                    s_tile_n[st] = -1;
                    mbar_arrive(&full_bar[st]);
                }
                break;
            }
            const int r0 = t * kTile;
            const int n = min(kTile, rows - r0);
            if (retrieval && new_row >= r0 && new_row < r0 + n) store_new_row();
            if (lane == 0) {
                int pg = 0;
                bool page_ok = true;
                if (PAGED && retrieval) {
                    pg = c.page_table[(size_t)b * a.max_pages + t];
                    if (pg < 0 || pg >= a.n_pages) {
                        atomicOr(c.status, DUO_DEV_BAD_PAGE);
                        page_ok = false;
                    }
                }
                s_tile_n[st] = page_ok ? n : 0;
                if (!page_ok) {
                    mbar_arrive(&full_bar[st]);  // an empty tile: every key of it is masked
                } else {
                    mbar_arrive_expect_tx(&full_bar[st], 2 * kMmaTileBytes);
                    const uint32_t dk = smem_u32(sKb + (size_t)st * kMmaTileBytes);
                    const uint32_t dv = smem_u32(sVb + (size_t)st * kMmaTileBytes);
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t off = h * (kMmaTileBytes / 2);
                        if (PAGED && retrieval) {
                            tma_load_4d(dk + off, mk, 64 * h, 0, slot, pg, &full_bar[st]);
                            tma_load_4d(dv + off, mv, 64 * h, 0, slot, pg, &full_bar[st]);
                        } else {
                            tma_load_3d(dk + off, mk, 64 * h, r0, z, &full_bar[st]);
                            tma_load_3d(dv + off, mv, 64 * h, r0, z, &full_bar[st]);
                        }
                    }
                }
                if (draw && i + 1 >= kStaticTiles) drawn = atomicAdd(&d.tile_ctr[pair], 1u);
            }
        }
    }

    // ------------------------------------------------------ consumers
    const int row = lane >> 2;   // query head of the group for this lane (rows >= G are padding)
    const int quad = lane & 3;
    float o[16][4];   // rows 8-15 of each accumulator stay zero
    float m_run = kNegBig, l_run = 0.f;
    if (warp < NW) {
        uint32_t qa[8][2];
        {
            const bool row_ok = row < G;
            const T* qp = static_cast<const T*>(d.q) + ((size_t)b * a.Hq + a.q_head0[slot] + (row_ok ? row : 0)) * D;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int d0 = 16 * ks + 2 * quad;
                qa[ks][0] = row_ok ? *reinterpret_cast<const uint32_t*>(qp + d0) : 0u;
                qa[ks][1] = row_ok ? *reinterpret_cast<const uint32_t*>(qp + d0 + 8) : 0u;
            }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        const float sl = a.scale * kLog2e;
        const int key_base = warp * 16;
        for (int t = 0;; ++t) {
            const int st = t % STAGES, round = t / STAGES;
            if (!mbar_wait(&full_bar[st], round & 1, c.status)) break;
            const int n = s_tile_n[st];
            if (n < 0) break;                // the producer has no more tiles
            const uint32_t tK = smem_u32(sKb + (size_t)st * kMmaTileBytes);
            uint8_t* tVp = sVb + (size_t)st * kMmaTileBytes;
            const uint32_t tV = smem_u32(tVp);
            const bool partial = n < key_base + 16;
            if (partial) {
                // V rows past the valid keys may hold anything: zero this warp's
                // rows so that P = 0 meets finite V in the MMA
                for (int i = lane; i < 16 * 16; i += 32) {
                    const int key = key_base + (i >> 4), piece = i & 15;
                    if (key >= n)
                        *reinterpret_cast<uint4*>(tVp + (piece >> 3) * (kMmaTileBytes / 2) + key * 128 +
                                                  (piece & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
                }
                __syncwarp();
            }
            // S = Q K^T for keys key_base .. key_base + 15
            float s0[4] = {}, s1[4] = {};
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int key = key_base + (lane & 7) + ((lane >> 4) & 1) * 8;
                const int c16 = 2 * ks + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(tK + sw_off(key, c16), b0, b1, b2, b3);
                mma_rows8(s0, qa[ks][0], qa[ks][1], b0, b1);
                mma_rows8(s1, qa[ks][0], qa[ks][1], b2, b3);
            }
            // this lane's keys: key_base + 2 quad + {0, 1} and + 8
            const int k0 = key_base + 2 * quad;
            float sv[4] = {s0[0] * sl, s0[1] * sl, s1[0] * sl, s1[1] * sl};
            const bool vk[4] = {k0 < n, k0 + 1 < n, k0 + 8 < n, k0 + 9 < n};
            float mx = kNegBig;
#pragma unroll
            for (int i = 0; i < 4; ++i) mx = vk[i] ? fmaxf(mx, sv[i]) : mx;
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run, mx);
            // O and l are rescaled only when some row's maximum grew (a warp
            // vote), which over a long cache is rare
            if (__any_sync(0xffffffffu, m_new > m_run)) {
                const float corr = exp2f(m_run - m_new);
                l_run *= corr;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    o[j][0] *= corr;
                    o[j][1] *= corr;
                }
                m_run = m_new;
            }
            // P rounded to bf16 for the PV MMA; the row sum uses the rounded values
            __nv_bfloat162 p01 = __floats2bfloat162_rn(vk[0] ? exp2f(sv[0] - m_run) : 0.f,
                                                       vk[1] ? exp2f(sv[1] - m_run) : 0.f);
            __nv_bfloat162 p23 = __floats2bfloat162_rn(vk[2] ? exp2f(sv[2] - m_run) : 0.f,
                                                       vk[3] ? exp2f(sv[3] - m_run) : 0.f);
            const uint32_t pa0 = *reinterpret_cast<uint32_t*>(&p01);
            const uint32_t pa1 = *reinterpret_cast<uint32_t*>(&p23);
            l_run += (bf16_lo(pa0) + bf16_hi(pa0)) + (bf16_lo(pa1) + bf16_hi(pa1));
            // O += P V over the 16 keys, 8 pairs of 8-column blocks of d
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int key = key_base + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int c16 = 2 * jj + (lane >> 4);
                uint32_t r0, r1, r2, r3;
                ldsm_x4_t(tV + sw_off(key, c16), r0, r1, r2, r3);
                mma_rows8(o[2 * jj], pa0, pa1, r0, r1);
                mma_rows8(o[2 * jj + 1], pa0, pa1, r2, r3);
            }
            __syncwarp();
            if (partial) fence_proxy_async_smem();  // the zero stores before the next TMA write
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    }
    __syncthreads();  // all tiles consumed: the stage buffers are free

    // warp states -> sM[warp][g][STRIDE]: m, l, -, -, o[D]
    constexpr int STRIDE = D + 4;
    float* sM = reinterpret_cast<float*>(sKb);
    if (warp < NW && row < G) {
        float* dst = sM + ((size_t)warp * G + row) * STRIDE;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            dst[4 + 8 * j + 2 * quad] = o[j][0];
            dst[4 + 8 * j + 2 * quad + 1] = o[j][1];
        }
        if (quad == 0) {
            dst[0] = m_run;
            dst[1] = l_run;
        }
    }
    __syncthreads();
    decode_finish<T, D, G, NW, kThreads, 2 * (size_t)STAGES * kMmaTileBytes>(sM, comb_bar, s_flag, a, c, d, b, slot,
                                                                         split, retrieval, fused);
}

template <int G, bool PAGED>
cudaError_t launch_mma_t(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d, int grid, cudaStream_t s) {
    const uint64_t row = 128 * 2;
    const uint32_t box3[3] = {64, (uint32_t)kTile, 1};
    CUtensorMap mKf{}, mVf{}, mKr{}, mVr{};
    bool have_f = false, have_r = false;
    if (a.R > 0 && d.n_ret_units > 0) {
        if (PAGED) {
            const uint64_t dims[4] = {128, (uint64_t)kTile, (uint64_t)a.R, (uint64_t)a.n_pages};
            const uint64_t st[3] = {row, row * kTile, row * kTile * a.R};
            const uint32_t box[4] = {64, (uint32_t)kTile, 1, 1};
            if (!encode_tmap_bf16(&mKf, c.k_full, 4, dims, st, box) || !encode_tmap_bf16(&mVf, c.v_full, 4, dims, st, box))
                return cudaErrorInvalidValue;
        } else {
            const uint64_t dims[3] = {128, (uint64_t)a.capacity, (uint64_t)a.B * a.R};
            const uint64_t st[2] = {row, row * a.capacity};
            if (!encode_tmap_bf16(&mKf, c.k_full, 3, dims, st, box3) || !encode_tmap_bf16(&mVf, c.v_full, 3, dims, st, box3))
                return cudaErrorInvalidValue;
        }
        have_f = true;
    }
    if (a.S > 0) {
        const uint64_t dims[3] = {128, (uint64_t)a.W, (uint64_t)a.B * a.S};
        const uint64_t st[2] = {row, row * a.W};
        if (!encode_tmap_bf16(&mKr, c.k_ring, 3, dims, st, box3) || !encode_tmap_bf16(&mVr, c.v_ring, 3, dims, st, box3))
            return cudaErrorInvalidValue;
        have_r = true;
    }
    if (!have_f) { mKf = mKr; mVf = mVr; }  // never read: there are no retrieval heads
    if (!have_r) { mKr = mKf; mVr = mVf; }  // never read: there are no streaming heads
    constexpr size_t smem = decode_mma_smem_bytes();
    auto kern = decode_mma_kernel<G, PAGED>;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t e = smem_limit_once(kern, (int)smem, configured);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, kMmaThreads, smem, s, mKf, mVf, mKr, mVr, a, c, d);
}

template <int G>
cudaError_t launch_mma_g(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d, int grid, cudaStream_t s) {
    if (a.page_size) return launch_mma_t<G, true>(a, c, d, grid, s);
    return launch_mma_t<G, false>(a, c, d, grid, s);
}

// Launch with programmatic stream serialization (PDL): the kernel may start
// while the previous grid on the stream finishes; its griddepcontrol.wait
// orders every dependent read after that grid.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int threads, size_t smem, cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <typename T, int D, int G, bool PAGED>
cudaError_t launch_t(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d, int grid, cudaStream_t s) {
    constexpr size_t smem = decode_smem_bytes<T, D, G>();
    auto kern = decode_kernel<T, D, G, PAGED>;
    constexpr int kThreads = (consumer_warps(G) + 1) * 32;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t e = smem_limit_once(kern, (int)smem, configured);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, kThreads, smem, s, a, c, d);
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

// ===========================================================================
// 8-bit full cache: decode_q8_kernel.  Streaming CTAs (after the retrieval
// ones in the grid) read the bf16 ring on the CUDA cores (decode_ring_simt).
// Per retrieval CTA as decode_mma_kernel -- a TMA producer warp, four
// consumer warps of 16 keys each, the same split plan and split-K combine --
// with a 64-token stage of 8 KB of K codes (a row per token, 128-byte
// swizzle), 8 KB of V codes (transposed, 64-byte swizzle) and the tile's 64 +
// 64 scales, five stages deep.
//
// The contractions run on mma.sync m16n8k16 in fp16 with fp32 accumulation:
//   S = q . codes: the codes widen to fp16 exactly (kvq8.cuh); the feature
//     order inside each 16-wide step is permuted the same way for q and K so
//     that a lane's four features (32 t + 4 kb + 0..3) come from one word of
//     its key's row; the key's scale multiplies S in fp32;
//   O += P V: p times the key's V scale, rounded to fp16, is the A operand;
//     the V layout puts a lane's four keys (2t, 2t+1, 2t+8, 2t+9) in one
//     word of each feature row.
// q, p * scale and the codes must fit fp16 (|K|, |V| below 8.3e6, |q| below
// 65504).
// ===========================================================================

constexpr int kQ8Stages = 5;
constexpr uint32_t kQ8Bytes = kTile * 128;          // 8 KB of K or V codes per stage
constexpr uint32_t kQ8ScBytes = 2 * kTile * 4;      // K and V scales of a stage

constexpr size_t decode_q8_smem_bytes() {
    return 2 * (size_t)kQ8Stages * kQ8Bytes + kQ8Stages * kQ8ScBytes + (2 * kQ8Stages + 1) * sizeof(uint64_t) + 64;
}

constexpr uint32_t kF16x2One = 0x3C003C00u;   // (1.0, 1.0) in fp16
constexpr float kTwo24 = 16777216.f;          // 2^24: undoes the subnormal codes' 2^-24

// O (16 x 8, fp32) += A (16 x 16, fp16) B (16 x 8, fp16) with the group's
// query heads in rows 0-7 of A and rows 8-15 zero, accumulating in place into
// all four accumulator registers: rows 8-15 of C stay zero (their rows of A
// are zero), so the pair c[2], c[3] is carried, never re-materialised.
__device__ __forceinline__ void mma_f16_rows8_acc(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// An 8-bit layer's streaming head in the same launch: the ring's min(len, W)
// bf16 rows (every one visible to the new token) on the CUDA cores.  The rows
// are staged in shared memory (rows padded to 272 bytes, so that lanes
// reading different rows hit different banks), then three passes: the
// G x n scores, one per thread at a time; the softmax of each head's row of
// scores, one warp per head; the outputs, one (head, 8 features) per thread.
// With a fused append the new token is first written to its ring slot.
constexpr int kRingRowBytes = 272;
constexpr int kRingMax = 128;        // ring rows this path stages (sink + recent)

template <int G>
__device__ __forceinline__ void decode_ring_simt(uint8_t* smem, const LayerArgs& a, const CacheArgs& c,
                                                 const DecodeArgs& d, int b, int slot, int L0, bool fused) {
    using T = __nv_bfloat16;
    constexpr int D = 128;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int s_idx = slot - a.R;
    T* kr = static_cast<T*>(c.k_ring) + ((size_t)b * a.S + s_idx) * a.W * D;
    T* vr = static_cast<T*>(c.v_ring) + ((size_t)b * a.S + s_idx) * a.W * D;
    int len = L0 < 0 ? 0 : L0;
    if (L0 < 0 && tid == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
    if (fused && L0 >= 0) {
        if (warp == 0) {
            const int rs = ring_slot(L0, a.sink, a.recent);
            const int h = a.kv_head[slot];
            if (bounds_ok(rs >= 0 && rs < a.W, c.status)) {
            const uint2* kn = reinterpret_cast<const uint2*>(static_cast<const T*>(d.k_new) + ((size_t)b * a.Hkv + h) * D);
            const uint2* vn = reinterpret_cast<const uint2*>(static_cast<const T*>(d.v_new) + ((size_t)b * a.Hkv + h) * D);
            reinterpret_cast<uint2*>(kr + (size_t)rs * D)[lane] = kn[lane];
            reinterpret_cast<uint2*>(vr + (size_t)rs * D)[lane] = vn[lane];
            if (s_idx == 0 && lane == 0) c.ring_pos[(size_t)b * a.W + rs] = L0;
            }
        }
        len = L0 + 1;
    }
    __syncthreads();
    const int nk = min(min(len, a.W), kRingMax);
    uint8_t* sK = smem;                                     // [kRingMax][272]
    uint8_t* sV = sK + kRingMax * kRingRowBytes;
    float* sS = reinterpret_cast<float*>(sV + kRingMax * kRingRowBytes);   // [G][kRingMax] scores, then p
    float* sQ = sS + G * kRingMax;                                          // [G][D] q * scale * log2 e
    float* sL = sQ + G * D;                                                 // [G] 1 / row sum
    for (int i = tid; i < nk * 16; i += nthr) {
        const int j = i >> 4, piece = i & 15;
        *reinterpret_cast<uint4*>(sK + j * kRingRowBytes + piece * 16) = reinterpret_cast<const uint4*>(kr + (size_t)j * D)[piece];
        *reinterpret_cast<uint4*>(sV + j * kRingRowBytes + piece * 16) = reinterpret_cast<const uint4*>(vr + (size_t)j * D)[piece];
    }
    const float sl = a.scale * kLog2e;
    for (int i = tid; i < G * D; i += nthr) {
        const int g = i / D, e = i % D;
        sQ[i] = __bfloat162float(static_cast<const T*>(d.q)[((size_t)b * a.Hq + a.q_head0[slot] + g) * D + e]) * sl;
    }
    __syncthreads();
    // scores
    for (int i = tid; i < G * nk; i += nthr) {
        const int g = i / nk, j = i % nk;
        const float* q = sQ + g * D;
        float acc = 0.f;
#pragma unroll 4
        for (int piece = 0; piece < 16; ++piece) {
            float kf[8];
            load_row_f32<T, 8>(reinterpret_cast<const T*>(sK + j * kRingRowBytes + piece * 16), kf);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(q[piece * 8 + e], kf[e], acc);
        }
        sS[g * kRingMax + j] = acc;
    }
    __syncthreads();
    // softmax of each head's scores: p in place, 1 / sum aside
    for (int g = warp; g < G; g += nthr >> 5) {
        float m = kNegBig;
        for (int j = lane; j < nk; j += 32) m = fmaxf(m, sS[g * kRingMax + j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int j = lane; j < nk; j += 32) {
            const float pj = exp2f(sS[g * kRingMax + j] - m);
            sS[g * kRingMax + j] = pj;
            l += pj;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) sL[g] = l > 0.f ? 1.f / l : 0.f;
    }
    __syncthreads();
    // outputs: (head, 8 consecutive features) per thread
    for (int i = tid; i < G * 16; i += nthr) {
        const int g = i >> 4, piece = i & 15;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < nk; ++j) {
            const float pj = sS[g * kRingMax + j];
            float vf[8];
            load_row_f32<T, 8>(reinterpret_cast<const T*>(sV + j * kRingRowBytes + piece * 16), vf);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(pj, vf[e], acc[e]);
        }
        const float inv = sL[g];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= inv;
        store_row<T, 8>(static_cast<T*>(d.out) + ((size_t)b * a.Hq + a.q_head0[slot] + g) * D + piece * 8, acc);
    }
}

constexpr size_t ring_simt_smem_bytes(int G) {
    return 2 * (size_t)kRingMax * kRingRowBytes + (size_t)G * kRingMax * 4 + (size_t)G * 128 * 4 + 8 * 4;
}
static_assert(ring_simt_smem_bytes(8) <= 2 * (size_t)kQ8Stages * kQ8Bytes + kQ8Stages * kQ8ScBytes,
              "the ring path must fit below the 8-bit kernel's barriers");

// The scores of a lane's four keys (k0, k0 + 1, k0 + 8, k0 + 9 of the stage)
// from the MMA sums with the code bias already removed: times the key's K
// scale and the softmax scale (log2 domain), and the keys' V scales.  Only
// a split's last tile can be partial (n < 64, the same for the whole warp):
// there keys at or past n get a score of -inf and a V scale of 0, so that
// neither a stale score nor a stale scale (whatever the cache holds past the
// length) reaches the sums.
__device__ __forceinline__ void quant_scores(float s0, float s1, float s2, float s3, const float* ksc,
                                             const float* vsc, int k0, int n, float sl, float (&sv)[4],
                                             float (&vs)[4]) {
    const float2 ks0 = *reinterpret_cast<const float2*>(ksc + k0);
    const float2 ks1 = *reinterpret_cast<const float2*>(ksc + k0 + 8);
    const float2 vs0 = *reinterpret_cast<const float2*>(vsc + k0);
    const float2 vs1 = *reinterpret_cast<const float2*>(vsc + k0 + 8);
    sv[0] = s0 * ks0.x * sl;
    sv[1] = s1 * ks0.y * sl;
    sv[2] = s2 * ks1.x * sl;
    sv[3] = s3 * ks1.y * sl;
    vs[0] = vs0.x;
    vs[1] = vs0.y;
    vs[2] = vs1.x;
    vs[3] = vs1.y;
    if (n < kTile) {
        const int kk[4] = {k0, k0 + 1, k0 + 8, k0 + 9};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            sv[i] = kk[i] < n ? sv[i] : -INFINITY;
            vs[i] = kk[i] < n ? vs[i] : 0.f;
        }
    }
}

// Runs before griddepcontrol.wait in the 8- and 4-bit kernels: asks L2 for
// the first kWarmTiles tiles of this split's contiguous row range (codes and
// scales), computed from a relaxed read of seq_len, so that the first loads
// after the wait hit L2.  A stale length only moves or wastes a prefetch;
// the rows are clamped to the cache and nothing is written.
__device__ __forceinline__ void warm_l2_quant_split(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d,
                                                    int b, int slot, int split, uint32_t k_row_bytes,
                                                    uint32_t v_tile_bytes) {
    int len = ld_relaxed_gpu(&c.seq_len[b]) + (d.k_new != nullptr ? 1 : 0);
    len = max(0, min(len, a.capacity));
    const int per = (len + d.nsplit - 1) / d.nsplit;
    const int chunk = (per + kTile - 1) / kTile * kTile;
    const int row_begin = min(len, split * chunk);
    const int row_end = min(len, row_begin + chunk);
    const size_t z = (size_t)b * a.R + slot;
    const uint8_t* kf = static_cast<const uint8_t*>(c.k_full);
    const uint8_t* vf = static_cast<const uint8_t*>(c.v_full);
    for (int k = 0; k < kWarmTiles; ++k) {
        const int r0 = row_begin + k * kTile;
        if (r0 >= row_end) break;
        bulk_prefetch_l2(kf + (z * a.capacity + r0) * k_row_bytes, kTile * k_row_bytes);
        bulk_prefetch_l2(vf + (z * (a.capacity / kTile) + r0 / kTile) * v_tile_bytes, v_tile_bytes);
        bulk_prefetch_l2(c.k_scale + z * a.capacity + r0, kTile * 4);
        bulk_prefetch_l2(c.v_scale + z * a.capacity + r0, kTile * 4);
    }
}

// The online softmax over one or more tiles in two parts: rescale_to_max
// takes the row maximum of this lane's scores (mx) over the quad and
// rescales O, l and the PV bias sums only when some row's maximum grew (a
// warp vote); softmax_exp forms p = 2^(s - m) and adds it to the row sum.
template <int NWS, int OW>
__device__ __forceinline__ void rescale_to_max(float mx, float& m_run, float& l_run, float (&o)[16][OW],
                                               float (&wsum)[NWS][OW]) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    if (__any_sync(0xffffffffu, m_new > m_run)) {
        const float corr = exp2f(m_run - m_new);
        l_run *= corr;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            o[j][0] *= corr;
            o[j][1] *= corr;
        }
#pragma unroll
        for (int j = 0; j < NWS; ++j) {
            wsum[j][0] *= corr;
            wsum[j][1] *= corr;
        }
        m_run = m_new;
    }
}

__device__ __forceinline__ void softmax_exp(const float (&sv)[4], float m_run, float& l_run, float (&pr)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) pr[i] = exp2f(sv[i] - m_run);
    l_run += (pr[0] + pr[1]) + (pr[2] + pr[3]);
}

template <int G>
__global__ void __maxnreg__(200)
    decode_q8_kernel(const __grid_constant__ CUtensorMap tmK8, const __grid_constant__ CUtensorMap tmV8,
                     const LayerArgs a, const CacheArgs c, const DecodeArgs d) {
    using T = __nv_bfloat16;
    constexpr int D = 128;
    constexpr int STAGES = kQ8Stages;
    constexpr int NW = kMmaWarps;
    constexpr int kThreads = kMmaThreads;
    static_assert(G <= 8, "the group must fit the 8 live rows of an m16 tile");

    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sK8 = smem;
    uint8_t* sV8 = smem + (size_t)STAGES * kQ8Bytes;
    float* sSc = reinterpret_cast<float*>(smem + 2 * (size_t)STAGES * kQ8Bytes);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + 2 * (size_t)STAGES * kQ8Bytes + STAGES * kQ8ScBytes);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* comb_bar = empty_bar + STAGES;
    int* s_flag = reinterpret_cast<int*>(comb_bar + 1);
    int* s_tile_n = s_flag + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
        if (threadIdx.x == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
        return;
    }

    // ---------------------------------------------------------- work unit
    const bool retrieval = (int)blockIdx.x < d.n_ret_units;
    int split = 0, slot, b;
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
    const int z = b * a.R + slot;
    const int tiles_per_head = a.capacity / kTile;
    const bool fused = d.k_new != nullptr;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NW);
        }
        mbar_init(comb_bar, 1);
        fence_barrier_init();
    }
    if (warp == NW && lane == 0) {
        prefetch_map(&tmK8);
        prefetch_map(&tmV8);
        if (retrieval) warm_l2_quant_split(a, c, d, b, slot, split, 128, kQ8Bytes);
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) *s_flag = c.seq_len[b];
    __syncthreads();
    const int L0 = *s_flag;
    if (fused && d.grid_ticket && threadIdx.x == 0) length_ticket(a, c, d);
    if (!retrieval) {
        decode_ring_simt<G>(smem, a, c, d, b, slot, L0, fused);
        return;
    }
    int len = L0;
    int new_row = -1;
    if (fused) {
        if (L0 < 0) {
            if (threadIdx.x == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
            len = 0;
        } else if (L0 >= a.capacity) {
            if (threadIdx.x == 0 && split == 0) atomicOr(c.status, DUO_DEV_FULL_CACHE_OVERFLOW);
        } else {
            new_row = L0;
            len = L0 + 1;
        }
    }
    if (len > a.capacity || len < 0) {
        if (threadIdx.x == 0 && split == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
        len = len < 0 ? 0 : a.capacity;
    }
    const int per = (len + d.nsplit - 1) / d.nsplit;
    const int chunk = (per + kTile - 1) / kTile * kTile;
    const int row_begin = min(len, split * chunk);
    const int row_end = min(len, row_begin + chunk);
    const int n_tiles = (row_end - row_begin + kTile - 1) / kTile;

    if (warp == NW) {
        // ------------------------------------------------------ producer
        if (new_row >= row_begin && new_row < row_end) {
            // the new token goes into the 8-bit cache first, quantized; the
            // tile that holds it is then read back through TMA
            const int h = a.kv_head[slot];
            const uint2 kw = reinterpret_cast<const uint2*>(static_cast<const T*>(d.k_new) + ((size_t)b * a.Hkv + h) * D)[lane];
            const uint2 vw = reinterpret_cast<const uint2*>(static_cast<const T*>(d.v_new) + ((size_t)b * a.Hkv + h) * D)[lane];
            const float kx[4] = {bf16_lo(kw.x), bf16_hi(kw.x), bf16_lo(kw.y), bf16_hi(kw.y)};
            const float vx[4] = {bf16_lo(vw.x), bf16_hi(vw.x), bf16_lo(vw.y), bf16_hi(vw.y)};
            float ks, vs;
            const uint32_t kc = q8_quantize(kx, ks);
            const uint32_t vc = q8_quantize(vx, vs);
            q8_store_row(a, c, 0, b, slot, new_row, kc, ks, lane);
            q8_store_row(a, c, 1, b, slot, new_row, vc, vs, lane);
            asm volatile("fence.proxy.async.global;" ::: "memory");
            __syncwarp();
        }
        if (lane == 0) {
            for (int t = 0; t < n_tiles; ++t) {
                const int st = t % STAGES, round = t / STAGES;
                if (round > 0 && !mbar_wait(&empty_bar[st], (round - 1) & 1, c.status)) break;
                const int r0 = row_begin + t * kTile;
                if (!bounds_ok((size_t)z < (size_t)a.B * a.R && r0 >= 0 && r0 + kTile <= a.capacity, c.status)) {
                    s_tile_n[st] = 0;                  // an empty tile: every key of it is masked
                    mbar_arrive(&full_bar[st]);
                    continue;
                }
                s_tile_n[st] = min(kTile, row_end - r0);
                mbar_arrive_expect_tx(&full_bar[st], 2 * kQ8Bytes + kQ8ScBytes);
                tma_load_3d(smem_u32(sK8 + (size_t)st * kQ8Bytes), &tmK8, 0, r0, z, &full_bar[st]);
                tma_load_3d(smem_u32(sV8 + (size_t)st * kQ8Bytes), &tmV8, 0, 0, z * tiles_per_head + r0 / kTile,
                            &full_bar[st]);
                bulk_g2s(sSc + st * 2 * kTile, c.k_scale + (size_t)z * a.capacity + r0, kTile * 4, &full_bar[st]);
                bulk_g2s(sSc + st * 2 * kTile + kTile, c.v_scale + (size_t)z * a.capacity + r0, kTile * 4,
                         &full_bar[st]);
            }
        }
    }

    // ------------------------------------------------------ consumers
    const int row = lane >> 2;   // query head of the group (rows >= G are padding) / key of an 8-key block
    const int quad = lane & 3;
    float o[16][4];   // rows 8-15 of each accumulator stay zero
    float m_run = kNegBig, l_run = 0.f;
    float wsum[1][4] = {};   // sum of the PV A operand per row (the code bias)
    if (warp < NW) {
        // q in fp16, features 32 quad + 4 kb + {0, 1} and {2, 3} for step kb.
        // The K operands keep the bias of the byte-to-fp16 step (1152 +
        // code), so a score is the MMA's sum minus 1152 times the row's sum
        // of q -- a fresh accumulator per tile, so no precision is lost.
        uint32_t qa[8][2];
        float q_corr = 0.f;
        {
            const bool row_ok = row < G;
            const uint4* qp = reinterpret_cast<const uint4*>(
                static_cast<const T*>(d.q) + ((size_t)b * a.Hq + a.q_head0[slot] + (row_ok ? row : 0)) * D + 32 * quad);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 w = row_ok ? qp[i] : make_uint4(0u, 0u, 0u, 0u);
                qa[2 * i][0] = f16x2_pack(bf16_lo(w.x), bf16_hi(w.x));
                qa[2 * i][1] = f16x2_pack(bf16_lo(w.y), bf16_hi(w.y));
                qa[2 * i + 1][0] = f16x2_pack(bf16_lo(w.z), bf16_hi(w.z));
                qa[2 * i + 1][1] = f16x2_pack(bf16_lo(w.w), bf16_hi(w.w));
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&qa[2 * i + h][e]));
                        q_corr += f.x + f.y;
                    }
            }
            q_corr += __shfl_xor_sync(0xffffffffu, q_corr, 1);
            q_corr += __shfl_xor_sync(0xffffffffu, q_corr, 2);
            q_corr *= 1152.f;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        const float sl = a.scale * kLog2e;
        const int key_base = warp * 16;
        // one pass over NT (1 or 2) consecutive tiles, as in the 4-bit kernel
        auto pass = [&](int t, auto nt_c) -> bool {
            constexpr int NT = decltype(nt_c)::value;
            int st[NT];
            bool ok = true;
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                st[i] = (t + i) % STAGES;
                ok = ok && mbar_wait(&full_bar[st[i]], ((t + i) / STAGES) & 1, c.status);
            }
            if (!ok) return false;
            // this lane's keys: key_base + 2 quad + {0, 1} and + 8
            const int k0 = key_base + 2 * quad;
            float sv[NT][4], vs[NT][4];
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                // S = q . codes for keys key_base + 8 nb + (lane >> 2)
                const uint8_t* tK = sK8 + (size_t)st[i] * kQ8Bytes;
                float s[2][4] = {};
#pragma unroll
                for (int nb = 0; nb < 2; ++nb) {
                    const int key = key_base + 8 * nb + row;
                    const uint4 lo = *reinterpret_cast<const uint4*>(tK + key * 128 + (((2 * quad) ^ (key & 7)) << 4));
                    const uint4 hi = *reinterpret_cast<const uint4*>(tK + key * 128 + (((2 * quad + 1) ^ (key & 7)) << 4));
                    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                    for (int kb = 0; kb < 8; ++kb) {
                        uint32_t b0, b1;
                        i8x4_to_f16x2_biased(w[kb], b0, b1);
                        mma_f16_rows8_acc(s[nb], qa[kb][0], qa[kb][1], b0, b1);
                    }
                }
                const float* ksc = sSc + st[i] * 2 * kTile;
                quant_scores(s[0][0] - q_corr, s[0][1] - q_corr, s[1][0] - q_corr, s[1][1] - q_corr, ksc,
                             ksc + kTile, k0, s_tile_n[st[i]], sl, sv[i], vs[i]);
            }
            float mx = kNegBig;
#pragma unroll
            for (int i = 0; i < NT; ++i) mx = fmaxf(mx, fmaxf(fmaxf(sv[i][0], sv[i][1]), fmaxf(sv[i][2], sv[i][3])));
            rescale_to_max(mx, m_run, l_run, o, wsum);
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                float pr[4];
                softmax_exp(sv[i], m_run, l_run, pr);
                // p times the key's V scale, the fp16 A operand of O += P V
                const uint32_t pa0 = f16x2_pack(pr[0] * vs[i][0], pr[1] * vs[i][1]);
                const uint32_t pa1 = f16x2_pack(pr[2] * vs[i][2], pr[3] * vs[i][3]);
                // O' += P U with U = (code + 128) 2^-24 (exact fp16 subnormals),
                // and the bias sum W += P 1 through the same MMA: O = 2^24 O' -
                // 128 W at the end.  Feature row 8 nd + (lane >> 2), this warp's
                // 16-key group (64-byte swizzle), the lane's four keys in one word
                mma_f16_rows8_acc(wsum[0], pa0, pa1, kF16x2One, kF16x2One);
                const uint8_t* tV = sV8 + (size_t)st[i] * kQ8Bytes;
#pragma unroll
                for (int nd = 0; nd < 16; ++nd) {
                    const int f = 8 * nd + row;
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(tV + f * 64 + ((warp ^ ((f >> 1) & 3)) << 4) +
                                                                          4 * quad);
                    uint32_t b0, b1;
                    i8x4_to_f16x2_sub(w, b0, b1);
                    mma_f16_rows8_acc(o[nd], pa0, pa1, b0, b1);
                }
            }
            __syncwarp();
            if (lane == 0) {
#pragma unroll
                for (int i = 0; i < NT; ++i) mbar_arrive(&empty_bar[st[i]]);
            }
            return true;
        };
        int t = 0;
        bool ok = true;
        for (; ok && t + 1 < n_tiles; t += 2) ok = pass(t, std::integral_constant<int, 2>{});
        if (ok && t < n_tiles) pass(t, std::integral_constant<int, 1>{});
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    }
    __syncthreads();  // all tiles consumed: the stage buffers are free

    // warp states -> sM[warp][g][STRIDE]: m, l, -, -, o[D]
    constexpr int STRIDE = D + 4;
    float* sM = reinterpret_cast<float*>(smem);
    if (warp < NW && row < G) {
        float* dst = sM + ((size_t)warp * G + row) * STRIDE;
        const float bias = 128.f * wsum[0][0];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            dst[4 + 8 * j + 2 * quad] = fmaf(o[j][0], kTwo24, -bias);
            dst[4 + 8 * j + 2 * quad + 1] = fmaf(o[j][1], kTwo24, -bias);
        }
        if (quad == 0) {
            dst[0] = m_run;
            dst[1] = l_run;
        }
    }
    __syncthreads();
    decode_finish<T, D, G, NW, kThreads, 2 * (size_t)STAGES * kQ8Bytes>(sM, comb_bar, s_flag, a, c, d, b, slot, split,
                                                                      true, fused);
}

template <int G>
cudaError_t launch_q8_g(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d, int grid, cudaStream_t s) {
    CUtensorMap mK{}, mV{};
    {
        const uint64_t dims[3] = {128, (uint64_t)a.capacity, (uint64_t)a.B * a.R};
        const uint64_t st[2] = {128, 128ull * a.capacity};
        const uint32_t box[3] = {128, (uint32_t)kTile, 1};
        if (!encode_tmap(&mK, c.k_full, 3, dims, st, box, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128))
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[3] = {(uint64_t)kTile, 128, (uint64_t)a.B * a.R * (a.capacity / kTile)};
        const uint64_t st[2] = {(uint64_t)kTile, 128ull * kTile};
        const uint32_t box[3] = {(uint32_t)kTile, 128, 1};
        if (!encode_tmap(&mV, c.v_full, 3, dims, st, box, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64))
            return cudaErrorInvalidValue;
    }
    constexpr size_t smem = decode_q8_smem_bytes();
    auto kern = decode_q8_kernel<G>;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t e = smem_limit_once(kern, (int)smem, configured);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, kMmaThreads, smem, s, mK, mV, a, c, d);
}

// ===========================================================================
// 4-bit full cache: decode_q4_kernel.  The 8-bit kernel's work units,
// producer/consumer pipeline, streaming path and split-K combine, over the
// 4-bit layouts of kvq4.cuh: a 64-token stage is 4 KB of K codes and 4 KB of
// V codes, each one contiguous bulk copy (the layouts are already in the
// order the consumers read, so no tensor map or swizzle is needed), plus the
// tile's 64 + 64 scales; eight stages, two CTAs to an SM.
//   S = q . codes: a lane's 16 bytes of a key's row hold its 32 permuted
//     features; each word gives two k-steps' B fragments by masking nibble
//     pairs into fp16 (u4x2_to_f16x2); q is permuted as for the 8-bit cache.
//   O += P V: one word per (feature pair, key quad) gives the B fragments of
//     feature rows 16 m + r and 16 m + 8 + r for the lane's four keys.
// ===========================================================================

constexpr int kQ4Stages = 8;
constexpr uint32_t kQ4ScBytes = 2 * kTile * 4;      // K and V scales of a stage

// The barriers sit above both the stage buffers of a retrieval CTA and the
// ring staging of a streaming CTA (which needs more for a group of 8).
template <int G>
constexpr size_t q4_bar_offset() {
    constexpr size_t stages = 2 * (size_t)kQ4Stages * kQ4TileBytes + kQ4Stages * kQ4ScBytes;
    constexpr size_t ring = (ring_simt_smem_bytes(G) + 15) / 16 * 16;
    return stages > ring ? stages : ring;
}
template <int G>
constexpr size_t decode_q4_smem_bytes() {
    return q4_bar_offset<G>() + (2 * kQ4Stages + 1) * sizeof(uint64_t) + 64;
}
// two CTAs to an SM (227 KB, 1 KB of it reserved per CTA).  Three (at most
// 128 registers, eight stages) were measured: no faster at 1M tokens and
// slower at 128K, the register cap costing spills.
static_assert(2 * (decode_q4_smem_bytes<8>() + 1024) <= 232448, "two 4-bit CTAs per SM");

template <int G>
__global__ void __maxnreg__(200)
    decode_q4_kernel(const LayerArgs a, const CacheArgs c, const DecodeArgs d) {
    using T = __nv_bfloat16;
    constexpr int D = 128;
    constexpr int STAGES = kQ4Stages;
    constexpr int NW = kMmaWarps;
    constexpr int kThreads = kMmaThreads;
    static_assert(G <= 8, "the group must fit the 8 live rows of an m16 tile");

    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sK4 = smem;
    uint8_t* sV4 = smem + (size_t)STAGES * kQ4TileBytes;
    float* sSc = reinterpret_cast<float*>(smem + 2 * (size_t)STAGES * kQ4TileBytes);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + q4_bar_offset<G>());
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* comb_bar = empty_bar + STAGES;
    int* s_flag = reinterpret_cast<int*>(comb_bar + 1);
    int* s_tile_n = s_flag + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---------------------------------------------------------- work unit
    const bool retrieval = (int)blockIdx.x < d.n_ret_units;
    int split = 0, slot, b;
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
    const size_t z = (size_t)b * a.R + slot;
    const bool fused = d.k_new != nullptr;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NW);
        }
        mbar_init(comb_bar, 1);
        fence_barrier_init();
    }
    if (retrieval && warp == NW && lane == 0) warm_l2_quant_split(a, c, d, b, slot, split, kQ4RowBytes, kQ4TileBytes);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) *s_flag = c.seq_len[b];
    __syncthreads();
    const int L0 = *s_flag;
    if (fused && d.grid_ticket && threadIdx.x == 0) length_ticket(a, c, d);
    if (!retrieval) {
        decode_ring_simt<G>(smem, a, c, d, b, slot, L0, fused);
        return;
    }
    int len = L0;
    int new_row = -1;
    if (fused) {
        if (L0 < 0) {
            if (threadIdx.x == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
            len = 0;
        } else if (L0 >= a.capacity) {
            if (threadIdx.x == 0 && split == 0) atomicOr(c.status, DUO_DEV_FULL_CACHE_OVERFLOW);
        } else {
            new_row = L0;
            len = L0 + 1;
        }
    }
    if (len > a.capacity || len < 0) {
        if (threadIdx.x == 0 && split == 0) atomicOr(c.status, DUO_DEV_BAD_LENGTH);
        len = len < 0 ? 0 : a.capacity;
    }
    const int per = (len + d.nsplit - 1) / d.nsplit;
    const int chunk = (per + kTile - 1) / kTile * kTile;
    const int row_begin = min(len, split * chunk);
    const int row_end = min(len, row_begin + chunk);
    const int n_tiles = (row_end - row_begin + kTile - 1) / kTile;

    if (warp == NW) {
        // ------------------------------------------------------ producer
        if (new_row >= row_begin && new_row < row_end) {
            // the new token goes into the 4-bit cache first, quantized; the
            // tile that holds it is then read back with bulk copies
            const int h = a.kv_head[slot];
            const uint2 kw = reinterpret_cast<const uint2*>(static_cast<const T*>(d.k_new) + ((size_t)b * a.Hkv + h) * D)[lane];
            const uint2 vw = reinterpret_cast<const uint2*>(static_cast<const T*>(d.v_new) + ((size_t)b * a.Hkv + h) * D)[lane];
            const float kx[4] = {bf16_lo(kw.x), bf16_hi(kw.x), bf16_lo(kw.y), bf16_hi(kw.y)};
            const float vx[4] = {bf16_lo(vw.x), bf16_hi(vw.x), bf16_lo(vw.y), bf16_hi(vw.y)};
            int kc[4], vc[4];
            float ks, vs;
            q4_quantize(kx, kc, ks);
            q4_quantize(vx, vc, vs);
            q4_store_row(a, c, 0, b, slot, new_row, kc, ks, lane);
            q4_store_row(a, c, 1, b, slot, new_row, vc, vs, lane);
            asm volatile("fence.proxy.async.global;" ::: "memory");
            __syncwarp();
        }
        if (lane == 0) {
            const uint8_t* kf = static_cast<const uint8_t*>(c.k_full);
            const uint8_t* vf = static_cast<const uint8_t*>(c.v_full);
            for (int t = 0; t < n_tiles; ++t) {
                const int st = t % STAGES, round = t / STAGES;
                if (round > 0 && !mbar_wait(&empty_bar[st], (round - 1) & 1, c.status)) break;
                const int r0 = row_begin + t * kTile;
                if (!bounds_ok((size_t)z < (size_t)a.B * a.R && r0 >= 0 && r0 + kTile <= a.capacity, c.status)) {
                    s_tile_n[st] = 0;                  // an empty tile: every key of it is masked
                    mbar_arrive(&full_bar[st]);
                    continue;
                }
                s_tile_n[st] = min(kTile, row_end - r0);
                mbar_arrive_expect_tx(&full_bar[st], 2 * kQ4TileBytes + kQ4ScBytes);
                // whole 64-token tiles: the capacity is a multiple of 64
                bulk_g2s(sK4 + (size_t)st * kQ4TileBytes, kf + (z * a.capacity + r0) * kQ4RowBytes, kQ4TileBytes,
                         &full_bar[st]);
                bulk_g2s(sV4 + (size_t)st * kQ4TileBytes, vf + (z * (a.capacity / kTile) + r0 / kTile) * kQ4TileBytes,
                         kQ4TileBytes, &full_bar[st]);
                bulk_g2s(sSc + st * 2 * kTile, c.k_scale + z * a.capacity + r0, kTile * 4, &full_bar[st]);
                bulk_g2s(sSc + st * 2 * kTile + kTile, c.v_scale + z * a.capacity + r0, kTile * 4, &full_bar[st]);
            }
        }
    }

    // ------------------------------------------------------ consumers
    // Nibbles are not shifted down one by one: a mask-and-or puts a word's
    // nibbles n at bits 0-3 / 16-19 under the fp16 exponent of 1024 (the
    // values 1024 + n) and those at bits 4-7 / 20-23 likewise (1024 + 16 n);
    // the MMA partner of a 16 n operand is pre-divided by 16 (exact in fp16).
    // q . K keeps the bias: every product is 1024 q + q n or 64 q' + q' n
    // (q' = q / 16), and since code = n - 8 the score is the MMA's sum minus
    // a per-row constant, 1032 (1152) times the sum of the partners -- a
    // fresh accumulator per tile, so the cancellation costs no precision.
    // P V accumulates over the whole cache, so its operands are un-biased
    // exactly instead: 1024 + n - 1032 = code, 1024 + 16 n - 1152 = 16 code.
    const int row = lane >> 2;   // query head of the group (rows >= G are padding) / key of an 8-key block
    const int quad = lane & 3;
    float o[16][4];   // rows 8-15 of each accumulator stay zero
    float m_run = kNegBig, l_run = 0.f;
    float wsum[2][4] = {};   // PV A operand sums per row: p vs, p vs / 16
    if (warp < NW) {
        // q in fp16, features 32 quad + 4 kb + {0, 1} (partners of the low
        // nibbles) and {2, 3} (partners of the high nibbles, divided by 16)
        uint32_t qa[8][2];
        float q_corr = 0.f;
        {
            const bool row_ok = row < G;
            const uint4* qp = reinterpret_cast<const uint4*>(
                static_cast<const T*>(d.q) + ((size_t)b * a.Hq + a.q_head0[slot] + (row_ok ? row : 0)) * D + 32 * quad);
            const __half2 sixteenth = __float2half2_rn(0.0625f);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 w = row_ok ? qp[i] : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t lo0 = f16x2_pack(bf16_lo(w.x), bf16_hi(w.x));
                const uint32_t lo1 = f16x2_pack(bf16_lo(w.z), bf16_hi(w.z));
                const uint32_t t0 = f16x2_pack(bf16_lo(w.y), bf16_hi(w.y));
                const uint32_t t1 = f16x2_pack(bf16_lo(w.w), bf16_hi(w.w));
                const __half2 hi0 = __hmul2(*reinterpret_cast<const __half2*>(&t0), sixteenth);
                const __half2 hi1 = __hmul2(*reinterpret_cast<const __half2*>(&t1), sixteenth);
                qa[2 * i][0] = lo0;
                qa[2 * i][1] = *reinterpret_cast<const uint32_t*>(&hi0);
                qa[2 * i + 1][0] = lo1;
                qa[2 * i + 1][1] = *reinterpret_cast<const uint32_t*>(&hi1);
                const float2 l0 = __half22float2(*reinterpret_cast<const __half2*>(&lo0));
                const float2 l1 = __half22float2(*reinterpret_cast<const __half2*>(&lo1));
                const float2 h0 = __half22float2(hi0), h1 = __half22float2(hi1);
                q_corr += 1032.f * ((l0.x + l0.y) + (l1.x + l1.y)) + 1152.f * ((h0.x + h0.y) + (h1.x + h1.y));
            }
            // the row's constant over all 128 features (the quad's four lanes)
            q_corr += __shfl_xor_sync(0xffffffffu, q_corr, 1);
            q_corr += __shfl_xor_sync(0xffffffffu, q_corr, 2);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        const float sl = a.scale * kLog2e;
        const int key_base = warp * 16;
        const __half2 sixteenth = __float2half2_rn(0.0625f);
        // One pass over NT (1 or 2) consecutive tiles: both full-barrier waits
        // first, then one straight-line block -- the tiles' q . K, one joint
        // row maximum (two shuffles and one rescale vote for both), their
        // exponentials and P V -- so that the two tiles' independent chains
        // interleave (a warp has little else to hide latency with: two CTAs
        // of four consumer warps per SM).  Returns false when a wait ran out.
        auto pass = [&](int t, auto nt_c) -> bool {
            constexpr int NT = decltype(nt_c)::value;
            int st[NT];
            bool ok = true;
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                st[i] = (t + i) % STAGES;
                ok = ok && mbar_wait(&full_bar[st[i]], ((t + i) / STAGES) & 1, c.status);
            }
            if (!ok) return false;
            // this lane's keys: key_base + 2 quad + {0, 1} and + 8
            const int k0 = key_base + 2 * quad;
            float sv[NT][4], vs[NT][4];
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                // S' = q . (biased codes) for keys key_base + 8 nb + (lane >> 2),
                // even and odd k-steps in separate accumulators
                const uint8_t* tK = sK4 + (size_t)st[i] * kQ4TileBytes;
                float s[2][2][4] = {};
#pragma unroll
                for (int nb = 0; nb < 2; ++nb) {
                    const int key = key_base + 8 * nb + row;
                    const uint4 kw = *reinterpret_cast<const uint4*>(tK + key * kQ4RowBytes + 16 * quad);
                    const uint32_t w[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t w8 = w[j] >> 8;
                        mma_f16_rows8_acc(s[nb][0], qa[2 * j][0], qa[2 * j][1], u4_lo_f16x2(w[j]), u4_hi_f16x2(w[j]));
                        mma_f16_rows8_acc(s[nb][1], qa[2 * j + 1][0], qa[2 * j + 1][1], u4_lo_f16x2(w8), u4_hi_f16x2(w8));
                    }
                }
                const float* ksc = sSc + st[i] * 2 * kTile;
                quant_scores(s[0][0][0] + s[0][1][0] - q_corr, s[0][0][1] + s[0][1][1] - q_corr,
                             s[1][0][0] + s[1][1][0] - q_corr, s[1][0][1] + s[1][1][1] - q_corr, ksc, ksc + kTile,
                             k0, s_tile_n[st[i]], sl, sv[i], vs[i]);
            }
            float mx = kNegBig;
#pragma unroll
            for (int i = 0; i < NT; ++i) mx = fmaxf(mx, fmaxf(fmaxf(sv[i][0], sv[i][1]), fmaxf(sv[i][2], sv[i][3])));
            rescale_to_max(mx, m_run, l_run, o, wsum);
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                float pr[4];
                softmax_exp(sv[i], m_run, l_run, pr);
                // p times the key's V scale, the fp16 A operand of O += P V, and
                // the same divided by 16 for the high-nibble feature rows
                const uint32_t pa0 = f16x2_pack(pr[0] * vs[i][0], pr[1] * vs[i][1]);
                const uint32_t pa1 = f16x2_pack(pr[2] * vs[i][2], pr[3] * vs[i][3]);
                const __half2 ph0 = __hmul2(*reinterpret_cast<const __half2*>(&pa0), sixteenth);
                const __half2 ph1 = __hmul2(*reinterpret_cast<const __half2*>(&pa1), sixteenth);
                const uint32_t pb0 = *reinterpret_cast<const uint32_t*>(&ph0);
                const uint32_t pb1 = *reinterpret_cast<const uint32_t*>(&ph1);
                // O' += P U: the word of feature pair (16 m + r, 16 m + 8 + r) and
                // this lane's key quad in the warp's 16-token group, its nibbles
                // taken as exact fp16 subnormals n 2^-24 (low) and 16 n 2^-24
                // (high, against p / 16); the bias sums W += P 1 ride on the same
                // MMA, and O = 2^24 O' - 8 W (low) or - 128 W (high) at the end
                mma_f16_rows8_acc(wsum[0], pa0, pa1, kF16x2One, kF16x2One);
                mma_f16_rows8_acc(wsum[1], pb0, pb1, kF16x2One, kF16x2One);
                const uint8_t* tV = sV4 + (size_t)st[i] * kQ4TileBytes;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(tV + 1024 * warp + 128 * m + 16 * row + 4 * quad);
                    const uint32_t w8 = w >> 8;
                    mma_f16_rows8_acc(o[2 * m], pa0, pa1, u4_lo_sub(w), u4_lo_sub(w8));
                    mma_f16_rows8_acc(o[2 * m + 1], pb0, pb1, u4_hi_sub(w), u4_hi_sub(w8));
                }
            }
            __syncwarp();
            if (lane == 0) {
#pragma unroll
                for (int i = 0; i < NT; ++i) mbar_arrive(&empty_bar[st[i]]);
            }
            return true;
        };
        int t = 0;
        bool ok = true;
        for (; ok && t + 1 < n_tiles; t += 2) ok = pass(t, std::integral_constant<int, 2>{});
        if (ok && t < n_tiles) pass(t, std::integral_constant<int, 1>{});
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    }
    __syncthreads();  // all tiles consumed: the stage buffers are free

    // warp states -> sM[warp][g][STRIDE]: m, l, -, -, o[D]
    constexpr int STRIDE = D + 4;
    float* sM = reinterpret_cast<float*>(smem);
    if (warp < NW && row < G) {
        float* dst = sM + ((size_t)warp * G + row) * STRIDE;
        // even n-tiles are low-nibble feature rows (bias 8 p vs), odd ones
        // high-nibble rows (bias 8 * 16 * p vs / 16)
        const float bias_lo = 8.f * wsum[0][0], bias_hi = 128.f * wsum[1][0];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float bias = (j & 1) ? bias_hi : bias_lo;
            dst[4 + 8 * j + 2 * quad] = fmaf(o[j][0], kTwo24, -bias);
            dst[4 + 8 * j + 2 * quad + 1] = fmaf(o[j][1], kTwo24, -bias);
        }
        if (quad == 0) {
            dst[0] = m_run;
            dst[1] = l_run;
        }
    }
    __syncthreads();
    decode_finish<T, D, G, NW, kThreads, 2 * (size_t)STAGES * kQ4TileBytes>(sM, comb_bar, s_flag, a, c, d, b, slot,
                                                                          split, true, fused);
}

template <int G>
cudaError_t launch_q4_g(const LayerArgs& a, const CacheArgs& c, const DecodeArgs& d, int grid, cudaStream_t s) {
    constexpr size_t smem = decode_q4_smem_bytes<G>();
    auto kern = decode_q4_kernel<G>;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t e = smem_limit_once(kern, (int)smem, configured);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, kMmaThreads, smem, s, a, c, d);
}

}  // namespace

cudaError_t launch_decode(const LayerArgs& a, const CacheArgs& c, const DecodePlan& plan, const void* q, void* out,
                          void* workspace, cudaStream_t s, const void* k_new, const void* v_new) {
    DecodeArgs d;
    d.k_new = k_new;
    d.v_new = v_new;
    d.grid_ticket = c.counters + 1;
    d.q = q;
    d.out = out;
    d.partial = static_cast<float*>(workspace);
    d.ticket = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + plan.ticket_offset);
    d.tile_ctr = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + plan.counter_offset);
    d.nsplit = plan.nsplit;
    d.n_ret_units = a.B * a.R * plan.nsplit;
    const long grid = (long)d.n_ret_units + (long)a.B * a.S;
    if (grid == 0) return cudaSuccess;
    // Drawing tiles balances a head's splits when they all run at once (one
    // wave of two CTAs per SM); in a grid of several waves a split that runs
    // early would drain its head's counter while its siblings wait for a
    // slot, so the splits keep their static share there.
    d.draw = grid <= 2L * sm_count() ? 1 : 0;
    if (grid > 0x7fffffffL) return cudaErrorInvalidConfiguration;
    if (a.kv_bits == 4 && a.R > 0) {
        // 4-bit full cache: as the 8-bit path, over nibble codes
        switch (a.G) {
            case 1: return launch_q4_g<1>(a, c, d, (int)grid, s);
            case 2: return launch_q4_g<2>(a, c, d, (int)grid, s);
            case 4: return launch_q4_g<4>(a, c, d, (int)grid, s);
            case 8: return launch_q4_g<8>(a, c, d, (int)grid, s);
        }
        return cudaErrorInvalidValue;
    }
    if (a.kv_bits == 8 && a.R > 0) {
        // 8-bit full cache: retrieval CTAs on the int8 tiles, streaming CTAs
        // over the bf16 ring on the CUDA cores, one launch
        switch (a.G) {
            case 1: return launch_q8_g<1>(a, c, d, (int)grid, s);
            case 2: return launch_q8_g<2>(a, c, d, (int)grid, s);
            case 4: return launch_q8_g<4>(a, c, d, (int)grid, s);
            case 8: return launch_q8_g<8>(a, c, d, (int)grid, s);
        }
        return cudaErrorInvalidValue;
    }
    if (a.dtype == DUO_BF16) {
        if (a.D == 128) {
            // bf16, head_dim 128: the tensor-core consumer
            switch (a.G) {
                case 1: return launch_mma_g<1>(a, c, d, (int)grid, s);
                case 2: return launch_mma_g<2>(a, c, d, (int)grid, s);
                case 4: return launch_mma_g<4>(a, c, d, (int)grid, s);
                case 8: return launch_mma_g<8>(a, c, d, (int)grid, s);
            }
            return cudaErrorInvalidValue;
        }
        return launch_d<__nv_bfloat16, 64>(a, c, d, (int)grid, s);
    }
    if (a.D == 128) return launch_d<float, 128>(a, c, d, (int)grid, s);
    return launch_d<float, 64>(a, c, d, (int)grid, s);
}

}  // namespace duo
