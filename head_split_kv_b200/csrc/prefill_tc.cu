// prefill_tc.cu -- chunked pre-fill attention on the 5th-generation tensor
// cores (tcgen05 MMA, accumulators in TMEM, operands staged by TMA).
//
// [Summary S2 "Chunked Pre-filling": fixed-length prompt chunks; both caches
//  are pre-filled.  Review S3 "Inference flow", pre-fill: retrieval heads use
//  full (FlashAttention-style) causal attention; streaming heads run in linear
//  time and constant memory.]
//
// One CTA owns 128 query rows of one query head (the chunk rows 128m..128m+127)
// and walks 64-key tiles:
//   retrieval head: every prior key from the full cache (tiles aligned to end
//     at the chunk start c0) and the chunk's own keys up to the diagonal;
//   streaming head: the ring (sinks + recent tokens before c0, positions from
//     ring_pos), the chunk's sink tile when c0 < sink, and the chunk tiles of
//     the recent band -- at most 7 tiles whatever the context length.
// Roles (192 threads):
//   warp 4  TMA producer: Q once (2 boxes of 64 columns, 128B swizzle), then
//           K and V tiles into 2-stage rings;
//   warp 5  MMA issuer (one thread): S = Q K^T (M128 N64 K128) into a
//           double-buffered TMEM tile, then O += P V (M128 N128 K64) with P
//           from shared memory and V read MN-major;
//   warps 0-3  softmax: thread t owns query row t (TMEM lane t): loads its S
//           row, masks by absolute position, keeps the running max in the
//           log2 domain with a lazy O rescale (only when the max grows by more
//           than 2^8), writes P as bf16 in the swizzled K-major layout, and at
//           the end divides O by the row sum and stores bf16.
// About 113 KB of shared memory and 256 TMEM columns per CTA, so two CTAs
// share an SM and their MMA and softmax phases interleave.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace duo {
namespace {

constexpr int BM = 128;            // query rows per CTA
constexpr int BN = 64;             // keys per tile
constexpr int HD = 128;            // head dim
constexpr int kThreadsTC = 192;
constexpr int kTmaWarp = 4, kMmaWarp = 5;
constexpr uint32_t kTmemCols = 256;
__device__ __forceinline__ constexpr uint32_t col_s(int st) { return st ? 64u : 0u; }  // S double buffer
constexpr uint32_t kColO = 128;
constexpr int kMaxRing = 128;      // sink + recent supported on this path
constexpr int kMaxChunkTiles = 8;

constexpr uint32_t kQBytes = BM * HD * 2;      // 32 KB (two 16 KB halves of d)
constexpr uint32_t kTileBytes = BN * HD * 2;   // 16 KB (two 8 KB halves)
constexpr uint32_t kPBytes = BM * BN * 2;      // 16 KB
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQBytes;
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;
constexpr uint32_t kOffP = kOffV + 2 * kTileBytes;
constexpr uint32_t kOffBar = kOffP + kPBytes;
constexpr uint32_t kOffHolder = kOffBar + 16 * 8;
constexpr uint32_t kOffPos = kOffHolder + 16;
constexpr uint32_t kSmemBytes = kOffPos + kMaxRing * 4;
static_assert(kSmemBytes + 1024 <= 233472 / 2, "two CTAs must fit on one SM");

enum { SRC_CACHE = 0, SRC_CHUNK = 1, SRC_RING = 2 };

struct TcArgs {
    LayerArgs a;
    int C;                 // chunk length
    int n_mtiles;          // ceil(C / 128)
    int n_ret_ctas;        // B * R * G * n_mtiles
    const int32_t* seq_len;
    const int32_t* ring_pos;
    int32_t* status;
    void* out;
};

// ------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// D (TMEM) = A (smem) * B (smem) [+ D]
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

#define DUO_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), \
                  "=r"(r[i + 6]), "=r"(r[i + 7])
#define DUO_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), "r"(r[i + 5]), \
                  "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive TMEM columns of this thread's lane -> registers (waits for the load)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : DUO_R8(0), DUO_R8(8), DUO_R8(16), DUO_R8(24)
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    uint32_t r[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        DUO_W8(0), DUO_W8(8), DUO_W8(16), DUO_W8(24)
        : "memory");
}

// 2^x on the SFU (PTX ex2.approx, flush-to-zero; 2^-inf = +0)
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout: start,
// leading and stride byte offsets >> 4, version 1, swizzle mode 2).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor for kind::f16: bf16 A and B, fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------ tile schedule

struct Sched {
    bool retrieval;
    int c0;          // chunk start position (cached tokens before the chunk)
    int m;           // query tile
    int n;           // tiles to visit
    int n_prior;     // retrieval: tiles from the full cache
    int n_ring;      // streaming: ring tiles
    int n_chunk;     // streaming: chunk tiles listed in chunk[]
    int chunk[kMaxChunkTiles];
};

struct Tile {
    int src, row, pos0;
    bool mask;
};

__device__ __forceinline__ Sched make_sched(const TcArgs& p, bool retrieval, int c0, int m) {
    const LayerArgs& a = p.a;
    Sched s;
    s.retrieval = retrieval;
    s.c0 = c0;
    s.m = m;
    const int q_last = min(p.C, BM * m + BM) - 1;    // last valid chunk row of this query tile
    if (retrieval) {
        s.n_prior = (c0 + BN - 1) / BN;
        s.n = s.n_prior + q_last / BN + 1;
        s.n_ring = s.n_chunk = 0;
    } else {
        s.n_prior = 0;
        const int held = min(c0, a.W);
        s.n_ring = (held + BN - 1) / BN;
        int lo = max(0, BM * m - a.recent + 1) / BN;
        const int hi = q_last / BN;
        int k = 0;
        if (c0 < a.sink && lo > 0) s.chunk[k++] = 0;   // the chunk's own sink tokens (sink <= 64)
        for (int u = lo; u <= hi && k < kMaxChunkTiles; ++u) s.chunk[k++] = u;
        s.n_chunk = k;
        s.n = s.n_ring + s.n_chunk;
    }
    return s;
}

__device__ __forceinline__ Tile tile_at(const Sched& s, int j) {
    Tile t;
    if (s.retrieval) {
        if (j < s.n_prior) {
            t.src = SRC_CACHE;
            t.row = s.c0 - BN * (s.n_prior - j);
            t.pos0 = t.row;
            t.mask = t.row < 0;
        } else {
            const int u = j - s.n_prior;
            t.src = SRC_CHUNK;
            t.row = BN * u;
            t.pos0 = s.c0 + BN * u;
            t.mask = u >= 2 * s.m;         // the two diagonal tiles of this 128-row query tile
        }
    } else if (j < s.n_ring) {
        t.src = SRC_RING;
        t.row = BN * j;
        t.pos0 = 0;
        t.mask = true;
    } else {
        const int u = s.chunk[j - s.n_ring];
        t.src = SRC_CHUNK;
        t.row = BN * u;
        t.pos0 = s.c0 + BN * u;
        t.mask = true;
    }
    return t;
}

// ------------------------------------------------------------------ kernel

__global__ void __launch_bounds__(kThreadsTC, 2)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                      const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKx,
                      const __grid_constant__ CUtensorMap tmVx, const __grid_constant__ CUtensorMap tmKr,
                      const __grid_constant__ CUtensorMap tmVr, const TcArgs p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const LayerArgs& a = p.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if ((smem_u32(smem) & 1023u) != 0) {   // the swizzled layouts need 1024-byte alignment
        if (tid == 0) atomicOr(p.status, DUO_DEV_BAD_LENGTH);
        return;
    }
    const uint32_t sQ = smem_u32(smem + kOffQ), sK = smem_u32(smem + kOffK), sV = smem_u32(smem + kOffV),
                   sP = smem_u32(smem + kOffP);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = bars + 3;
    uint64_t* v_full = bars + 5;
    uint64_t* v_empty = bars + 7;
    uint64_t* s_full = bars + 9;
    uint64_t* s_empty = bars + 11;
    uint64_t* p_full = bars + 13;
    uint64_t* o_done = bars + 14;
    uint32_t* holder = reinterpret_cast<uint32_t*>(smem + kOffHolder);
    int* sPos = reinterpret_cast<int*>(smem + kOffPos);

    // ------------------------------------------------------- work item
    const int per_m_ret = a.B * a.R * a.G, per_m_str = a.B * a.S * a.G;
    const bool retrieval = (int)blockIdx.x < p.n_ret_ctas;
    int idx = retrieval ? (int)blockIdx.x : (int)blockIdx.x - p.n_ret_ctas;
    const int per_m = retrieval ? per_m_ret : per_m_str;
    const int m = p.n_mtiles - 1 - idx / per_m;        // heaviest query tiles first
    idx %= per_m;
    const int g = idx % a.G;
    const int hs = (idx / a.G) % (retrieval ? a.R : a.S);
    const int b = idx / (a.G * (retrieval ? a.R : a.S));
    const int slot = retrieval ? hs : a.R + hs;
    const int q_idx = a.q_head0[slot] + g;
    const int kv_idx = a.kv_head[slot];
    int c0 = p.seq_len[b];
    if (c0 < 0) c0 = 0;
    if (retrieval && c0 > a.capacity) {
        if (tid == 0 && m == p.n_mtiles - 1) atomicOr(p.status, DUO_DEV_BAD_LENGTH);
        c0 = a.capacity;
    }
    const Sched sc = make_sched(p, retrieval, c0, m);
    const int n = sc.n;

    // ------------------------------------------------------- set-up
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], 4);
        }
        mbar_init(p_full, 4);
        mbar_init(o_done, 1);
        fence_barrier_init();
    }
    if (!retrieval)
        for (int i = tid; i < kMaxRing; i += kThreadsTC)
            sPos[i] = (i < a.W && c0 > 0) ? p.ring_pos[(size_t)b * a.W + i] : -1;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *holder;

    if (warp == kTmaWarp) {
        // --------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_map(&tmQ);
            mbar_arrive_expect_tx(q_full, kQBytes);
            tma_load_4d(sQ, &tmQ, 0, q_idx, BM * m, b, q_full);
            tma_load_4d(sQ + kQBytes / 2, &tmQ, 64, q_idx, BM * m, b, q_full);
            const int cache_z = b * a.R + slot, ring_z = b * a.S + (slot - a.R);
            for (int j = 0; j < n; ++j) {
                const Tile t = tile_at(sc, j);
                const int st = j & 1;
                for (int kv = 0; kv < 2; ++kv) {
                    uint64_t* full = kv ? &v_full[st] : &k_full[st];
                    uint64_t* empty = kv ? &v_empty[st] : &k_empty[st];
                    if (j >= 2 && !mbar_wait(empty, ((j >> 1) - 1) & 1, p.status)) goto producer_done;
                    mbar_arrive_expect_tx(full, kTileBytes);
                    const uint32_t dst = (kv ? sV : sK) + st * kTileBytes;
                    for (int half = 0; half < 2; ++half) {
                        const uint32_t d2 = dst + half * (kTileBytes / 2);
                        const int x = 64 * half;
                        if (t.src == SRC_CACHE)
                            tma_load_3d(d2, kv ? &tmVc : &tmKc, x, t.row, cache_z, full);
                        else if (t.src == SRC_CHUNK)
                            tma_load_4d(d2, kv ? &tmVx : &tmKx, x, kv_idx, t.row, b, full);
                        else
                            tma_load_3d(d2, kv ? &tmVr : &tmKr, x, t.row, ring_z, full);
                    }
                }
            }
        producer_done:;
        }
    } else if (warp == kMmaWarp) {
        // --------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(BM, HD, 0, 1);
            bool ok = mbar_wait(q_full, 0, p.status);
            auto issue_pv = [&](int i) {
                const int vs = i & 1;
                ok = ok && mbar_wait(p_full, i & 1, p.status);
                ok = ok && mbar_wait(&v_full[vs], (i >> 1) & 1, p.status);
                if (!ok) return;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t ad = sw128_desc(sP + kk * 32, 16, 1024);
                    const uint64_t bd = sw128_desc(sV + vs * kTileBytes + kk * 2048, kTileBytes / 2, 1024);
                    tc_mma(tmem + kColO, ad, bd, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(o_done);
                tc_commit(&v_empty[vs]);
            };
            for (int j = 0; j < n && ok; ++j) {
                const int st = j & 1;
                ok = ok && mbar_wait(&k_full[st], (j >> 1) & 1, p.status);
                if (j >= 2) ok = ok && mbar_wait(&s_empty[st], ((j >> 1) - 1) & 1, p.status);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint64_t ad = sw128_desc(sQ + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = sw128_desc(sK + st * kTileBytes + (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32,
                                                   16, 1024);
                    tc_mma(tmem + col_s(st), ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[st]);
                tc_commit(&k_empty[st]);
                if (j >= 1) issue_pv(j - 1);
            }
            if (ok && n >= 1) issue_pv(n - 1);
        }
    } else {
        // --------------------------------------------------- softmax
        const int row = tid;                                  // 0..127 = TMEM lane
        const int P = c0 + BM * m + row;                      // absolute query position
        const float sl = a.scale * kLog2e;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        float m_ref = -INFINITY, l_sum = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int st = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[st], (j >> 1) & 1, p.status));
            if (!ok) break;
            tc_fence_after();
            float s[64];
            {
                float lo[32], hi[32];
                tmem_ld32(lane_base + col_s(st), lo);
                tmem_ld32(lane_base + col_s(st) + 32, hi);
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    s[c] = lo[c];
                    s[32 + c] = hi[c];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[st]);       // one arrival per warp
            const Tile t = tile_at(sc, j);
            if (t.mask) {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const int kp = t.src == SRC_RING ? (t.row + c < a.W ? sPos[t.row + c] : -1) : t.pos0 + c;
                    bool vis = kp >= 0 && kp <= P;
                    if (!sc.retrieval) vis = vis && (kp < a.sink || P - kp < a.recent);
                    if (!vis) s[c] = -INFINITY;
                }
            }
            // row maximum of the raw scores (8 independent chains), then into
            // the log2 domain: the scale is positive, so it commutes with max
            float mx;
            {
                float m8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) m8[i] = s[i];
#pragma unroll
                for (int c = 8; c < 64; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
                mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                           fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                mx *= sl;
            }
            const float m_new = fmaxf(m_ref, mx);
            const bool need = m_new > m_ref + 8.f;            // lazy rescale threshold: 2^8
            const float m_use = need ? m_new : m_ref;
            const float m_safe = m_use == -INFINITY ? 0.f : m_use;
            const float corr = need ? exp2_approx(m_ref - m_use) : 1.f;
            // p = 2^(s*scale*log2e - m), rounded once to bf16 for the PV MMA;
            // the row sum uses the same rounded values, so each output is a
            // convex combination of V rows
            uint32_t pk[32];
            float rs8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) rs8[i] = 0.f;
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) {
                const float p0 = exp2_approx(fmaf(s[2 * c2], sl, -m_safe));
                const float p1 = exp2_approx(fmaf(s[2 * c2 + 1], sl, -m_safe));
                __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                pk[c2] = *reinterpret_cast<uint32_t*>(&h);
                rs8[c2 & 7] += bf16_lo(pk[c2]) + bf16_hi(pk[c2]);
            }
            const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
            l_sum = l_sum * corr + rs;
            m_ref = m_use;
            if (j >= 1) {
                ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, p.status));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        float o[32];
                        tmem_ld32(lane_base + kColO + 32 * ch, o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= corr;
                        tmem_st32(lane_base + kColO + 32 * ch, o);
                    }
                    tmem_wait_st();
                }
            }
            // P row -> shared memory, K-major with the 128-byte swizzle
            uint8_t* prow = smem + kOffP + row * 128;
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16)
                *reinterpret_cast<uint4*>(prow + ((c16 ^ (row & 7)) * 16)) =
                    make_uint4(pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);               // one arrival per warp
        }
        // epilogue: O / l -> bf16
        if (ok && n >= 1) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (n - 1) & 1, p.status));
        if (ok) {
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            const int crow = BM * m + row;
            __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.out) + (((size_t)b * p.C + crow) * a.Hq + q_idx) * HD;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                tmem_ld32(lane_base + kColO + 32 * ch, o);
                if (crow < p.C) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v8[e] = o[8 * q4 + e] * inv;
                        store_row<__nv_bfloat16, 8>(op + 32 * ch + 8 * q4, v8);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

}  // namespace

bool prefill_tc_supported(const LayerArgs& a) {
    return a.dtype == DUO_BF16 && a.D == HD && a.page_size == 0 && a.sink <= BN && a.W <= kMaxRing &&
           a.recent <= 256;
}

cudaError_t launch_prefill_tc(const LayerArgs& a, const CacheArgs& c, const void* q, const void* k_chunk,
                              const void* v_chunk, int C, void* out, cudaStream_t s) {
    if (!prefill_tc_supported(a)) return cudaErrorNotSupported;
    const uint64_t row = HD * 2;
    CUtensorMap mQ, mKx, mVx, mKc, mVc, mKr, mVr;
    {
        const uint64_t d[4] = {HD, (uint64_t)a.Hq, (uint64_t)C, (uint64_t)a.B};
        const uint64_t st[3] = {row, row * a.Hq, row * a.Hq * C};
        const uint32_t bx[4] = {64, 1, BM, 1};
        if (!encode_tmap_bf16(&mQ, q, 4, d, st, bx)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t d[4] = {HD, (uint64_t)a.Hkv, (uint64_t)C, (uint64_t)a.B};
        const uint64_t st[3] = {row, row * a.Hkv, row * a.Hkv * C};
        const uint32_t bx[4] = {64, 1, BN, 1};
        if (!encode_tmap_bf16(&mKx, k_chunk, 4, d, st, bx) || !encode_tmap_bf16(&mVx, v_chunk, 4, d, st, bx))
            return cudaErrorInvalidValue;
    }
    const uint32_t bx3[3] = {64, BN, 1};
    if (a.R > 0) {
        const uint64_t d[3] = {HD, (uint64_t)a.capacity, (uint64_t)a.B * a.R};
        const uint64_t st[2] = {row, row * a.capacity};
        if (!encode_tmap_bf16(&mKc, c.k_full, 3, d, st, bx3) || !encode_tmap_bf16(&mVc, c.v_full, 3, d, st, bx3))
            return cudaErrorInvalidValue;
    } else {
        mKc = mKx;  // never read: there are no retrieval heads
        mVc = mVx;
    }
    if (a.S > 0) {
        const uint64_t d[3] = {HD, (uint64_t)a.W, (uint64_t)a.B * a.S};
        const uint64_t st[2] = {row, row * a.W};
        if (!encode_tmap_bf16(&mKr, c.k_ring, 3, d, st, bx3) || !encode_tmap_bf16(&mVr, c.v_ring, 3, d, st, bx3))
            return cudaErrorInvalidValue;
    } else {
        mKr = mKx;  // never read: there are no streaming heads
        mVr = mVx;
    }
    TcArgs p;
    p.a = a;
    p.C = C;
    p.n_mtiles = (C + BM - 1) / BM;
    p.n_ret_ctas = a.B * a.R * a.G * p.n_mtiles;
    p.seq_len = c.seq_len;
    p.ring_pos = c.ring_pos;
    p.status = c.status;
    p.out = out;
    const long grid = (long)a.B * a.Hkv * a.G * p.n_mtiles;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffffL) return cudaErrorInvalidConfiguration;
    static bool configured = false;  // function attributes are per process, set once
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    prefill_tc_kernel<<<(unsigned)grid, kThreadsTC, kSmemBytes, s>>>(mQ, mKc, mVc, mKx, mVx, mKr, mVr, p);
    return cudaGetLastError();
}

}  // namespace duo
