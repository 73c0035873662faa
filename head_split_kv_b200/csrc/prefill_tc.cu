// prefill_tc.cu -- chunked pre-fill attention on the 5th-generation tensor
// cores: two query tiles per CTA share every K/V tile, S and P live in TMEM.
//
// [Summary S2 "Chunked Pre-filling": fixed-length prompt chunks; both caches
//  are pre-filled.  Review S3 "Inference flow", pre-fill: retrieval heads use
//  full (FlashAttention-style) causal attention; streaming heads run in linear
//  time and constant memory.]
//
// One CTA (one per SM: 193 KB of shared memory, all 512 TMEM columns) owns
// 256 query rows of one query head, as two 128-row tiles Q0 (chunk rows
// 256m .. 256m+127) and Q1 (256m+128 .. 256m+255), and walks 128-key tiles:
//   retrieval head: every prior key from the full cache (tiles aligned to end
//     at the chunk start c0) and the chunk's own keys up to Q1's diagonal; Q0
//     stops one tile earlier when the last tile lies wholly above its diagonal;
//   streaming head: the ring (sinks + recent tokens before c0, positions from
//     ring_pos), the chunk's sink tile when c0 < sink, and the chunk tiles of
//     the two tiles' recent bands -- a handful of tiles at any context length;
//     in whole-chunk mode (DUO_STREAM_CHUNK) the ring, then the chunk's keys up
//     to Q1's diagonal, masked like a retrieval head's chunk tiles.
// TMEM: S0 | S1 | O0 | O1, 128 columns each.  After softmax warpgroup i has
// read S_i it writes P_i as packed bf16 over the last 64 columns of S_i, and
// the PV product reads P_i from TMEM (the A operand), so P never touches
// shared memory and the tensor core's shared-memory reads per FLOP are
// half those of 64-key tiles with P staged in shared memory.
// Roles (320 threads):
//   warps 0-3  softmax of Q0 (thread t owns row t = TMEM lane t),
//   warps 4-7  softmax of Q1 (warp w reads lanes 32 (w % 4) ..),
//   warp 8     TMA producer: Q0 and Q1 once, then K and V tiles into 2-stage
//              rings (64-column x 64-row boxes, 128-byte swizzle),
//   warp 9     MMA issuer (one thread), in the order
//                QK0(0) QK1(0) | PV0(0) QK0(1) PV1(0) QK1(1) | PV0(1) ...
//              so that while one softmax warpgroup works on its S, the tensor
//              core multiplies the other tile's operands.
// Softmax keeps the running maximum in the log2 domain with a lazy O rescale
// (only when the maximum grows by more than 2^8; the commit that signals S_i
// also covers the previous PV_i, so O_i is complete when it is rescaled) and
// at the end divides O by the row sum and stores bf16.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace duo {
namespace {

constexpr int BM = 128;            // query rows per tile (two tiles per CTA)
constexpr int BN = 128;            // keys per K/V tile
constexpr int HD = 128;            // head dim
constexpr int kBox = 64;           // rows per TMA box (tiles are loaded as 2 x 2 boxes)
constexpr int kTmaWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ constexpr uint32_t col_s(int i) { return 128u * (uint32_t)i; }       // S_i (and P_i)
__device__ __forceinline__ constexpr uint32_t col_o(int i) { return 256u + 128u * (uint32_t)i; }  // O_i
constexpr int kMaxRing = 128;      // sink + recent held by one tile

constexpr uint32_t kQBytes = BM * HD * 2;      // 32 KB per query tile (two 16 KB halves of d)
constexpr uint32_t kTileBytes = BN * HD * 2;   // 32 KB per K or V tile (two 16 KB halves of d)
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr uint32_t kBoxBytes = kBox * 128;     // 8 KB: 64 rows x 64 columns
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + 2 * kQBytes;
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;
constexpr uint32_t kOffBar = kOffV + 2 * kTileBytes;
constexpr uint32_t kOffHolder = kOffBar + 16 * 8;
constexpr uint32_t kSmemBytes = kOffHolder + 16;
static_assert(kSmemBytes + 1024 <= 232448, "one CTA per SM");

enum { SRC_CACHE = 0, SRC_CHUNK = 1, SRC_RING = 2 };

struct TcArgs {
    LayerArgs a;
    int C;                 // chunk length
    int n_mpairs;          // ceil(C / 256)
    int n_ret_ctas;        // B * R * G * n_mpairs
    const int32_t* seq_len;
    int32_t* status;
    void* out;
};

// ------------------------------------------------------------ tile schedule
//
// Tiles are listed in visiting order; tile j is described by tile_at(j).
struct Sched {
    bool retrieval;
    bool chunk;      // streaming head in whole-chunk mode: ring, then the chunk causally
    int c0;          // chunk start position (cached tokens before the chunk)
    int m;           // query-tile pair: chunk rows 256m .. 256m+255
    int n;           // tiles visited by Q1
    int n0;          // tiles visited by Q0 (n or n - 1)
    int n_prior;     // retrieval: tiles from the full cache
    int n_ring;      // streaming: ring tiles (0 or 1)
    int sink_tile;   // streaming: 1 if the chunk's tile 0 is listed before the band
    int lo;          // first chunk tile of the band (streaming) / 0 (retrieval)
};

struct Tile {
    int src, row, pos0;
};

__device__ __forceinline__ Sched make_sched(const TcArgs& p, bool retrieval, int c0, int m) {
    const LayerArgs& a = p.a;
    Sched s;
    s.retrieval = retrieval;
    s.c0 = c0;
    s.m = m;
    const int n_ct = (p.C + BN - 1) / BN;                 // chunk tiles that hold keys
    const int hi = min(2 * m + 1, n_ct - 1);              // last chunk tile (Q1's diagonal)
    s.chunk = !retrieval && a.stream_chunk;
    if (retrieval) {
        s.n_prior = (c0 + BN - 1) / BN;
        s.n_ring = 0;
        s.sink_tile = 0;
        s.lo = 0;
        s.n = s.n_prior + hi + 1;
    } else if (s.chunk) {
        s.n_prior = 0;
        s.n_ring = min(c0, a.W) > 0 ? 1 : 0;
        s.sink_tile = 0;
        s.lo = 0;
        s.n = s.n_ring + hi + 1;
    } else {
        s.n_prior = 0;
        s.n_ring = min(c0, a.W) > 0 ? 1 : 0;
        s.lo = max(0, 2 * BM * m - a.recent + 1) / BN;    // first key of Q0's band
        s.sink_tile = (c0 < a.sink && s.lo > 0) ? 1 : 0;  // the chunk's own sink tokens (sink <= 128)
        s.n = s.n_ring + s.sink_tile + (hi - s.lo + 1);
    }
    // Q0's rows end at 256m + 127: the tile 2m + 1, when listed, lies wholly
    // above its diagonal and is the last one
    s.n0 = (hi == 2 * m + 1) ? s.n - 1 : s.n;
    return s;
}

__device__ __forceinline__ Tile tile_at(const Sched& s, int j) {
    Tile t;
    if (s.retrieval) {
        if (j < s.n_prior) {
            t.src = SRC_CACHE;
            t.row = s.c0 - BN * (s.n_prior - j);
            t.pos0 = t.row;
        } else {
            const int u = j - s.n_prior;
            t.src = SRC_CHUNK;
            t.row = BN * u;
            t.pos0 = s.c0 + BN * u;
        }
    } else if (j < s.n_ring) {
        t.src = SRC_RING;
        t.row = 0;
        t.pos0 = 0;
    } else {
        const int k = j - s.n_ring;
        const int u = (s.sink_tile && k == 0) ? 0 : s.lo + k - s.sink_tile;
        t.src = SRC_CHUNK;
        t.row = BN * u;
        t.pos0 = s.c0 + BN * u;
    }
    return t;
}

// Whether query tile `qi` needs the mask on tile j: every Lambda-mode
// streaming tile and ring tile, the retrieval tile that starts before
// position 0, and the chunk tiles that reach past the query tile's first row.
__device__ __forceinline__ bool needs_mask(const Sched& s, const Tile& t, int qi) {
    if (!s.retrieval && !s.chunk) return true;
    if (t.src == SRC_RING) return true;
    if (t.src == SRC_CACHE) return t.row < 0;
    return t.row + BN - 1 > BM * (2 * s.m + qi);
}

// ------------------------------------------------------------------ masks
//
// A row's visible keys in one 128-key tile, set as bits (column c = bit c % 32
// of word c / 32), so that masking costs a bit test per score.  The ranges
// follow from the key positions of the tile:
//   cache / chunk tile, keys pos0 + c: causal (retrieval head, whole-chunk
//     streaming head) c <= P - pos0 and pos0 + c >= 0; Lambda streaming head
//     additionally pos0 + c < sink or pos0 + c > P - recent;
//   ring tile, the streaming cache as it stood at the chunk start c0: slot s
//     < min(c0, sink) holds sink s; the recent slots hold positions
//     max(sink, c0 - recent) .. c0 - 1, position p in slot
//     sink + (p - sink) % recent.  Whole-chunk mode sees all of them, Lambda
//     mode the positions above P - recent.

// columns lo .. hi (inclusive, clipped to the tile)
__device__ __forceinline__ void set_columns(uint32_t (&m)[4], int lo, int hi) {
    lo = max(lo, 0);
    hi = min(hi, BN - 1);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const int a = max(lo - 32 * w, 0), b = min(hi - 32 * w, 31);
        if (a <= b) m[w] |= (0xffffffffu >> (31 - b)) & (0xffffffffu << a);
    }
}

__device__ __forceinline__ void visible_columns(const LayerArgs& a, const Sched& sc, const Tile& t, int P,
                                                uint32_t (&m)[4]) {
    if (t.src != SRC_RING) {
        const int last = P - t.pos0;                      // causal: columns 0 .. last
        if (sc.retrieval || sc.chunk) {
            set_columns(m, -t.pos0, last);
        } else {
            set_columns(m, 0, min(last, a.sink - 1 - t.pos0));
            set_columns(m, P - a.recent + 1 - t.pos0, last);
        }
        return;
    }
    const int c0 = sc.c0;
    set_columns(m, 0, min(c0, a.sink) - 1);               // the sinks
    int lo = max(a.sink, c0 - a.recent);                  // oldest recent position held
    if (!sc.chunk) lo = max(lo, P - a.recent + 1);
    const int len = c0 - lo;                              // positions lo .. c0 - 1
    if (len <= 0) return;
    const int start = (lo - a.sink) % a.recent;           // slot of lo, relative to the recent block
    set_columns(m, a.sink + start, a.sink + min(start + len, a.recent) - 1);
    if (start + len > a.recent) set_columns(m, a.sink, a.sink + start + len - a.recent - 1);
}

// ------------------------------------------------------------------ softmax

// One row's share of one tile: S (128 columns at s_addr) from TMEM, the
// running maximum m_ref (log2 domain, lazy: raised only when the tile's
// maximum exceeds it by more than 2^8) and row sum l_sum updated, and
// p = 2^(s * scale * log2e - m) written back as packed bf16 over the second
// half of S for the PV MMA.  Returns the factor by which O must be rescaled
// (1 unless `need`).
//
// S is read in two 64-column halves (a whole row would need more registers
// than three warps per SM sub-partition leave): keys 0..63 for the maximum
// only, then keys 64..127, which stay in registers; p of keys 64..127 goes to
// columns 96..127, then keys 0..63 (loaded again) to columns 64..95.  The row
// sum adds the rounded p, so each output is a convex combination of V rows.
__device__ __forceinline__ float softmax_tile(uint32_t s_addr, float sl, float& m_ref, float& l_sum, bool& need) {
    // maximum of 64 raw scores: three-input max, 4 chains
    auto max_half = [](const float (&v)[64]) {
        float m4[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
        for (int c = 4; c < 60; c += 8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) m4[i] = fmax3(m4[i], v[c + i], v[c + 4 + i]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) m4[i] = fmaxf(m4[i], v[60 + i]);
        return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
    };
    float s[64];
    tmem_ld64(s_addr, s);
    float mx = max_half(s);
    tmem_ld64(s_addr + 64, s);
    // into the log2 domain: the scale is positive, so it commutes with max
    mx = fmaxf(mx, max_half(s)) * sl;
    const float m_new = fmaxf(m_ref, mx);
    need = m_new > m_ref + 8.f;                           // lazy rescale threshold: 2^8
    const float m_use = need ? m_new : m_ref;
    const float m_safe = m_use == -INFINITY ? 0.f : m_use;
    const float corr = need ? exp2_approx(m_ref - m_use) : 1.f;
    const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(-m_safe, -m_safe);
    float2 rs2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    auto exp_half = [&](const float (&v)[64], uint32_t taddr) {
        uint32_t pk[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
            const float2 x = ffma2(make_float2(v[2 * c2], v[2 * c2 + 1]), sl2, nm2);
            const float2 e = make_float2(exp2_approx(x.x), exp2_approx(x.y));
            __nv_bfloat162 hb = __floats2bfloat162_rn(e.x, e.y);
            pk[c2] = *reinterpret_cast<uint32_t*>(&hb);
            rs2[c2 & 3] = fadd2(rs2[c2 & 3], make_float2(bf16_lo(pk[c2]), bf16_hi(pk[c2])));
        }
        tmem_st32(taddr, pk);
    };
    exp_half(s, s_addr + 96);
    tmem_ld64(s_addr, s);
    exp_half(s, s_addr + 64);
    const float rs = ((rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y)) + ((rs2[2].x + rs2[2].y) + (rs2[3].x + rs2[3].y));
    l_sum = l_sum * corr + rs;
    m_ref = m_use;
    return corr;
}

// A masked tile (diagonal, first prior tile, streaming tiles): this row's
// invisible scores are overwritten with -inf in TMEM, so the softmax itself
// never tests a mask and keeps no mask state across its loop.  Costs one more
// TMEM round trip on the few masked tiles of a query tile; a streaming tile
// is 6x cheaper than with a per-score position test.
__device__ __forceinline__ void mask_tile_in_tmem(const LayerArgs& a, const Sched& sc, const Tile& t, int P,
                                               uint32_t s_addr) {
    uint32_t vis[4] = {0u, 0u, 0u, 0u};   // the tile's keys this row sees, a bit per column
    visible_columns(a, sc, t, P, vis);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float v[64];
        tmem_ld64(s_addr + 64 * h, v);
        uint32_t r[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const int col = 64 * h + 32 * half + c;
                r[c] = ((vis[col >> 5] >> (col & 31)) & 1u) ? __float_as_uint(v[32 * half + c])
                                                            : __float_as_uint(-INFINITY);
            }
            tmem_st32(s_addr + 64 * h + 32 * half, r);
        }
    }
    tmem_wait_st();
}

// ------------------------------------------------------------------ kernel

__global__ void __launch_bounds__(kThreads, 1)
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
    const uint32_t sQ = smem_u32(smem + kOffQ), sK = smem_u32(smem + kOffK), sV = smem_u32(smem + kOffV);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;    // [2]
    uint64_t* k_empty = bars + 3;   // [2]
    uint64_t* v_full = bars + 5;    // [2]
    uint64_t* v_empty = bars + 7;   // [2]
    uint64_t* s_full = bars + 9;    // [2]: per query tile
    uint64_t* p_full = bars + 11;   // [2]: per query tile
    uint64_t* o_done = bars + 13;   // [2]: per query tile, once
    uint32_t* holder = reinterpret_cast<uint32_t*>(smem + kOffHolder);

    // ------------------------------------------------------- work item
    const int per_m_ret = a.B * a.R * a.G, per_m_str = a.B * a.S * a.G;
    const bool retrieval = (int)blockIdx.x < p.n_ret_ctas;
    int idx = retrieval ? (int)blockIdx.x : (int)blockIdx.x - p.n_ret_ctas;
    const int per_m = retrieval ? per_m_ret : per_m_str;
    const int m = p.n_mpairs - 1 - idx / per_m;        // heaviest query tiles first
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
        if (tid == 0 && m == p.n_mpairs - 1) atomicOr(p.status, DUO_DEV_BAD_LENGTH);
        c0 = a.capacity;
    }
    const Sched sc = make_sched(p, retrieval, c0, m);

    // ------------------------------------------------------- set-up
    if (warp == kMmaWarp) tmem_alloc(holder, kTmemCols);
    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&o_done[i], 1);
        }
        fence_barrier_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *holder;

    if (warp == kTmaWarp) {
        // --------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_map(&tmQ);
            mbar_arrive_expect_tx(q_full, 2 * kQBytes);
            for (int qi = 0; qi < 2; ++qi)
                for (int half = 0; half < 2; ++half)
                    tma_load_4d(sQ + qi * kQBytes + half * (kQBytes / 2), &tmQ, 64 * half, q_idx, BM * (2 * m + qi),
                                b, q_full);
            const int cache_z = b * a.R + slot, ring_z = b * a.S + (slot - a.R);
            for (int j = 0; j < sc.n; ++j) {
                const Tile t = tile_at(sc, j);
                const int st = j & 1;
                for (int kv = 0; kv < 2; ++kv) {
                    uint64_t* full = kv ? &v_full[st] : &k_full[st];
                    uint64_t* empty = kv ? &v_empty[st] : &k_empty[st];
                    if (j >= 2 && !mbar_wait(empty, ((j >> 1) - 1) & 1, p.status)) goto producer_done;
                    mbar_arrive_expect_tx(full, kTileBytes);
                    const uint32_t dst = (kv ? sV : sK) + st * kTileBytes;
                    for (int half = 0; half < 2; ++half)
                        for (int rh = 0; rh < 2; ++rh) {
                            const uint32_t d2 = dst + half * kHalfBytes + rh * kBoxBytes;
                            const int x = 64 * half, row = t.row + kBox * rh;
                            if (t.src == SRC_CACHE)
                                tma_load_3d(d2, kv ? &tmVc : &tmKc, x, row, cache_z, full);
                            else if (t.src == SRC_CHUNK)
                                tma_load_4d(d2, kv ? &tmVx : &tmKx, x, kv_idx, row, b, full);
                            else
                                tma_load_3d(d2, kv ? &tmVr : &tmKr, x, row, ring_z, full);
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
            const int n = sc.n, n0 = sc.n0;
            bool ok = mbar_wait(q_full, 0, p.status);
            // S_qi = Q_qi K_j^T: 8 MMAs of K 16 over the two 64-column halves of d
            auto issue_qk = [&](int qi, int j) {
                const int st = j & 1;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint64_t ad =
                        sw128_desc(sQ + qi * kQBytes + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = sw128_desc(sK + st * kTileBytes + (kk >> 2) * kHalfBytes + (kk & 3) * 32, 16,
                                                   1024);
                    tc_mma(tmem + col_s(qi), ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[qi]);
            };
            // O_qi += P_qi V_j: P from TMEM (columns 64..127 of S_qi, 8 per K 16), V
            // read MN-major
            auto issue_pv = [&](int qi, int j) {
                const int st = j & 1;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bd = sw128_desc(sV + st * kTileBytes + kk * 2048, kHalfBytes, 1024);
                    tc_mma_ta(tmem + col_o(qi), tmem + col_s(qi) + 64 + 8 * kk, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
            };
            ok = ok && mbar_wait(&k_full[0], 0, p.status);
            if (ok) {
                tc_fence_after();
                if (n0 > 0) issue_qk(0, 0);
                issue_qk(1, 0);
                tc_commit(&k_empty[0]);
            }
            for (int j = 0; j < n && ok; ++j) {
                const bool next = j + 1 < n;
                if (next) ok = ok && mbar_wait(&k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, p.status);
                ok = ok && mbar_wait(&v_full[j & 1], (j >> 1) & 1, p.status);
                if (j < n0) {
                    ok = ok && mbar_wait(&p_full[0], j & 1, p.status);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(0, j);
                    if (j == n0 - 1) tc_commit(&o_done[0]);
                    if (j + 1 < n0) issue_qk(0, j + 1);
                }
                ok = ok && mbar_wait(&p_full[1], j & 1, p.status);
                if (!ok) break;
                tc_fence_after();
                issue_pv(1, j);
                tc_commit(&v_empty[j & 1]);
                if (j == n - 1) tc_commit(&o_done[1]);
                if (next) {
                    issue_qk(1, j + 1);
                    tc_commit(&k_empty[(j + 1) & 1]);
                }
            }
        }
    } else {
        // --------------------------------------------------- softmax
        const int qi = warp >> 2;                             // query tile of this warpgroup
        const int row = tid & 127;                            // TMEM lane
        const int crow = BM * (2 * m + qi) + row;             // chunk row
        const int P = c0 + crow;                              // absolute query position
        const int n_me = qi ? sc.n : sc.n0;
        const float sl = a.scale * kLog2e;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        float m_ref = -INFINITY, l_sum = 0.f;
        bool ok = true;
        for (int j = 0; j < n_me; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[qi], j & 1, p.status));
            if (!ok) break;
            tc_fence_after();
            const Tile t = tile_at(sc, j);
            if (needs_mask(sc, t, qi)) mask_tile_in_tmem(a, sc, t, P, lane_base + col_s(qi));
            bool need;
            const float corr = softmax_tile(lane_base + col_s(qi), sl, m_ref, l_sum, need);
            // O_qi holds every PV up to tile j - 1 (the commit behind s_full
            // covered them); rescale it before PV_qi(j) is issued
            if (j >= 1 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    float o[32];
                    tmem_ld32(lane_base + col_o(qi) + 32 * ch, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= corr;
                    tmem_st32f(lane_base + col_o(qi) + 32 * ch, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[qi]);          // one arrival per warp
        }
        // epilogue: O / l -> bf16
        if (ok && n_me >= 1) ok = __all_sync(0xffffffffu, mbar_wait(&o_done[qi], 0, p.status));
        if (ok && n_me >= 1) {
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.out) + (((size_t)b * p.C + crow) * a.Hq + q_idx) * HD;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                tmem_ld32(lane_base + col_o(qi) + 32 * ch, o);
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
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool prefill_tc_supported(const LayerArgs& a) {
    return a.dtype == DUO_BF16 && a.D == HD && a.page_size == 0 && a.sink <= BN && a.W <= kMaxRing;
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
        const uint32_t bx[4] = {64, 1, kBox, 1};
        if (!encode_tmap_bf16(&mKx, k_chunk, 4, d, st, bx) || !encode_tmap_bf16(&mVx, v_chunk, 4, d, st, bx))
            return cudaErrorInvalidValue;
    }
    const uint32_t bx3[3] = {64, kBox, 1};
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
    p.n_mpairs = (C + 2 * BM - 1) / (2 * BM);
    p.n_ret_ctas = a.B * a.R * a.G * p.n_mpairs;
    p.seq_len = c.seq_len;
    p.status = c.status;
    p.out = out;
    const long grid = (long)a.B * a.Hkv * a.G * p.n_mpairs;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffffL) return cudaErrorInvalidConfiguration;
    static bool configured = false;  // function attributes are per process, set once
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(kSmemBytes + 1024));
        if (e != cudaSuccess) return e;
        configured = true;
    }
    prefill_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes + 1024, s>>>(mQ, mKc, mVc, mKx, mVx, mKr, mVr, p);
    return cudaGetLastError();
}

}  // namespace duo
