// prefill_tc.cu -- chunked pre-fill attention on the 5th-generation tensor
// cores: two query tiles per CTA share every K/V tile, S and P live in TMEM.
//
// [Summary S2 "Chunked Pre-filling": fixed-length prompt chunks; both caches
//  are pre-filled.  Review S3 "Inference flow", pre-fill: retrieval heads use
//  full (FlashAttention-style) causal attention; streaming heads run in linear
//  time and constant memory.]
//
// One CTA (one per SM: 198 KB of shared memory, all 512 TMEM columns) owns
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
// Key-range splits: with a workspace, a long retrieval unit (one query-tile
// pair of one query head) is taken by ns CTAs, each over 1/ns of its key
// tiles, so that the chunk's CTAs fill whole waves of SMs; each writes its
// rows' (m, l, O) to the workspace and the CTA that takes the unit's last
// ticket merges them (prefill_plan picks ns on the host).
// Gated mix: with no length array every sequence starts at position 0 and the
// launch covers whole sequences.  Two other epilogues serve it (compile-time
// variants, so the pre-fill carries neither): EPI_MIX reads back the
// streaming attention an earlier launch left in out and stores
// alpha * (this causal attention) + (1 - alpha) * (that); EPI_DOT stores
// nothing and adds sign * <dout row, attention row> over the CTA's rows into
// dalpha[kv] (the gate gradient, one launch per sign).  Both load the row
// they combine with before waiting for the last MMAs, so its latency hides
// behind them.
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
constexpr int kMaxSplit = 8;       // key-range splits per retrieval unit
constexpr int kMinSplitTiles = 48; // no split shorter than 48 key tiles (6,144 keys)
// One query tile's partial record of one split: the lazily raised row maxima
// (log2 domain), the row sums, then O unnormalised as [32 column groups][128
// rows][4], so that a warp's 32 rows write one 512-byte run per group.
constexpr int kPartFloats = 2 * BM + BM * HD;

constexpr uint32_t kQBytes = BM * HD * 2;      // 32 KB per query tile (two 16 KB halves of d)
constexpr uint32_t kTileBytes = BN * HD * 2;   // 32 KB per K or V tile (two 16 KB halves of d)
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr uint32_t kBoxBytes = kBox * 128;     // 8 KB: 64 rows x 64 columns
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + 2 * kQBytes;
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;
constexpr uint32_t kOffBar = kOffV + 2 * kTileBytes;
constexpr uint32_t kOffHolder = kOffBar + 16 * 8;
// quantized prior tiles: the tile's 128 k scales, then its 128 v scales / 16,
// four tiles deep (a K stage is refilled after its QK MMAs, while the softmax
// may still be on that tile; four slots outlast it -- see the producer)
constexpr uint32_t kScaleTileBytes = 2 * BN * 4;
constexpr uint32_t kOffScale = kOffHolder + 128;  // a tensor copy's shared destination is 128-byte aligned
constexpr uint32_t kSmemBytes = kOffScale + 4 * kScaleTileBytes;
static_assert(kSmemBytes + 1024 <= 232448, "one CTA per SM");
static_assert(kOffQ % 1024 == 0 && kOffK % 1024 == 0 && kOffV % 1024 == 0, "swizzled TMA destinations");
static_assert(kOffScale % 128 == 0 && kScaleTileBytes % 128 == 0, "TMA destinations");

enum { SRC_CACHE = 0, SRC_CHUNK = 1, SRC_RING = 2 };

struct TcArgs {
    LayerArgs a;
    int C;                 // chunk length
    int n_mpairs;          // ceil(C / 256)
    int n_units;           // retrieval units B * R * G * n_mpairs
    int ns;                // CTAs per retrieval unit (key-range splits; 1 = none)
    int n_ret_ctas;        // n_units * ns
    float* part;           // [n_units][ns][2][kPartFloats] partial records (ns > 1)
    uint32_t* ticket;      // [n_units] arrivals; the last split merges them
    EpiArgs epi;           // gated-mix epilogues (EPI_MIX, EPI_DOT)
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

constexpr int kFmaExpEvery = 4;   // one exp2 pair in 4 on the FMA pipe

// 2^x for a pair of x <= 0 (or -inf) on the FMA pipe, by Cody-Waite range
// reduction and a polynomial: x = n + f with n = rint(x) (adding 1.5 * 2^23
// rounds x to an integer held in the low mantissa bits) and f in [-0.5, 0.5];
// 2^f by a cubic whose coefficients were fitted here to minimise the largest
// relative error on [-0.5, 0.5] (7.5e-5, far below the 2^-9 half-step of the
// bf16 p it feeds); 2^n by adding n to the exponent field.  x is clamped at
// -125 so that the exponent stays normal: a masked key (x = -inf) gets
// about 2^-125 instead of 0, 1e-38 of the row's largest weight.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    constexpr float kShift = 12582912.f;  // 1.5 * 2^23
    constexpr float c0 = 0.9999280571937561f, c1 = 0.6932610273361206f, c2 = 0.24261116981506348f,
                    c3 = 0.055171627551317215f;
    x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
    const float2 t = fadd2(x, make_float2(kShift, kShift));
    const float2 n = fadd2(t, make_float2(-kShift, -kShift));
    const float2 f = ffma2(n, make_float2(-1.f, -1.f), x);
    float2 q = ffma2(make_float2(c3, c3), f, make_float2(c2, c2));
    q = ffma2(q, f, make_float2(c1, c1));
    q = ffma2(q, f, make_float2(c0, c0));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

// One row's share of one tile: S (128 columns at s_addr) from TMEM in one
// round trip, the keys the row does not see set to -inf when `masked` (bit c
// of vis = column c visible), the running maximum m_ref (log2 domain, lazy:
// raised only when the tile's maximum exceeds it by more than 2^8) and row sum
// l_sum updated, and p = 2^(s * scale * log2e - m) written back as packed bf16
// over the second half of S for the PV MMA (keys 0..63 to columns 64..95,
// keys 64..127 to columns 96..127).  Returns the factor by which O must be
// rescaled (1 unless `need`).  The row sum adds the rounded p, so each output
// is a convex combination of V rows (summing the fp32 exponentials instead
// is two integer operations a pair cheaper, but lets the weights drift from
// summing to 1 by the bf16 rounding, which put outputs of magnitude 4..8
// beyond the 2e-2 bound).
//
// The exponentials: one tile costs a softmax warp 128 exp2 per row, as many
// cycles on the SFU as the tile's two MMAs take on the tensor core, so the
// SFU is the co-bottleneck.  One pair in kFmaExpEvery is computed on the FMA
// pipe instead (exp2_fma2).  Measured on the 131K prompt: one pair in 4 or
// in 8 (equal within run-to-run noise) beat SFU-only by 2-5 %; one in 3 was
// slower.
//
// qsc (a quantized layer's prior tile, else NULL): the tile's keys are
// codes, and qsc holds the keys' k scales, then their v scales / 16 (read
// four at a time): the scores are multiplied by
// the k scales before anything else, and p by v scale / 16 on the way to the
// PV operand, which is fp16 for these tiles (the V codes are staged times 16
// in fp16, exactly): fp16's 11-bit significand keeps the rounding of p times
// the scale, which the row sum (of the unscaled fp32 p) cannot absorb, at
// 2^-11 of the value.  p <= 2^8 (the lazy rescale) keeps p v_scale / 16
// within fp16 for v scales up to 4095.  Other tiles: P in bf16, the row sum
// of the rounded P.
__device__ __forceinline__ float softmax_tile(uint32_t s_addr, float sl, bool masked, const uint32_t (&vis)[4],
                                              float& m_ref, float& l_sum, bool& need, const float* qsc) {
    float s[128];
    tmem_ld128(s_addr, s);
    if (qsc) {
        const float4* k4 = reinterpret_cast<const float4*>(qsc);
#pragma unroll
        for (int i = 0; i < 32; ++i) {   // packed fp32 pairs: one instruction per two scores
            const float4 ks = k4[i];
            const float2 a = fmul2(make_float2(s[4 * i], s[4 * i + 1]), make_float2(ks.x, ks.y));
            const float2 b = fmul2(make_float2(s[4 * i + 2], s[4 * i + 3]), make_float2(ks.z, ks.w));
            s[4 * i] = a.x;
            s[4 * i + 1] = a.y;
            s[4 * i + 2] = b.x;
            s[4 * i + 3] = b.y;
        }
    }
    if (masked) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
            if (!((vis[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
    }
    // maximum of the raw scores: three-input max, 4 chains
    float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
    for (int c = 4; c < 124; c += 8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) m4[i] = fmax3(m4[i], s[c + i], s[c + 4 + i]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) m4[i] = fmaxf(m4[i], s[124 + i]);
    // into the log2 domain: the scale is positive, so it commutes with max
    const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl;
    const float m_new = fmaxf(m_ref, mx);
    need = m_new > m_ref + 8.f;                           // lazy rescale threshold: 2^8
    const float m_use = need ? m_new : m_ref;
    const float m_safe = m_use == -INFINITY ? 0.f : m_use;
    const float corr = need ? exp2_approx(m_ref - m_use) : 1.f;
    const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(-m_safe, -m_safe);
    float2 rs2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
            const float2 x = ffma2(make_float2(s[64 * h + 2 * c2], s[64 * h + 2 * c2 + 1]), sl2, nm2);
            const float2 e = (c2 % kFmaExpEvery == kFmaExpEvery - 1) ? exp2_fma2(x)
                                                                  : make_float2(exp2_approx(x.x), exp2_approx(x.y));
            if (qsc) {
                const float4 vq = reinterpret_cast<const float4*>(qsc + BN)[16 * h + (c2 >> 1)];
                const float2 pv = fmul2(e, (c2 & 1) ? make_float2(vq.z, vq.w) : make_float2(vq.x, vq.y));
                __half2 hh = __floats2half2_rn(pv.x, pv.y);
                pk[c2] = *reinterpret_cast<uint32_t*>(&hh);
                rs2[c2 & 3] = fadd2(rs2[c2 & 3], e);
            } else {
                __nv_bfloat162 hb = __floats2bfloat162_rn(e.x, e.y);
                pk[c2] = *reinterpret_cast<uint32_t*>(&hb);
                rs2[c2 & 3] = fadd2(rs2[c2 & 3], make_float2(bf16_lo(pk[c2]), bf16_hi(pk[c2])));
            }
        }
        tmem_st32(s_addr + 64 + 32 * h, pk);
    }
    const float rs = ((rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y)) + ((rs2[2].x + rs2[2].y) + (rs2[3].x + rs2[3].y));
    l_sum = l_sum * corr + rs;
    m_ref = m_use;
    return corr;
}

// ------------------------------------------------------------------ split records
//
// One row of a split's record of a query tile: its running maximum, row sum
// and unnormalised O row (read from TMEM at o_addr; zeros when the split had
// no tile for it).  Not inlined, like the merge below.
__device__ __noinline__ void write_split_record(float* rec, int row, bool have, float m_ref, float l_sum,
                                                uint32_t o_addr) {
    rec[row] = have ? m_ref : -INFINITY;
    rec[BM + row] = have ? l_sum : 0.f;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        float o[32];
        if (have) {
            tmem_ld32(o_addr + 32 * ch, o);
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.f;
        }
#pragma unroll
        for (int g4 = 0; g4 < 8; ++g4)
            reinterpret_cast<float4*>(rec + 2 * BM)[(8 * ch + g4) * BM + row] =
                make_float4(o[4 * g4], o[4 * g4 + 1], o[4 * g4 + 2], o[4 * g4 + 3]);
    }
}

// ------------------------------------------------------------------ split merge
//
// The split that arrives last merges the ns_use records of one query tile,
// row by row (thread = row): the splits' maxima and sums give each record's
// weight, and the weighted sum of the unnormalised O rows over the total
// weight is the row's output.  Not inlined, so that its registers do not
// count against the softmax loop's: the kernel runs at the 168 a thread
// that ten warps leave (an SM sub-partition holds three of them in its 16K
// registers).
__device__ __noinline__ void merge_split_records(const float* base, int ns_use, int row, bool store,
                                                 __nv_bfloat16* op, int bar_id) {
    constexpr size_t kSplitStride = 2 * (size_t)kPartFloats;
    float w[kMaxSplit];
    float M = -INFINITY, L = 0.f;
#pragma unroll
    for (int sp = 0; sp < kMaxSplit; ++sp)
        if (sp < ns_use) M = fmaxf(M, __ldcg(base + sp * kSplitStride + row));
#pragma unroll
    for (int sp = 0; sp < kMaxSplit; ++sp) {
        w[sp] = 0.f;
        if (sp < ns_use) {
            const float ms = __ldcg(base + sp * kSplitStride + row);
            w[sp] = ms == -INFINITY ? 0.f : exp2f(ms - M);
            L += w[sp] * __ldcg(base + sp * kSplitStride + BM + row);
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll 1
    for (int g8 = 0; g8 < HD / 8; ++g8) {
        float v8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int sp = 0; sp < kMaxSplit; ++sp) {
            if (sp < ns_use) {
                const float4* o4 = reinterpret_cast<const float4*>(base + sp * kSplitStride + 2 * BM);
                const float4 x0 = __ldcg(o4 + (2 * g8) * BM + row);
                const float4 x1 = __ldcg(o4 + (2 * g8 + 1) * BM + row);
                v8[0] += w[sp] * x0.x; v8[1] += w[sp] * x0.y; v8[2] += w[sp] * x0.z; v8[3] += w[sp] * x0.w;
                v8[4] += w[sp] * x1.x; v8[5] += w[sp] * x1.y; v8[6] += w[sp] * x1.z; v8[7] += w[sp] * x1.w;
            }
        }
        if (store) {
#pragma unroll
            for (int e = 0; e < 8; ++e) v8[e] *= inv;
            store_row<__nv_bfloat16, 8>(op + 8 * g8, v8);
        }
    }
    // The records are dead once the warpgroup has read them (only this, the
    // last split of the unit, reads them; every writer took its ticket after
    // a fence): drop their lines from L2 without writing them back, so the
    // splits cost L2 traffic, not DRAM writes.  A record is 520 whole
    // 128-byte lines at a 128-byte-aligned offset of the workspace.
    static_assert(kPartFloats * sizeof(float) % 128 == 0, "records are whole L2 lines");
    constexpr int kLines = (int)(kPartFloats * sizeof(float) / 128);
    asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
    for (int sp = 0; sp < ns_use; ++sp)
        for (int ln = row; ln < kLines; ln += BM)
            asm volatile("discard.global.L2 [%0], 128;" ::"l"(base + sp * kSplitStride + (size_t)ln * 32) : "memory");
}

// ------------------------------------------------------------------ kernel

// EPI: EPI_STORE (pre-fill: store, or key-range split records), EPI_MIX or
// EPI_DOT (the gated mix's epilogues; no key-range splits).  Ten warps leave
// 168 registers a thread (three of them share an SM sub-partition's 16K);
// the split epilogue keeps its indices in shared memory and its record
// write and merge out of line, so that the softmax loop fits without spills.
// QS: the full cache is a quantized layer's staging area -- K codes in bf16,
// V codes times 16 in fp16, both exact -- and tmS its per-row (k scale,
// v scale / 16) pairs, applied in the softmax; the PV MMAs of those tiles
// run in fp16.
template <int EPI, bool QS>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                      const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKx,
                      const __grid_constant__ CUtensorMap tmVx, const __grid_constant__ CUtensorMap tmKr,
                      const __grid_constant__ CUtensorMap tmVr, const __grid_constant__ CUtensorMap tmS,
                      const TcArgs p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const LayerArgs& a = p.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if ((smem_u32(smem) & 1023u) != 0) {   // the swizzled layouts need 1024-byte alignment
        if (tid == 0 && p.status) atomicOr(p.status, DUO_DEV_BAD_LENGTH);
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
    const bool retrieval = (int)blockIdx.x < p.n_ret_ctas;
    int unit = 0, split = 0, m, g, hs, b;
    if (retrieval) {
        // (sequence, KV head) outermost, then the split, then the query tile
        // pair (heaviest first) and the query head of the group: the CTAs
        // that read one KV head's key range run side by side and share its
        // tiles in L2
        const int per_group = p.n_mpairs * a.G;
        const int r = (int)blockIdx.x;
        const int inner = r % per_group;
        split = (r / per_group) % p.ns;
        const int bh = r / (per_group * p.ns);
        g = inner % a.G;
        m = p.n_mpairs - 1 - inner / a.G;
        hs = bh % a.R;
        b = bh / a.R;
        unit = (bh * p.n_mpairs + m) * a.G + g;
    } else {
        int idx = (int)blockIdx.x - p.n_ret_ctas;
        const int per_m = a.B * a.S * a.G;
        m = p.n_mpairs - 1 - idx / per_m;              // heaviest query tiles first
        idx %= per_m;
        g = idx % a.G;
        hs = (idx / a.G) % a.S;
        b = idx / (a.G * a.S);
    }
    const int slot = retrieval ? hs : a.R + hs;
    const int q_idx = a.q_head0[slot] + g;
    const int kv_idx = a.kv_head[slot];
    int c0 = p.seq_len ? p.seq_len[b] : 0;            // no lengths: whole sequences, no cache
    if (c0 < 0) c0 = 0;
    if (retrieval && c0 > a.capacity) {
        if (tid == 0 && m == p.n_mpairs - 1 && p.status) atomicOr(p.status, DUO_DEV_BAD_LENGTH);
        c0 = a.capacity;
    }
    const Sched sc = make_sched(p, retrieval, c0, m);
    // Key-range split of a retrieval unit: split `split` of ns_use takes the
    // unit's tiles [j0, j1); units too short to split run whole, and the CTAs
    // of splits they do not use leave before any set-up.
    int ns_use = 1, j0 = 0, j1 = sc.n;
    if (retrieval && p.ns > 1) {
        ns_use = min(p.ns, max(1, sc.n / kMinSplitTiles));
        if (split >= ns_use) return;
        j0 = split * sc.n / ns_use;
        j1 = (split + 1) * sc.n / ns_use;
    }
    const int nl = j1 - j0;                           // tiles of this CTA for Q1
    const int nl0 = max(0, min(j1, sc.n0) - j0);      // ... and for Q0

    // ------------------------------------------------------- set-up
    if (warp == kMmaWarp) tmem_alloc(holder, kTmemCols);
    if (tid == 0) {
        // what the split epilogue needs, parked here instead of in registers
        // held across the softmax loop
        holder[2] = (uint32_t)unit;
        holder[3] = (uint32_t)split;
        holder[4] = (uint32_t)ns_use;
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
            for (int j = 0; j < nl; ++j) {
                const Tile t = tile_at(sc, j0 + j);
                const int st = j & 1;
                for (int kv = 0; kv < 2; ++kv) {
                    uint64_t* full = kv ? &v_full[st] : &k_full[st];
                    uint64_t* empty = kv ? &v_empty[st] : &k_empty[st];
                    if (j >= 2 && !mbar_wait(empty, ((j >> 1) - 1) & 1, p.status)) goto producer_done;
                    // a quantized prior tile's scales ride with its K tile, into
                    // slot j % 4: the K stage of tile j + 4 is free once QK(j + 2)
                    // is done, which comes after the softmax of tile j + 1
                    const bool scales = QS && kv == 0 && t.src == SRC_CACHE;
                    mbar_arrive_expect_tx(full, kTileBytes + (scales ? kScaleTileBytes : 0u));
                    if (scales)   // x = t.row + the staging shift: a multiple of four floats
                        tma_load_3d(smem_u32(smem + kOffScale) + (j & 3) * kScaleTileBytes, &tmS,
                                    t.row + ((4 - (c0 & 3)) & 3), 0, cache_z, full);
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
            constexpr uint32_t idesc_pv16 = idesc_f16(BM, HD, 0, 1);   // a quantized prior tile: fp16 P and V
            const int n = nl, n0 = nl0;
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
                const uint32_t idesc = QS && tile_at(sc, j0 + j).src == SRC_CACHE ? idesc_pv16 : idesc_pv;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bd = sw128_desc(sV + st * kTileBytes + kk * 2048, kHalfBytes, 1024);
                    tc_mma_ta(tmem + col_o(qi), tmem + col_s(qi) + 64 + 8 * kk, bd, idesc, (j > 0 || kk > 0) ? 1u : 0u);
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
    } else if (warp < kTmaWarp) {
        // --------------------------------------------------- softmax
        const int qi = warp >> 2;                             // query tile of this warpgroup
        const int row = tid & 127;                            // TMEM lane
        const int crow = BM * (2 * m + qi) + row;             // chunk row
        const int P = c0 + crow;                              // absolute query position
        const int n_me = qi ? nl : nl0;
        const float sl = a.scale * kLog2e;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        float m_ref = -INFINITY, l_sum = 0.f;
        bool ok = true;
        for (int j = 0; j < n_me; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[qi], j & 1, p.status));
            if (!ok) break;
            tc_fence_after();
            const Tile t = tile_at(sc, j0 + j);
            const bool masked = needs_mask(sc, t, qi);
            uint32_t vis[4] = {0u, 0u, 0u, 0u};   // the tile's keys this row sees, a bit per column
            if (masked) visible_columns(a, sc, t, P, vis);
            bool need;
            const float* qsc = QS && t.src == SRC_CACHE
                                   ? reinterpret_cast<const float*>(smem + kOffScale + (j & 3) * kScaleTileBytes)
                                   : nullptr;
            const float corr = softmax_tile(lane_base + col_s(qi), sl, masked, vis, m_ref, l_sum, need, qsc);
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
        // epilogue: O / l -> bf16 (or the gated mix's epilogues)
        const size_t row_off = (((size_t)b * p.C + crow) * a.Hq + q_idx) * HD;
        // the output row (and the record of a split) exist: CTA-uniform
        const bool out_ok = bounds_ok(b < a.B && q_idx >= 0 && q_idx < a.Hq, p.status);
        uint4 pre[16];   // EPI_MIX / EPI_DOT: this row of out / dout, loaded before the wait below
        if constexpr (EPI != EPI_STORE) {
            const uint4* src = reinterpret_cast<const uint4*>(
                static_cast<const __nv_bfloat16*>(EPI == EPI_MIX ? p.out : p.epi.dout) + row_off);
#pragma unroll
            for (int i = 0; i < 16; ++i) pre[i] = crow < p.C && out_ok ? src[i] : make_uint4(0u, 0u, 0u, 0u);
        }
        if (ok && n_me >= 1) ok = __all_sync(0xffffffffu, mbar_wait(&o_done[qi], 0, p.status));
        __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.out) + row_off;
        if (!out_ok) {
            // debug build: the check failed, nothing is written
        } else if (EPI != EPI_STORE || holder[4] == 1u) {
            if (ok && n_me >= 1) {
                tc_fence_after();
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                const float al = EPI == EPI_MIX ? p.epi.alpha[kv_idx] : 0.f;
                float dot = 0.f;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    float o[32];
                    tmem_ld32(lane_base + col_o(qi) + 32 * ch, o);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v8[e] = o[8 * q4 + e] * inv;
                        if constexpr (EPI == EPI_STORE) {
                            if (crow < p.C) store_row<__nv_bfloat16, 8>(op + 32 * ch + 8 * q4, v8);
                        } else {
                            const uint4 u = pre[4 * ch + q4];
                            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                            if constexpr (EPI == EPI_MIX) {
                                // out held the streaming attention: mix it in
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    v8[2 * e] = al * v8[2 * e] + (1.f - al) * bf16_lo(w[e]);
                                    v8[2 * e + 1] = al * v8[2 * e + 1] + (1.f - al) * bf16_hi(w[e]);
                                }
                                if (crow < p.C) store_row<__nv_bfloat16, 8>(op + 32 * ch + 8 * q4, v8);
                            } else {
                                // <dout row, attention row>; rows past the sequence hold dout = 0
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    dot = fmaf(v8[2 * e], bf16_lo(w[e]), fmaf(v8[2 * e + 1], bf16_hi(w[e]), dot));
                            }
                        }
                    }
                }
                if constexpr (EPI == EPI_DOT) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                    if (lane == 0) atomicAdd(&p.epi.dalpha[kv_idx], p.epi.sign * dot);
                }
            }
        } else if (EPI == EPI_STORE &&
                   bounds_ok((int)holder[2] < p.n_units && (int)holder[3] < p.ns && (int)holder[4] <= p.ns, p.status)) {
            // (1) this split's record of the query tile: m, l and O unnormalised
            const bool have = ok && n_me >= 1;               // warp-uniform
            const int unit_ = (int)holder[2], split_ = (int)holder[3], ns_use_ = (int)holder[4];
            float* rec = p.part + (((size_t)unit_ * p.ns + split_) * 2 + qi) * kPartFloats;
            if (have) tc_fence_after();
            write_split_record(rec, row, have, m_ref, l_sum, lane_base + col_o(qi));
            // (2) a ticket per unit, taken once the 256 softmax threads have
            // written; the CTA that arrives last merges (no CTA ever waits)
            __threadfence();
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (tid == 0) holder[1] = (atomicAdd(&p.ticket[unit_], 1u) == (unsigned)ns_use_ - 1) ? 1u : 0u;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (holder[1]) {
                __threadfence();
                merge_split_records(p.part + (size_t)unit_ * p.ns * 2 * kPartFloats + (size_t)qi * kPartFloats,
                                    ns_use_, row, crow < p.C, op, 2 + qi);
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

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        return 148;
    return n;
}

// Key-range splits per retrieval unit for a chunk of C queries.  One CTA fills
// an SM, so n_units CTAs run in ceil(n_units / n_sms) waves and the last one
// may leave SMs idle (256 units on 148 SMs: 1.73 waves, 13.5 % of SM time).
// Splitting every unit's key tiles ns ways makes n_units * ns CTAs of about
// equal work: take the smallest ns whose waves are at least 95 % full (else
// the fullest).  The device then uses fewer splits for units shorter than
// kMinSplitTiles tiles per split (early chunks of a prompt).
PrefillPlan prefill_plan(const LayerArgs& a, int C, int n_sms) {
    PrefillPlan pl{};
    pl.ns = 1;
    const long units = (long)a.B * a.R * a.G * ((C + 2 * BM - 1) / (2 * BM));
    if (units > 0 && n_sms > 0) {
        double best = 0.0;
        for (int ns = 1; ns <= kMaxSplit; ++ns) {
            const long items = units * ns;
            const long waves = (items + n_sms - 1) / n_sms;
            const double fill = (double)items / ((double)waves * n_sms);
            if (fill > best + 1e-9) {
                best = fill;
                pl.ns = ns;
            }
            if (fill >= 0.95) break;
        }
    }
    if (pl.ns > 1) {
        const size_t part = (size_t)units * pl.ns * 2 * kPartFloats * sizeof(float);
        pl.ticket_offset = (part + 255) / 256 * 256;
        pl.bytes = pl.ticket_offset + ((size_t)units * sizeof(uint32_t) + 255) / 256 * 256;
    } else {
        pl.ticket_offset = 0;
        pl.bytes = 256;
    }
    return pl;
}

size_t prefill_workspace_bytes(const LayerArgs& a, int max_chunk) {
    // the plan depends on the number of 256-query tile pairs; a workspace
    // sized here serves every chunk length up to max_chunk
    const int n_sms = sm_count();
    size_t bytes = 256;
    for (int mp = 1; mp <= (max_chunk + 2 * BM - 1) / (2 * BM); ++mp) {
        const size_t b = prefill_plan(a, mp * 2 * BM, n_sms).bytes;
        if (b > bytes) bytes = b;
    }
    return bytes;
}

cudaError_t launch_prefill_tc(const LayerArgs& a, const CacheArgs& c, const void* q, const void* k_chunk,
                              const void* v_chunk, int C, void* out, void* workspace, size_t ws_bytes,
                              cudaStream_t s, const EpiArgs* epi, const float* qscale) {
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
    if (a.R > 0 && c.k_full != nullptr) {
        const uint64_t d[3] = {HD, (uint64_t)a.capacity, (uint64_t)a.B * a.R};
        const uint64_t st[2] = {row, row * a.capacity};
        if (!encode_tmap_bf16(&mKc, c.k_full, 3, d, st, bx3) || !encode_tmap_bf16(&mVc, c.v_full, 3, d, st, bx3))
            return cudaErrorInvalidValue;
    } else {
        mKc = mKx;  // never read: no retrieval heads, or no cache (c0 = 0)
        mVc = mVx;
    }
    if (a.S > 0 && c.k_ring != nullptr) {
        const uint64_t d[3] = {HD, (uint64_t)a.W, (uint64_t)a.B * a.S};
        const uint64_t st[2] = {row, row * a.W};
        if (!encode_tmap_bf16(&mKr, c.k_ring, 3, d, st, bx3) || !encode_tmap_bf16(&mVr, c.v_ring, 3, d, st, bx3))
            return cudaErrorInvalidValue;
    } else {
        mKr = mKx;  // never read: no streaming heads, or no cache (c0 = 0)
        mVr = mVx;
    }
    CUtensorMap mS = mKx;   // never read unless the cache holds codes
    if (qscale != nullptr) {
        // [B * R][2][capacity + 4] fp32: per head a row of k scales and a row
        // of v scales / 16, shifted by the staging so that every prior tile
        // starts on a multiple of four floats; a box is a tile's 128 scales of
        // both rows
        const uint64_t d[3] = {(uint64_t)a.capacity + 4, 2, (uint64_t)a.B * a.R};
        const uint64_t st[2] = {4ull * (a.capacity + 4), 8ull * (a.capacity + 4)};
        const uint32_t bx[3] = {BN, 2, 1};
        if (!encode_tmap(&mS, qscale, 3, d, st, bx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 0)) return cudaErrorInvalidValue;
    }
    TcArgs p;
    p.a = a;
    p.C = C;
    p.n_mpairs = (C + 2 * BM - 1) / (2 * BM);
    p.n_units = a.B * a.R * a.G * p.n_mpairs;
    const PrefillPlan plan = prefill_plan(a, C, sm_count());
    const int mode = epi ? epi->mode : EPI_STORE;
    const bool split = plan.ns > 1 && workspace != nullptr && ws_bytes >= plan.bytes && mode == EPI_STORE;
    p.ns = split ? plan.ns : 1;
    p.part = split ? static_cast<float*>(workspace) : nullptr;
    p.ticket = split ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + plan.ticket_offset) : nullptr;
    p.n_ret_ctas = p.n_units * p.ns;
    p.seq_len = c.seq_len;
    p.status = c.status;
    p.out = out;
    p.epi = epi ? *epi : EpiArgs{EPI_STORE, nullptr, nullptr, nullptr, 0.f};
    const long grid = (long)p.n_ret_ctas + (long)a.B * a.S * a.G * p.n_mpairs;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffffL) return cudaErrorInvalidConfiguration;
    static std::atomic<unsigned long long> configured[4] = {{0}, {0}, {0}, {0}};
    const bool qs = qscale != nullptr;
    if (qs && mode != EPI_STORE) return cudaErrorInvalidValue;
    {
        cudaError_t e = cudaErrorInvalidValue;
        constexpr int kS = (int)(kSmemBytes + 1024);
        if (mode == EPI_STORE && !qs) e = smem_limit_once(prefill_tc_kernel<EPI_STORE, false>, kS, configured[0]);
        if (mode == EPI_STORE && qs) e = smem_limit_once(prefill_tc_kernel<EPI_STORE, true>, kS, configured[3]);
        if (mode == EPI_MIX) e = smem_limit_once(prefill_tc_kernel<EPI_MIX, false>, kS, configured[1]);
        if (mode == EPI_DOT) e = smem_limit_once(prefill_tc_kernel<EPI_DOT, false>, kS, configured[2]);
        if (e != cudaSuccess) return e;
    }
    if (split) {
        // the ticket words sit after this chunk length's partial records, so
        // a call with another chunk length may find there what an earlier
        // call's records left: clear them first
        const cudaError_t e = cudaMemsetAsync(p.ticket, 0, (size_t)p.n_units * sizeof(uint32_t), s);
        if (e != cudaSuccess) return e;
    }
    const unsigned g = (unsigned)grid;
    constexpr size_t kS = kSmemBytes + 1024;
    if (mode == EPI_MIX)
        prefill_tc_kernel<EPI_MIX, false><<<g, kThreads, kS, s>>>(mQ, mKc, mVc, mKx, mVx, mKr, mVr, mS, p);
    else if (mode == EPI_DOT)
        prefill_tc_kernel<EPI_DOT, false><<<g, kThreads, kS, s>>>(mQ, mKc, mVc, mKx, mVx, mKr, mVr, mS, p);
    else if (qs)
        prefill_tc_kernel<EPI_STORE, true><<<g, kThreads, kS, s>>>(mQ, mKc, mVc, mKx, mVx, mKr, mVr, mS, p);
    else
        prefill_tc_kernel<EPI_STORE, false><<<g, kThreads, kS, s>>>(mQ, mKc, mVc, mKx, mVx, mKr, mVr, mS, p);
    return cudaGetLastError();
}

namespace {

__global__ void exp2_fma_probe_kernel(const float* x, float* y, int64_t n) {
    for (int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < n;
         i += 2 * (int64_t)gridDim.x * blockDim.x) {
        const float x1 = i + 1 < n ? x[i + 1] : 0.f;
        const float2 e = exp2_fma2(make_float2(x[i], x1));
        y[i] = e.x;
        if (i + 1 < n) y[i + 1] = e.y;
    }
}

}  // namespace

cudaError_t launch_exp2_fma_probe(const float* x, float* y, int64_t n, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int64_t pairs = (n + 1) / 2;
    const int grid = (int)(pairs < 148 * 8 * 256 ? (pairs + 255) / 256 : 148 * 8);
    exp2_fma_probe_kernel<<<grid, 256, 0, s>>>(x, y, n);
    return cudaGetLastError();
}

}  // namespace duo
