/*
 * duo.h -- C ABI of libduo.so: head-split (retrieval / streaming) attention
 * for DuoAttention on NVIDIA B200 (sm_100a).
 *
 * The method (sources cited by page title and section):
 *   [Review]  "DuoAttention: Efficient Long-Context LLM Inference with
 *             Retrieval and Streaming Heads", paper review, xllm-io.github.io,
 *             S3 "Core formula", "Retrieval-head identification",
 *             "Inference flow", "Deployment optimisation"; S5 "Ablations".
 *   [Summary] paperlayer.ai summary of arXiv:2410.10819v1, S2 bullets
 *             "Optimization-based Identification", "Binarizing Attention
 *             Implementations", "Chunked Pre-filling".
 *
 * Retrieval heads attend causally over a full KV cache that grows with the
 * context; streaming heads keep only the first `sink` tokens and the last
 * `recent` tokens (the Lambda-shaped mask) in a constant-size cache.
 *
 * Conventions shared by every entry point
 *   - Every tensor argument is a device pointer owned by the caller, except
 *     where a comment says "host".  Except for duo_check_status, the library
 *     never allocates, frees or synchronises; work is queued on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream).
 *   - Layouts are dense row-major with the head dimension innermost
 *     (contiguous).  Pointers must be 16-byte aligned.
 *   - Element type is bf16 (bit patterns, 2 bytes) or fp32, as
 *     duo_layer_desc.dtype says; every tensor of a call has that type.
 *     Accumulation is always fp32; bf16 results are rounded to nearest even
 *     once, at the final store.
 *   - Head order: with io_order = DUO_ORDER_MODEL, q / k / v / out use the
 *     model's head order and the kernels gather and scatter through kv_perm
 *     (the concatenation back into model order [Review S3 "Inference flow"]
 *     is the address of the final store).  With DUO_ORDER_BLOCK they are
 *     already in [retrieval | streaming] block order, as after reordering
 *     the projection weights [Review S3 "Deployment optimisation"].
 *     Query head h of the model belongs to KV head h / G, G = n_q_heads /
 *     n_kv_heads [Summary S2 "Optimization-based Identification"].
 *   - Return value: DUO_OK, or an error code with a message available from
 *     duo_last_error() (thread-local).  Argument checks run on the host
 *     before anything is queued; on an error nothing is queued.  Conditions
 *     only the device can see (a full cache, a bad page id, a wait that ran
 *     out) set bits in the state's device status word and skip the access;
 *     they never trap.  duo_check_status() reads that word back.
 */
#ifndef DUO_H
#define DUO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* duo_stream_t; /* = cudaStream_t */

typedef enum {
    DUO_OK = 0,
    DUO_ERR_INVALID_ARG = 1, /* null pointer, bad enum, bad permutation     */
    DUO_ERR_SHAPE = 2,       /* inconsistent sizes                          */
    DUO_ERR_DTYPE = 3,       /* unknown element type                        */
    DUO_ERR_CAPACITY = 4,    /* workspace or cache too small                */
    DUO_ERR_UNSUPPORTED = 5, /* valid, but not built (e.g. head_dim 96)     */
    DUO_ERR_CUDA = 6,        /* a CUDA runtime call failed                  */
    DUO_ERR_DEVICE = 7       /* duo_check_status found device status bits  */
} duo_status;

/* element types */
enum { DUO_BF16 = 0, DUO_FP32 = 1 };
/* head order of q / k / v / out */
enum { DUO_ORDER_MODEL = 0, DUO_ORDER_BLOCK = 1 };
/* storage of the retrieval heads' full cache */
enum {
    DUO_KV_PLAIN = 0, /* the layer's dtype, as the activations               */
    DUO_KV_INT8 = 1,  /* 8-bit codes + one fp32 scale per row (see duo_kv_state) */
    DUO_KV_INT4 = 2   /* 4-bit codes + one fp32 scale per row (see duo_kv_state) */
};
/* what a streaming head sees in duo_prefill_chunk (decode is the same for both) */
enum {
    DUO_STREAM_LAMBDA = 0, /* the Lambda mask per query: sinks + its last `recent` tokens */
    DUO_STREAM_CHUNK = 1   /* sinks + the `recent` tokens before the chunk + the whole chunk up to itself */
};
/* duo_permute_heads directions */
enum { DUO_MODEL_TO_BLOCK = 0, DUO_BLOCK_TO_MODEL = 1 };
/* workspace queries */
enum { DUO_OP_DECODE = 0, DUO_OP_PREFILL = 1 };
/* device status bits (OR-ed into duo_kv_state.status) */
enum {
    DUO_DEV_FULL_CACHE_OVERFLOW = 1, /* append past capacity: row not written */
    DUO_DEV_BAD_PAGE = 2,            /* page table entry missing / out of pool */
    DUO_DEV_WAIT_TIMEOUT = 4,        /* a bounded device wait ran out          */
    DUO_DEV_BAD_LENGTH = 8,          /* a sequence length outside [0, capacity] */
    DUO_DEV_BOUNDS = 16              /* debug build only (libduo_debug.so, built with
                                        DUO_DEBUG_BOUNDS): an index check failed and
                                        the access it guarded was skipped           */
};

#define DUO_MAX_KV_HEADS 64
#define DUO_STATE_COUNTER_WORDS 4

/* One attention layer.  Fill it with duo_desc_init(). */
typedef struct {
    int32_t batch;        /* B: sequences                                     */
    int32_t n_q_heads;    /* Hq                                               */
    int32_t n_kv_heads;   /* Hkv (Hq % Hkv == 0)                              */
    int32_t head_dim;     /* d: 64 or 128                                     */
    int32_t sink;         /* attention-sink tokens of streaming heads (16)    */
    int32_t recent;       /* recent tokens of streaming heads (64)            */
    int32_t dtype;        /* DUO_BF16 or DUO_FP32                             */
    int32_t page_size;    /* 0: contiguous full cache; 64: paged full cache   */
    float scale;          /* softmax scale; 1/sqrt(d) when <= 0               */
    int32_t n_retrieval;  /* R: retrieval KV heads (block slots 0..R-1)       */
    int32_t io_order;     /* DUO_ORDER_MODEL or DUO_ORDER_BLOCK               */
    int32_t stream_prefill; /* DUO_STREAM_LAMBDA (default) or DUO_STREAM_CHUNK */
    int32_t kv_quant;     /* DUO_KV_PLAIN (default), DUO_KV_INT8 or DUO_KV_INT4 (bf16, d 128, contiguous, sink + recent <= 128) */
    int32_t kv_perm[DUO_MAX_KV_HEADS]; /* block slot i holds model KV head kv_perm[i] */
} duo_layer_desc;

/*
 * The two caches of one layer, all caller-owned device memory.
 *   R = n_retrieval, S = n_kv_heads - R, W = sink + recent.
 *
 * Full cache (retrieval heads) [Review S3 "Inference flow"]:
 *   contiguous (page_size 0): k_full, v_full = [B][R][capacity][d];
 *     token p of sequence b, retrieval slot r is row (b*R + r)*capacity + p.
 *   paged (page_size 64): k_full, v_full = [n_pages][R][64][d]; token p of
 *     sequence b lives in page page_table[b*max_pages + p/64], row p%64.
 *     capacity = max_pages * 64.
 * Streaming ring (streaming heads) [Review S3 "Inference flow"]:
 *   k_ring, v_ring = [B][S][W][d]; position p lives in slot p if p < sink,
 *   else in slot sink + (p - sink) % recent, evicting the token `recent`
 *   positions older.  ring_pos = [B][W] int32, the position held by each
 *   slot (-1 = empty); all streaming heads of a sequence share it.
 * 8-bit full cache (desc->kv_quant = DUO_KV_INT8; bf16 activations, d = 128,
 *   contiguous, capacity a multiple of 64) -- the pages pair the method with a
 *   quantized KV cache [Review S5 "Decoding performance"] without a scheme;
 *   this one is per row and symmetric: amax = max |x| over the row's d
 *   values, code = x * (127 / amax) rounded to nearest even, scale =
 *   amax / 127, each an fp32 operation (a zero row: scale 0, codes 0);
 *   attention reads code * scale:
 *   k_full = int8 [B][R][capacity][d] codes, row per token as above;
 *   v_full = int8 [B][R][capacity/64][d][64]: per 64-token tile the codes
 *     transposed (a row of 64 bytes per feature), the 16 tokens of each
 *     16-token group stored in the order 0 1 8 9 2 3 10 11 4 5 12 13 6 7 14 15;
 *   k_scale, v_scale = fp32 [B][R][capacity].
 *   K and V values must stay within +-8.3e6 (the fp16 operands of the
 *   decode MMAs hold code * 1 and p * scale).
 * 4-bit full cache (desc->kv_quant = DUO_KV_INT4; the same constraints) --
 *   the paper review's "Quantization combination" pairs 8-bit weights with a
 *   4-bit KV cache, again without a scheme; this one is the 8-bit scheme with
 *   7 levels a side: scale = amax / 7, code = x * (7 / amax) rounded to
 *   nearest even (-7..7), stored as the nibble code + 8:
 *   k_full = [B][R][capacity][64] bytes, a row per token; byte 16q + 4j + c
 *     of a row holds, with e = 32q + 8j, the features (e, e+2), (e+4, e+6),
 *     (e+1, e+3), (e+5, e+7) for c = 0, 1, 2, 3 (first in the low nibble);
 *   v_full = [B][R][capacity/64][4096] bytes: per 64-token tile, 16-token
 *     group g, feature block m, row r (0..7) and key quad k (0..3) a word at
 *     1024g + 128m + 16r + 4k whose bytes are the group's tokens 2k, 2k+8,
 *     2k+1, 2k+9, each holding features 16m + r (low) and 16m + 8 + r (high);
 *   k_scale, v_scale as for the 8-bit cache.
 * seq_len = [B] int32: tokens appended so far per sequence.
 * counters = DUO_STATE_COUNTER_WORDS uint32 words that must be zero before
 *   the first call; every call leaves them zero.
 * status = one int32 word of DUO_DEV_* bits; the library only ORs into it.
 * Initial values: ring_pos all -1, seq_len 0, status 0 (or a state built by
 *   the caller that keeps these invariants).
 */
typedef struct {
    void* k_full;
    void* v_full;
    int32_t* page_table; /* paged only, else NULL                    */
    int32_t capacity;    /* tokens per sequence in the full cache    */
    int32_t max_pages;   /* paged: columns of page_table             */
    int32_t n_pages;     /* paged: pages in the pool                 */
    int32_t reserved0;
    void* k_ring;
    void* v_ring;
    int32_t* ring_pos;
    int32_t* seq_len;
    uint32_t* counters;
    int32_t* status;
    float* k_scale;      /* 8-bit full cache only, else NULL         */
    float* v_scale;
} duo_kv_state;

/* ------------------------------------------------------------------------ */
/* Library information                                                      */
/* ------------------------------------------------------------------------ */

/* Message of the last error on this thread ("" after success). */
const char* duo_last_error(void);
/* Name of a status code. */
const char* duo_status_string(duo_status s);
/* ABI version: 4 (duo_gated_mix and duo_gated_mix_grad_alpha take a device
 * status word; version 3 added stream_prefill, kv_quant and the 8-bit
 * cache's scales). */
int32_t duo_abi_version(void);

/* ------------------------------------------------------------------------ */
/* Set-up (host only)                                                       */
/* ------------------------------------------------------------------------ */

/*
 * duo_partition_heads -- gate binarisation and head partition.
 * [Review S3 "Retrieval-head identification": alpha = 1[alpha >= tau];
 *  Summary S2 "Binarizing Attention Implementations": tau is a sparsity
 *  quantile; Review S3 "Deployment optimisation": heads are regrouped into a
 *  contiguous retrieval block and a streaming block.]
 *
 * alpha        host float[n_kv_heads], the optimised gate of each KV head.
 * tau          threshold, used when target_n_retrieval < 0: gate = alpha >= tau.
 * target_n_retrieval  >= 0: keep exactly that many heads, those with the
 *              largest alpha, ties going to the lower head index (the
 *              quantile threshold).
 * gate         host uint8[n_kv_heads] out: 1 = retrieval head.
 * kv_perm      host int32[n_kv_heads] out: block slot i holds model head
 *              kv_perm[i]; retrieval heads first, each block ascending.
 * kv_inv_perm  host int32[n_kv_heads] out: kv_inv_perm[kv_perm[i]] = i.
 * n_retrieval  host int32 out.
 * Errors: DUO_ERR_INVALID_ARG (null, n_kv_heads outside 1..DUO_MAX_KV_HEADS,
 * NaN alpha), DUO_ERR_SHAPE (target above n_kv_heads).
 */
duo_status duo_partition_heads(const float* alpha, int32_t n_kv_heads, float tau,
                               int32_t target_n_retrieval, uint8_t* gate, int32_t* kv_perm,
                               int32_t* kv_inv_perm, int32_t* n_retrieval);

/*
 * duo_desc_init -- fill a layer descriptor with the deployment defaults
 * (sink 16, recent 64 [Review S5 "Ablations" item 3], scale 1/sqrt(d),
 * contiguous full cache, model head order) and the given partition.
 * kv_perm: host int32[n_kv_heads] from duo_partition_heads.
 * Errors: DUO_ERR_INVALID_ARG / DUO_ERR_SHAPE / DUO_ERR_DTYPE /
 * DUO_ERR_UNSUPPORTED for values the kernels do not take.
 */
duo_status duo_desc_init(duo_layer_desc* desc, int32_t batch, int32_t n_q_heads,
                         int32_t n_kv_heads, int32_t head_dim, int32_t dtype,
                         const int32_t* kv_perm, int32_t n_retrieval);

/* Checks a filled descriptor the way every entry point does. */
duo_status duo_desc_validate(const duo_layer_desc* desc);

/*
 * duo_workspace_bytes -- device workspace needed by duo_decode_attn
 * (op DUO_OP_DECODE) or duo_prefill_chunk (op DUO_OP_PREFILL, max_tokens =
 * largest chunk).  The workspace holds split-K partial results and ticket
 * words.  A decode workspace must be zero-filled once before its first use
 * (every call leaves the ticket words zero again); a pre-fill workspace needs
 * no initialisation (each call clears the ticket words it uses).  Returns 0
 * for an invalid descriptor.
 */
size_t duo_workspace_bytes(const duo_layer_desc* desc, int32_t op, int32_t max_tokens);

/*
 * duo_prefill_workspace_bytes -- the workspace duo_prefill_chunk takes for
 * chunks of up to max_chunk tokens on this layer and state: what
 * duo_workspace_bytes(desc, DUO_OP_PREFILL, max_chunk) gives, plus, for an
 * 8- or 4-bit full cache, the staging area of its cached rows
 * (B * R * capacity * 528 bytes, which depends on the state's capacity).  st: host pointer to the state (only its sizes are read).
 * Returns 0 for an invalid descriptor or state.
 */
size_t duo_prefill_workspace_bytes(const duo_layer_desc* desc, const duo_kv_state* st, int32_t max_chunk);

/* ------------------------------------------------------------------------ */
/* Device entry points                                                      */
/* ------------------------------------------------------------------------ */

/*
 * duo_permute_heads -- physical reorder of head blocks between model order
 * and [retrieval | streaming] block order [Review S3 "Deployment
 * optimisation"].  Works for activations and for projection weights alike.
 *
 * x, y        [rows][n_kv_heads * heads_per_kv][head_elems] of elem_bytes
 *             each (1, 2, 4 or 8); x and y must not overlap.
 * direction   DUO_MODEL_TO_BLOCK: y[.., i*hpk + g, ..] = x[.., kv_perm[i]*hpk + g, ..]
 *             DUO_BLOCK_TO_MODEL: the inverse.
 * Errors: DUO_ERR_INVALID_ARG, DUO_ERR_SHAPE, DUO_ERR_CUDA.
 */
duo_status duo_permute_heads(const duo_layer_desc* desc, const void* x, void* y, int64_t rows,
                             int32_t heads_per_kv, int64_t head_elems, int32_t elem_bytes,
                             int32_t direction, duo_stream_t stream);

/*
 * duo_append_kv -- add T tokens per sequence to the two caches.
 * [Review S3 "Inference flow": each layer keeps a full cache for retrieval
 *  heads and a sink + recent cache for streaming heads; Summary S2
 *  "Chunked Pre-filling": pre-fill fills both caches.]
 *
 * k_new, v_new [B][T][Hkv][d], head order per desc->io_order.  Token t of
 * sequence b gets position p = seq_len[b] + t.  Retrieval heads: written to
 * the full cache at p.  Streaming heads: written to the ring only if
 * p < sink or p >= seq_len[b] + T - recent (the tokens that survive), and
 * ring_pos is updated.  seq_len[b] += T once every row is written.
 * With an 8-bit full cache the retrieval rows are quantized on the way in
 * (codes and scale as duo_kv_state describes).
 * T == 0 is a no-op.  A row past capacity (or with no page) is not written
 * and sets DUO_DEV_FULL_CACHE_OVERFLOW (DUO_DEV_BAD_PAGE).
 * Errors: DUO_ERR_INVALID_ARG, DUO_ERR_SHAPE, DUO_ERR_CUDA.
 */
duo_status duo_append_kv(const duo_layer_desc* desc, const duo_kv_state* st, const void* k_new,
                         const void* v_new, int32_t T, duo_stream_t stream);

/*
 * duo_decode_attn -- attention of one new token per sequence, both head
 * types in one launch [Review S3 "Inference flow", decode: Q/K/V are split
 * along the head dimension, each part attends against its own cache, and the
 * results are concatenated before the output projection].
 *
 * Call after duo_append_kv of the token (the token attends to itself).
 * q   [B][Hq][d]; out [B][Hq][d]; head order per desc->io_order.
 * Retrieval heads: out = softmax(scale q K^T) V over cache rows
 * 0..seq_len[b]-1, split-K across CTAs with a last-CTA combine.  Streaming
 * heads: the same over the min(seq_len[b], W) ring slots.  The G query heads
 * of a KV head share every K/V tile.  With an 8-bit full cache the scores
 * are q . codes * k_scale and the values code * v_scale, the scales applied
 * per key to the scores and to p (half the bytes per cached token).
 * workspace: >= duo_workspace_bytes(desc, DUO_OP_DECODE, 0) bytes, zeroed once.
 * Concurrent calls must not share a workspace.
 * Launch overlap: the bf16 / d 128 decode is launched with programmatic
 * dependent launch, so it can start while the kernel before it on the stream
 * finishes, and with a contiguous full cache it loads its first cache tiles
 * that lie at least 128 rows below seq_len before waiting for that kernel
 * (the 8- and 4-bit decodes only ask L2 for their first tiles then: a hint,
 * whatever the rows hold).
 * Every other kernel of the library lets dependents start only when it
 * completes, and the decode kernels write nothing there, so library calls
 * need no care; a caller kernel launched just before it on the same stream
 * that triggers programmatic launch completion early must not write those
 * rows, nor lower seq_len, before it completes.
 * Errors: DUO_ERR_INVALID_ARG, DUO_ERR_SHAPE, DUO_ERR_CAPACITY (workspace),
 * DUO_ERR_UNSUPPORTED, DUO_ERR_CUDA.
 */
duo_status duo_decode_attn(const duo_layer_desc* desc, const duo_kv_state* st, const void* q,
                           void* out, void* workspace, size_t ws_bytes, duo_stream_t stream);

/*
 * duo_decode_step -- duo_append_kv (T = 1) followed by duo_decode_attn, in one
 * launch [Review S3 "Inference flow", decode: both caches take the new token,
 * then each part of the head split attends against its own cache].
 *
 * k_new, v_new [B][Hkv][d] (the new token's K/V, head order per io_order);
 * q, out, workspace as for duo_decode_attn.  Results, caches, ring_pos and
 * seq_len end exactly as after the two separate calls: the CTA whose rows
 * include the new position reads the token from k_new / v_new and stores it
 * into the full cache or the ring, and the last CTA of the launch advances
 * seq_len.  Uses state counter word 1.
 * Errors: as duo_decode_attn.
 */
duo_status duo_decode_step(const duo_layer_desc* desc, const duo_kv_state* st, const void* q, const void* k_new,
                           const void* v_new, void* out, void* workspace, size_t ws_bytes, duo_stream_t stream);

/*
 * duo_prefill_chunk -- attention of a chunk of C prompt tokens per sequence
 * [Summary S2 "Chunked Pre-filling"; Review S3 "Inference flow", pre-fill:
 *  retrieval heads use full causal attention, streaming heads need linear
 *  time and constant memory].
 *
 * Call BEFORE duo_append_kv of the same chunk: the caches hold tokens
 * 0..seq_len[b]-1 and the chunk's own keys come from k_chunk / v_chunk.
 * q [B][C][Hq][d]; k_chunk, v_chunk [B][C][Hkv][d]; out [B][C][Hq][d].
 * Query c of the chunk has position P = seq_len[b] + c; c0 = seq_len[b].
 *   Retrieval head: keys 0..P (causal), prior ones from the full cache.
 *   Streaming head, desc->stream_prefill = DUO_STREAM_LAMBDA: keys j <= P
 *     with j < sink or P - j < recent (Lambda), prior ones from the ring.
 *   Streaming head, DUO_STREAM_CHUNK: keys j <= P with j < sink or
 *     j >= c0 - recent -- the ring as it stood before the chunk and the whole
 *     chunk up to the query (the reading under which pre-fill gains grow as
 *     the chunk shrinks [Review S5 "Pre-filling performance"]); the first
 *     chunk of a prompt is then causal for every head.
 * bf16 with d = 128 runs on the tcgen05 tensor cores (TMA-fed tiles, TMEM
 * accumulators); fp32 and d = 64 run on the CUDA cores.
 * workspace: duo_workspace_bytes(desc, DUO_OP_PREFILL, C) bytes (no
 *   initialisation needed: each call clears the ticket words it uses), or
 *   NULL / smaller.  With it, the bf16 path splits the key tiles of long
 *   retrieval query tiles across several CTAs so that the chunk's CTAs fill
 *   whole waves of SMs; the splits' partial (max, sum, unnormalised output)
 *   rows go to the workspace and the split that finishes last merges them.
 *   Without it the kernel runs unsplit (same results up to rounding).
 *   Concurrent calls must not share a workspace.
 * The full cache must be contiguous (page_size 0).  With an 8- or 4-bit
 * full cache the call first stages the cached rows below seq_len at the
 * start of the workspace -- the K codes as bf16 values, the V codes times
 * 16 as fp16 values (both exact), and each row's k and v scales -- and the
 * pre-fill reads its prior tiles from there, multiplying each score by its
 * key's k scale and each p by its v scale (so code * scale is never rounded
 * to bf16); for those tiles p * v_scale / 16 is the fp16 operand of the PV
 * product (rounded at 2^-11 of its value), which holds v scales up to 4095
 * (|V| up to 520,000 for 8-bit codes, 28,000 for 4-bit); the workspace is
 * then required: duo_prefill_workspace_bytes(desc, st, C) bytes (the staging
 * area -- 512 bytes of codes per token of the capacity and retrieval head
 * and two rows of capacity + 4 fp32 scales per retrieval head -- then the
 * split records; DUO_ERR_CAPACITY when it is missing or smaller than the
 * staging area).
 * Errors: DUO_ERR_INVALID_ARG, DUO_ERR_SHAPE, DUO_ERR_CAPACITY,
 * DUO_ERR_UNSUPPORTED, DUO_ERR_CUDA.
 */
duo_status duo_prefill_chunk(const duo_layer_desc* desc, const duo_kv_state* st, const void* q,
                             const void* k_chunk, const void* v_chunk, int32_t C, void* out,
                             void* workspace, size_t ws_bytes, duo_stream_t stream);

/*
 * duo_gated_mix -- the head-identification forward over whole sequences, no
 * cache: attn = alpha * full_attn + (1 - alpha) * streaming_attn per head,
 * with full_attn = softmax(Q K^T (.) M_causal) V and streaming_attn the same
 * under the Lambda mask [Review S3 "Core formula"], one continuous alpha per
 * KV head shared by its query heads [Summary S2 "Optimization-based
 * Identification"].
 *
 * alpha [Hkv] fp32 device, in model KV head order.
 * q [B][N][Hq][d]; k, v [B][N][Hkv][d]; out [B][N][Hq][d]; model head order
 * (kv_perm and io_order are not used).  bf16 with d = 128 runs on the tcgen05
 * tensor cores in two launches (the streaming attention written to out, then
 * the causal attention mixed with it as it is stored), so out must not alias
 * q, k or v; other dtypes and head sizes run on the CUDA cores, one pass over
 * Q K^T feeding both softmax states.
 * status: one int32 device word (required), caller-owned; the call only ORs
 *   DUO_DEV_* bits into it.  A bounded device wait that runs out sets
 *   DUO_DEV_WAIT_TIMEOUT there and the rows it guarded are not written, so a
 *   caller that reads the word back after the call (zeroed before it) knows
 *   whether out is complete.  The call itself does not read it back.
 * Errors: DUO_ERR_INVALID_ARG, DUO_ERR_SHAPE, DUO_ERR_UNSUPPORTED, DUO_ERR_CUDA.
 */
duo_status duo_gated_mix(const duo_layer_desc* desc, const float* alpha, const void* q,
                         const void* k, const void* v, int32_t N, void* out, int32_t* status,
                         duo_stream_t stream);

/*
 * duo_decode_attn_noalloc -- duo_decode_attn without a caller workspace.
 * (No counterpart on the pages: this is a deployment convenience.)
 *
 * Some callers cannot hand the library device memory for scratch: a plugin
 * running inside a host engine whose allocator owns every byte of HBM, a
 * thin C binding with no device-memory management of its own, or a decode
 * loop that must never call cudaMalloc / cudaFree because those calls can
 * synchronise the whole device.  This entry point computes exactly what
 * duo_decode_attn computes (same kernel, same split plan), but keeps the
 * split-K partial results and ticket words in a statically sized array that
 * is part of the library image; it calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 * q, out, desc and st are as for duo_decode_attn; there is no workspace.
 * Scratch limit: DUO_NOALLOC_SCRATCH_BYTES (2 MiB), i.e. duo_workspace_bytes(
 * desc, DUO_OP_DECODE, st->capacity) must not exceed it; larger layers get
 * DUO_ERR_CAPACITY with the two sizes in the message (use duo_decode_attn).
 * Every GPU that loads the library holds the array until the process exits.
 * The first call on each device looks up the array's device address with
 * that device current (cudaGetSymbolAddress); make that first call before
 * any stream capture begins.  The address belongs to the device's context:
 * after a reset (cudaDeviceReset) the next call finds a new context and looks
 * the address up again, so the first call after a reset must also come
 * before any capture.
 * All calls on a device share the one array and it keeps the previous call's
 * contents: each call clears the ticket words it needs on `stream` before the
 * kernel runs.  Calls that can overlap on the GPU (other streams, other host
 * threads) race on the array and must be serialised by the caller.
 * Errors: as duo_decode_attn, plus DUO_ERR_CAPACITY for a layer too large
 * for the array.
 */
#define DUO_NOALLOC_SCRATCH_BYTES (2u << 20)
duo_status duo_decode_attn_noalloc(const duo_layer_desc* desc, const duo_kv_state* st, const void* q,
                                   void* out, duo_stream_t stream);

/*
 * duo_gated_mix_grad_alpha -- gradient of a loss with respect to the gates of
 * duo_gated_mix, given the gradient dout of its output.  The mix is linear
 * in alpha, d attn / d alpha = full_attn - streaming_attn [Review S3 "Core
 * formula"], and the gates are the only parameters head identification
 * trains [Review S3 "Retrieval-head identification"], so
 *   dalpha[kv] = sum over the query heads h of KV head kv, the sequences,
 *                rows i and features of dout[i][h] * (full - streaming)[i][h].
 *
 * q [B][N][Hq][d]; k, v [B][N][Hkv][d]; dout [B][N][Hq][d] (same dtype);
 * model head order as for duo_gated_mix.  dalpha [Hkv] fp32 device: zeroed
 * by the call, then accumulated with atomics (one add per 32 rows), so the
 * last bits vary with the order the CTAs finish in.  bf16 with d = 128 runs
 * on the tcgen05 tensor cores in two launches that store no attention: by
 * linearity dalpha = <dout, full_attn> - <dout, streaming_attn>, and each
 * launch adds one of the two terms from its epilogue; other dtypes and head
 * sizes run on the CUDA cores.
 * status: one int32 device word (required), as for duo_gated_mix.
 * Errors: DUO_ERR_INVALID_ARG, DUO_ERR_SHAPE, DUO_ERR_UNSUPPORTED, DUO_ERR_CUDA.
 */
duo_status duo_gated_mix_grad_alpha(const duo_layer_desc* desc, const void* q, const void* k, const void* v,
                                    int32_t N, const void* dout, float* dalpha, int32_t* status,
                                    duo_stream_t stream);

/*
 * duo_exp2_fma_probe -- y[i] = the pre-fill softmax's FMA-pipe 2^x of x[i]
 * (Cody-Waite range reduction to x = n + f, f in [-0.5, 0.5], a fitted cubic
 * for 2^f and n added to the exponent field; inputs below -125, -inf
 * included, give the value at -125, 2^-125 within the cubic's 7.5e-5).
 * duo_prefill_chunk computes one exponential pair in four this way and the
 * rest on the SFU; this entry point exposes the routine so that its error
 * can be checked against 2^x.  It is not a step of the attention path: the
 * paper review's S3 "Core formula" only fixes the softmax, not how its
 * exponentials are evaluated.
 * x, y: n fp32 values in device memory (caller-owned; may alias).  n >= 0.
 * Asynchronous on `stream`.
 * Errors: DUO_ERR_INVALID_ARG (NULL with n > 0, n < 0), DUO_ERR_CUDA.
 */
duo_status duo_exp2_fma_probe(const float* x, float* y, int64_t n, duo_stream_t stream);

/*
 * duo_wait_probe -- runs the library's bounded device wait to its limit, so
 * that its failure path can be observed.  Not a step of the attention path
 * (the pages describe no device waits): the kernels wait on mbarriers for
 * their tensor copies and MMAs, each wait bounded in wall time (2 s), after
 * which it ORs DUO_DEV_WAIT_TIMEOUT into the status word and the kernel
 * skips what the wait guarded instead of hanging.  This probe launches one
 * warp that waits, through that same routine, on an mbarrier nothing ever
 * arrives on, with a limit of limit_us microseconds; nothing else is in
 * flight, so the kernel then simply returns.
 * status: one int32 device word, caller-owned; DUO_DEV_WAIT_TIMEOUT is ORed
 *   into it.  limit_us in 1..1000000.  Asynchronous on `stream`.
 * Errors: DUO_ERR_INVALID_ARG, DUO_ERR_CUDA.
 */
duo_status duo_wait_probe(int32_t* status, uint32_t limit_us, duo_stream_t stream);

/*
 * duo_check_status -- synchronise `stream`, copy the state's device status
 * word to *host_status and return DUO_ERR_DEVICE if any bit is set.
 * The only entry point that blocks.
 */
duo_status duo_check_status(const duo_kv_state* st, int32_t* host_status, duo_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* DUO_H */
