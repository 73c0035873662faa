// duo_abi.cu -- the extern "C" entry points of libduo.so: argument checks,
// the host-side gate binarisation / head partition, workspace planning, and
// dispatch to the kernels.  See include/duo.h for the contract of each call.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace {

thread_local std::string g_last_error;

duo_status fail(duo_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
duo_status fail(duo_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

duo_status ok() {
    g_last_error.clear();
    return DUO_OK;
}

duo_status cuda_fail(cudaError_t e, const char* where) {
    return fail(DUO_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

duo_status check_desc(const duo_layer_desc* d) {
    if (!d) return fail(DUO_ERR_INVALID_ARG, "desc is NULL");
    if (d->batch < 1) return fail(DUO_ERR_SHAPE, "batch must be >= 1 (got %d)", d->batch);
    if (d->n_kv_heads < 1 || d->n_kv_heads > DUO_MAX_KV_HEADS)
        return fail(DUO_ERR_INVALID_ARG, "n_kv_heads must be in 1..%d (got %d)", DUO_MAX_KV_HEADS, d->n_kv_heads);
    if (d->n_q_heads < 1 || d->n_q_heads % d->n_kv_heads)
        return fail(DUO_ERR_SHAPE, "n_q_heads (%d) must be a positive multiple of n_kv_heads (%d)", d->n_q_heads,
                    d->n_kv_heads);
    const int g = d->n_q_heads / d->n_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8)
        return fail(DUO_ERR_UNSUPPORTED, "query group size %d is not built (1, 2, 4 or 8)", g);
    if (d->head_dim <= 0) return fail(DUO_ERR_SHAPE, "head_dim must be positive (got %d)", d->head_dim);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(DUO_ERR_UNSUPPORTED, "head_dim %d is not built (64 or 128)", d->head_dim);
    if (d->dtype != DUO_BF16 && d->dtype != DUO_FP32) return fail(DUO_ERR_DTYPE, "unknown dtype %d", d->dtype);
    if (d->sink < 0 || d->recent < 1 || d->sink + d->recent > 1024)
        return fail(DUO_ERR_SHAPE, "need sink >= 0, recent >= 1, sink + recent <= 1024 (got %d, %d)", d->sink,
                    d->recent);
    if (d->page_size != 0 && d->page_size != 64)
        return fail(DUO_ERR_UNSUPPORTED, "page_size must be 0 or 64 (got %d)", d->page_size);
    if (d->n_retrieval < 0 || d->n_retrieval > d->n_kv_heads)
        return fail(DUO_ERR_SHAPE, "n_retrieval %d outside 0..%d", d->n_retrieval, d->n_kv_heads);
    if (d->io_order != DUO_ORDER_MODEL && d->io_order != DUO_ORDER_BLOCK)
        return fail(DUO_ERR_INVALID_ARG, "unknown io_order %d", d->io_order);
    if (d->stream_prefill != DUO_STREAM_LAMBDA && d->stream_prefill != DUO_STREAM_CHUNK)
        return fail(DUO_ERR_INVALID_ARG, "unknown stream_prefill %d", d->stream_prefill);
    if (d->kv_quant != DUO_KV_PLAIN && d->kv_quant != DUO_KV_INT8 && d->kv_quant != DUO_KV_INT4)
        return fail(DUO_ERR_INVALID_ARG, "unknown kv_quant %d", d->kv_quant);
    if (d->kv_quant != DUO_KV_PLAIN &&
        (d->dtype != DUO_BF16 || d->head_dim != 128 || d->page_size != 0 || d->sink + d->recent > 128))
        return fail(DUO_ERR_UNSUPPORTED,
                    "the 8- and 4-bit full caches are built for bf16, head_dim 128, contiguous, sink + recent <= 128");
    if (!std::isfinite(d->scale)) return fail(DUO_ERR_INVALID_ARG, "scale is not finite");
    bool seen[DUO_MAX_KV_HEADS] = {};
    for (int i = 0; i < d->n_kv_heads; ++i) {
        const int h = d->kv_perm[i];
        if (h < 0 || h >= d->n_kv_heads || seen[h])
            return fail(DUO_ERR_INVALID_ARG, "kv_perm is not a permutation of 0..%d (slot %d holds %d)",
                        d->n_kv_heads - 1, i, h);
        seen[h] = true;
    }
    return DUO_OK;
}

void fill_args(const duo_layer_desc* d, duo::LayerArgs& a) {
    a.B = d->batch;
    a.Hq = d->n_q_heads;
    a.Hkv = d->n_kv_heads;
    a.G = a.Hq / a.Hkv;
    a.D = d->head_dim;
    a.R = d->n_retrieval;
    a.S = a.Hkv - a.R;
    a.sink = d->sink;
    a.recent = d->recent;
    a.W = d->sink + d->recent;
    a.dtype = d->dtype;
    a.stream_chunk = d->stream_prefill == DUO_STREAM_CHUNK ? 1 : 0;
    a.kv_bits = d->kv_quant == DUO_KV_INT8 ? 8 : d->kv_quant == DUO_KV_INT4 ? 4 : 0;
    a.page_size = d->page_size;
    a.capacity = a.max_pages = a.n_pages = 0;
    a.scale = d->scale > 0.f ? d->scale : 1.0f / std::sqrt(static_cast<float>(d->head_dim));
    for (int i = 0; i < DUO_MAX_KV_HEADS; ++i) {
        a.q_head0[i] = 0;
        a.kv_head[i] = 0;
        a.slot_of[i] = 0;
    }
    for (int i = 0; i < a.Hkv; ++i) {
        const int h = d->io_order == DUO_ORDER_MODEL ? d->kv_perm[i] : i;
        a.kv_head[i] = h;
        a.q_head0[i] = h * a.G;
        a.slot_of[h] = i;
    }
}

duo_status check_state(const duo_layer_desc* d, const duo_kv_state* st, duo::LayerArgs& a, duo::CacheArgs& c) {
    if (!st) return fail(DUO_ERR_INVALID_ARG, "state is NULL");
    if (!st->seq_len || !st->counters || !st->status)
        return fail(DUO_ERR_INVALID_ARG, "state.seq_len, state.counters and state.status are required");
    const int R = d->n_retrieval, S = d->n_kv_heads - d->n_retrieval;
    if (R > 0) {
        if (!st->k_full || !st->v_full) return fail(DUO_ERR_INVALID_ARG, "full cache pointers are NULL");
        if (!aligned16(st->k_full) || !aligned16(st->v_full))
            return fail(DUO_ERR_INVALID_ARG, "full cache pointers must be 16-byte aligned");
        if (st->capacity < 1) return fail(DUO_ERR_SHAPE, "capacity must be >= 1 (got %d)", st->capacity);
        if (d->page_size) {
            if (!st->page_table) return fail(DUO_ERR_INVALID_ARG, "paged cache needs page_table");
            if (st->max_pages < 1 || st->n_pages < 1)
                return fail(DUO_ERR_SHAPE, "paged cache needs max_pages >= 1 and n_pages >= 1");
            if ((int64_t)st->max_pages * d->page_size != st->capacity)
                return fail(DUO_ERR_SHAPE, "capacity (%d) must equal max_pages * page_size (%d * %d)", st->capacity,
                            st->max_pages, d->page_size);
        }
    }
    if (S > 0) {
        if (!st->k_ring || !st->v_ring || !st->ring_pos)
            return fail(DUO_ERR_INVALID_ARG, "ring pointers are NULL");
        if (!aligned16(st->k_ring) || !aligned16(st->v_ring))
            return fail(DUO_ERR_INVALID_ARG, "ring pointers must be 16-byte aligned");
    }
    a.capacity = R > 0 ? st->capacity : 0;
    a.max_pages = st->max_pages;
    a.n_pages = st->n_pages;
    c.k_full = st->k_full;
    c.v_full = st->v_full;
    c.page_table = st->page_table;
    c.k_ring = st->k_ring;
    c.v_ring = st->v_ring;
    c.ring_pos = st->ring_pos;
    c.seq_len = st->seq_len;
    c.counters = st->counters;
    c.status = st->status;
    c.k_scale = st->k_scale;
    c.v_scale = st->v_scale;
    if (d->kv_quant != DUO_KV_PLAIN && R > 0) {
        if (!st->k_scale || !st->v_scale)
            return fail(DUO_ERR_INVALID_ARG, "an 8- or 4-bit cache needs k_scale and v_scale");
        if (!aligned16(st->k_scale) || !aligned16(st->v_scale))
            return fail(DUO_ERR_INVALID_ARG, "k_scale / v_scale must be 16-byte aligned");
        if (st->capacity % 64) return fail(DUO_ERR_SHAPE, "an 8- or 4-bit cache's capacity must be a multiple of 64");
    }
    return DUO_OK;
}

}  // namespace

// ===========================================================================
// Split-K plan (host): enough CTAs to keep every SM streaming, and no split
// longer than 16K tokens.
// ===========================================================================
namespace duo {
DecodePlan decode_plan(const LayerArgs& a) {
    DecodePlan p{};
    const long pairs = (long)a.B * a.R;
    int ns = 1;
    if (pairs > 0) {
        // 148 SMs x 2 resident CTAs; the streaming CTAs share the same wave
        const long slots = 296, streaming = (long)a.B * a.S;
        const long target_ctas = slots - streaming >= pairs ? slots - streaming : slots;
        ns = (int)(target_ctas / pairs);
        if (ns < 1) ns = 1;
        const int by_len = (a.capacity + 16383) / 16384;
        if (by_len > ns) ns = by_len;
        if (ns > 128) ns = 128;
        if (ns < 1) ns = 1;
    }
    p.nsplit = ns;
    p.partial_floats = (size_t)pairs * ns * a.G * (a.D + 4);
    p.ticket_offset = ((p.partial_floats * sizeof(float)) + 255) / 256 * 256;
    p.counter_offset = p.ticket_offset + ((size_t)pairs * sizeof(uint32_t) + 255) / 256 * 256;
    p.bytes = p.counter_offset + ((size_t)pairs * sizeof(uint32_t) + 255) / 256 * 256;
    if (pairs == 0) p.bytes = 256;
    return p;
}
}  // namespace duo

// ===========================================================================
// extern "C"
// ===========================================================================
extern "C" {

const char* duo_last_error(void) { return g_last_error.c_str(); }

const char* duo_status_string(duo_status s) {
    switch (s) {
        case DUO_OK: return "DUO_OK";
        case DUO_ERR_INVALID_ARG: return "DUO_ERR_INVALID_ARG";
        case DUO_ERR_SHAPE: return "DUO_ERR_SHAPE";
        case DUO_ERR_DTYPE: return "DUO_ERR_DTYPE";
        case DUO_ERR_CAPACITY: return "DUO_ERR_CAPACITY";
        case DUO_ERR_UNSUPPORTED: return "DUO_ERR_UNSUPPORTED";
        case DUO_ERR_CUDA: return "DUO_ERR_CUDA";
        case DUO_ERR_DEVICE: return "DUO_ERR_DEVICE";
    }
    return "DUO_ERR_UNKNOWN";
}

int32_t duo_abi_version(void) { return 4; }

duo_status duo_partition_heads(const float* alpha, int32_t n_kv_heads, float tau, int32_t target_n_retrieval,
                               uint8_t* gate, int32_t* kv_perm, int32_t* kv_inv_perm, int32_t* n_retrieval) {
    if (!alpha || !gate || !kv_perm || !kv_inv_perm || !n_retrieval)
        return fail(DUO_ERR_INVALID_ARG, "duo_partition_heads: NULL argument");
    if (n_kv_heads < 1 || n_kv_heads > DUO_MAX_KV_HEADS)
        return fail(DUO_ERR_INVALID_ARG, "n_kv_heads must be in 1..%d (got %d)", DUO_MAX_KV_HEADS, n_kv_heads);
    for (int h = 0; h < n_kv_heads; ++h)
        if (std::isnan(alpha[h])) return fail(DUO_ERR_INVALID_ARG, "alpha[%d] is NaN", h);
    if (target_n_retrieval > n_kv_heads)
        return fail(DUO_ERR_SHAPE, "target_n_retrieval %d exceeds n_kv_heads %d", target_n_retrieval, n_kv_heads);
    if (target_n_retrieval < 0) {
        if (std::isnan(tau)) return fail(DUO_ERR_INVALID_ARG, "tau is NaN");
        for (int h = 0; h < n_kv_heads; ++h) gate[h] = alpha[h] >= tau ? 1 : 0;
    } else {
        // exactly k heads: the largest alpha, ties to the lower index
        for (int h = 0; h < n_kv_heads; ++h) gate[h] = 0;
        for (int k = 0; k < target_n_retrieval; ++k) {
            int best = -1;
            for (int h = 0; h < n_kv_heads; ++h)
                if (!gate[h] && (best < 0 || alpha[h] > alpha[best])) best = h;
            gate[best] = 1;
        }
    }
    int n = 0;
    for (int h = 0; h < n_kv_heads; ++h)
        if (gate[h]) kv_perm[n++] = h;
    *n_retrieval = n;
    for (int h = 0; h < n_kv_heads; ++h)
        if (!gate[h]) kv_perm[n++] = h;
    for (int i = 0; i < n_kv_heads; ++i) kv_inv_perm[kv_perm[i]] = i;
    return ok();
}

duo_status duo_desc_init(duo_layer_desc* desc, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                         int32_t head_dim, int32_t dtype, const int32_t* kv_perm, int32_t n_retrieval) {
    if (!desc || !kv_perm) return fail(DUO_ERR_INVALID_ARG, "duo_desc_init: NULL argument");
    std::memset(desc, 0, sizeof(*desc));
    desc->batch = batch;
    desc->n_q_heads = n_q_heads;
    desc->n_kv_heads = n_kv_heads;
    desc->head_dim = head_dim;
    desc->sink = 16;
    desc->recent = 64;
    desc->dtype = dtype;
    desc->page_size = 0;
    desc->scale = 0.f;
    desc->n_retrieval = n_retrieval;
    desc->io_order = DUO_ORDER_MODEL;
    desc->stream_prefill = DUO_STREAM_LAMBDA;
    desc->kv_quant = DUO_KV_PLAIN;
    if (n_kv_heads < 1 || n_kv_heads > DUO_MAX_KV_HEADS)
        return fail(DUO_ERR_INVALID_ARG, "n_kv_heads must be in 1..%d (got %d)", DUO_MAX_KV_HEADS, n_kv_heads);
    for (int i = 0; i < n_kv_heads; ++i) desc->kv_perm[i] = kv_perm[i];
    const duo_status s = check_desc(desc);
    return s == DUO_OK ? ok() : s;
}

duo_status duo_desc_validate(const duo_layer_desc* desc) {
    const duo_status s = check_desc(desc);
    return s == DUO_OK ? ok() : s;
}

size_t duo_workspace_bytes(const duo_layer_desc* desc, int32_t op, int32_t max_tokens) {
    if (check_desc(desc) != DUO_OK) return 0;
    if (op == DUO_OP_DECODE) {
        duo::LayerArgs a;
        fill_args(desc, a);
        a.capacity = max_tokens > 0 ? max_tokens : 1;
        return duo::decode_plan(a).bytes;
    }
    if (op == DUO_OP_PREFILL) {
        duo::LayerArgs a;
        fill_args(desc, a);
        if (a.dtype != DUO_BF16 || a.D != 128) return 256;   // the CUDA-core path needs none
        return duo::prefill_workspace_bytes(a, max_tokens > 0 ? max_tokens : 1);
    }
    return 0;
}

size_t duo_prefill_workspace_bytes(const duo_layer_desc* desc, const duo_kv_state* st, int32_t max_chunk) {
    if (check_desc(desc) != DUO_OK || !st) return 0;
    duo::LayerArgs a;
    duo::CacheArgs c;
    fill_args(desc, a);
    if (check_state(desc, st, a, c) != DUO_OK) return 0;
    size_t bytes = duo_workspace_bytes(desc, DUO_OP_PREFILL, max_chunk);
    if (a.kv_bits && a.R > 0) bytes += (duo::dequant_staging_bytes(a) + 255) / 256 * 256;
    return bytes;
}

duo_status duo_permute_heads(const duo_layer_desc* desc, const void* x, void* y, int64_t rows,
                             int32_t heads_per_kv, int64_t head_elems, int32_t elem_bytes, int32_t direction,
                             duo_stream_t stream) {
    duo_status s = check_desc(desc);
    if (s != DUO_OK) return s;
    if (!x || !y) return fail(DUO_ERR_INVALID_ARG, "duo_permute_heads: NULL tensor");
    if (rows < 0 || heads_per_kv < 1 || head_elems < 1)
        return fail(DUO_ERR_SHAPE, "duo_permute_heads: need rows >= 0, heads_per_kv >= 1, head_elems >= 1");
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
        return fail(DUO_ERR_INVALID_ARG, "elem_bytes must be 1, 2, 4 or 8 (got %d)", elem_bytes);
    if (direction != DUO_MODEL_TO_BLOCK && direction != DUO_BLOCK_TO_MODEL)
        return fail(DUO_ERR_INVALID_ARG, "unknown direction %d", direction);
    const int64_t total = rows * (int64_t)desc->n_kv_heads * heads_per_kv * head_elems * elem_bytes;
    const char* xa = static_cast<const char*>(x);
    const char* ya = static_cast<const char*>(y);
    if (xa < ya + total && ya < xa + total) return fail(DUO_ERR_INVALID_ARG, "x and y overlap");
    if (rows == 0) return ok();
    const cudaError_t e = duo::launch_permute(x, y, rows, desc->n_kv_heads, desc->kv_perm, heads_per_kv,
                                              head_elems, elem_bytes, direction, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_permute_heads");
}

duo_status duo_append_kv(const duo_layer_desc* desc, const duo_kv_state* st, const void* k_new, const void* v_new,
                         int32_t T, duo_stream_t stream) {
    duo_status s = check_desc(desc);
    if (s != DUO_OK) return s;
    duo::LayerArgs a;
    duo::CacheArgs c;
    fill_args(desc, a);
    if ((s = check_state(desc, st, a, c)) != DUO_OK) return s;
    if (T < 0) return fail(DUO_ERR_SHAPE, "T must be >= 0 (got %d)", T);
    if (T == 0) return ok();
    if (!k_new || !v_new) return fail(DUO_ERR_INVALID_ARG, "k_new / v_new is NULL");
    if (!aligned16(k_new) || !aligned16(v_new)) return fail(DUO_ERR_INVALID_ARG, "k_new / v_new not 16-byte aligned");
    const cudaError_t e = duo::launch_append(a, c, k_new, v_new, T, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_append_kv");
}

duo_status duo_decode_attn(const duo_layer_desc* desc, const duo_kv_state* st, const void* q, void* out,
                           void* workspace, size_t ws_bytes, duo_stream_t stream) {
    duo_status s = check_desc(desc);
    if (s != DUO_OK) return s;
    duo::LayerArgs a;
    duo::CacheArgs c;
    fill_args(desc, a);
    if ((s = check_state(desc, st, a, c)) != DUO_OK) return s;
    if (!q || !out) return fail(DUO_ERR_INVALID_ARG, "q / out is NULL");
    if (!aligned16(q) || !aligned16(out)) return fail(DUO_ERR_INVALID_ARG, "q / out not 16-byte aligned");
    const duo::DecodePlan plan = duo::decode_plan(a);
    if (!workspace) return fail(DUO_ERR_INVALID_ARG, "workspace is NULL");
    if (!aligned16(workspace)) return fail(DUO_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    if (ws_bytes < plan.bytes)
        return fail(DUO_ERR_CAPACITY, "workspace holds %zu bytes, decode needs %zu", ws_bytes, plan.bytes);
    const cudaError_t e = duo::launch_decode(a, c, plan, q, out, workspace, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_decode_attn");
}

duo_status duo_decode_step(const duo_layer_desc* desc, const duo_kv_state* st, const void* q, const void* k_new,
                           const void* v_new, void* out, void* workspace, size_t ws_bytes, duo_stream_t stream) {
    duo_status s = check_desc(desc);
    if (s != DUO_OK) return s;
    duo::LayerArgs a;
    duo::CacheArgs c;
    fill_args(desc, a);
    if ((s = check_state(desc, st, a, c)) != DUO_OK) return s;
    if (!q || !out || !k_new || !v_new) return fail(DUO_ERR_INVALID_ARG, "q / k_new / v_new / out is NULL");
    if (!aligned16(q) || !aligned16(out) || !aligned16(k_new) || !aligned16(v_new))
        return fail(DUO_ERR_INVALID_ARG, "q / k_new / v_new / out not 16-byte aligned");
    const duo::DecodePlan plan = duo::decode_plan(a);
    if (!workspace) return fail(DUO_ERR_INVALID_ARG, "workspace is NULL");
    if (!aligned16(workspace)) return fail(DUO_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    if (ws_bytes < plan.bytes)
        return fail(DUO_ERR_CAPACITY, "workspace holds %zu bytes, decode needs %zu", ws_bytes, plan.bytes);
    const cudaError_t e = duo::launch_decode(a, c, plan, q, out, workspace, (cudaStream_t)stream, k_new, v_new);
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_decode_step");
}

duo_status duo_prefill_chunk(const duo_layer_desc* desc, const duo_kv_state* st, const void* q, const void* k_chunk,
                             const void* v_chunk, int32_t C, void* out, void* workspace, size_t ws_bytes,
                             duo_stream_t stream) {
    duo_status s = check_desc(desc);
    if (s != DUO_OK) return s;
    duo::LayerArgs a;
    duo::CacheArgs c;
    fill_args(desc, a);
    if ((s = check_state(desc, st, a, c)) != DUO_OK) return s;
    if (C < 1) return fail(DUO_ERR_SHAPE, "chunk length must be >= 1 (got %d)", C);
    if (!q || !k_chunk || !v_chunk || !out) return fail(DUO_ERR_INVALID_ARG, "q / k_chunk / v_chunk / out is NULL");
    if (!aligned16(q) || !aligned16(k_chunk) || !aligned16(v_chunk) || !aligned16(out))
        return fail(DUO_ERR_INVALID_ARG, "pre-fill tensors must be 16-byte aligned");
    if (desc->page_size != 0)
        return fail(DUO_ERR_UNSUPPORTED, "duo_prefill_chunk takes a contiguous full cache (page_size 0)");
    cudaError_t e;
    if (a.kv_bits && a.R > 0) {
        // an 8- or 4-bit full cache: its rows below seq_len are staged in
        // the workspace -- K codes as bf16, V codes x16 as fp16, each row's scales --
        // and the tensor-core pre-fill reads the codes as its cache and
        // applies the scales to the scores and to p; the rest of the
        // workspace serves the key-range splits
        const size_t staging = (duo::dequant_staging_bytes(a) + 255) / 256 * 256;
        if (!workspace || ws_bytes < staging)
            return fail(DUO_ERR_CAPACITY,
                        "an 8- or 4-bit layer's pre-fill needs a workspace of duo_prefill_workspace_bytes (at least "
                        "%zu bytes; given %zu)", staging, workspace ? ws_bytes : (size_t)0);
        if (!aligned16(workspace)) return fail(DUO_ERR_INVALID_ARG, "workspace not 16-byte aligned");
        duo::LayerArgs ap = a;
        ap.kv_bits = 0;
        if (!duo::prefill_tc_supported(ap))
            return fail(DUO_ERR_UNSUPPORTED, "tensor-core pre-fill cannot take this layer");
        e = duo::launch_dequant(a, c, workspace, (cudaStream_t)stream);
        if (e == cudaSuccess) {
            const size_t code_bytes = (size_t)a.B * a.R * a.capacity * 128 * 2;   // one of K, V
            duo::CacheArgs cp = c;
            cp.k_full = workspace;
            cp.v_full = static_cast<uint8_t*>(workspace) + code_bytes;
            cp.k_scale = cp.v_scale = nullptr;
            const float* qscale = reinterpret_cast<const float*>(static_cast<uint8_t*>(workspace) + 2 * code_bytes);
            e = duo::launch_prefill_tc(ap, cp, q, k_chunk, v_chunk, C, out, static_cast<uint8_t*>(workspace) + staging,
                                       ws_bytes - staging, (cudaStream_t)stream, nullptr, qscale);
        }
    } else if (a.dtype == DUO_BF16 && a.D == 128) {
        if (!duo::prefill_tc_supported(a))
            return fail(DUO_ERR_UNSUPPORTED, "tensor-core pre-fill cannot take this layer");
        e = duo::launch_prefill_tc(a, c, q, k_chunk, v_chunk, C, out, workspace, ws_bytes, (cudaStream_t)stream);
    } else {
        e = duo::launch_simt_attention(a, &c, nullptr, q, k_chunk, v_chunk, C, out, 0, (cudaStream_t)stream);
    }
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_prefill_chunk");
}

duo_status duo_gated_mix(const duo_layer_desc* desc, const float* alpha, const void* q, const void* k, const void* v,
                         int32_t N, void* out, int32_t* status, duo_stream_t stream) {
    duo_status s = check_desc(desc);
    if (s != DUO_OK) return s;
    if (!alpha || !q || !k || !v || !out || !status) return fail(DUO_ERR_INVALID_ARG, "duo_gated_mix: NULL argument");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(DUO_ERR_INVALID_ARG, "duo_gated_mix tensors must be 16-byte aligned");
    if (N < 0) return fail(DUO_ERR_SHAPE, "N must be >= 0 (got %d)", N);
    if (N == 0) return ok();
    {
        // out is written while q, k and v are still being read
        const size_t es = desc->dtype == DUO_BF16 ? 2 : 4;
        const size_t rows = (size_t)desc->batch * (size_t)N;
        const size_t nq = rows * desc->n_q_heads * desc->head_dim * es;
        const size_t nkv = rows * desc->n_kv_heads * desc->head_dim * es;
        const uintptr_t o = (uintptr_t)out;
        auto hits = [&](const void* p, size_t n) { return o < (uintptr_t)p + n && (uintptr_t)p < o + nq; };
        if (hits(q, nq) || hits(k, nkv) || hits(v, nkv))
            return fail(DUO_ERR_INVALID_ARG, "duo_gated_mix: out overlaps q, k or v");
    }
    duo::LayerArgs a;
    fill_args(desc, a);
    // the mix runs in model head order over whole sequences
    for (int i = 0; i < a.Hkv; ++i) {
        a.kv_head[i] = i;
        a.q_head0[i] = i * a.G;
        a.slot_of[i] = i;
    }
    // bf16, d 128: both attentions on the tensor cores, as two launches of
    // the pre-fill kernel over one chunk with no cache -- every KV head in
    // the streaming block (Lambda mask) writes the streaming attention to
    // out, then every KV head in the retrieval block (causal) mixes its
    // result with it in the epilogue
    duo::LayerArgs as = a, ac = a;
    as.R = 0;
    as.S = a.Hkv;
    ac.R = a.Hkv;
    ac.S = 0;
    for (duo::LayerArgs* x : {&as, &ac}) {
        x->page_size = 0;
        x->capacity = 0;
        x->stream_chunk = 0;
        x->kv_bits = 0;
    }
    if (duo::prefill_tc_supported(as) && duo::prefill_tc_supported(ac)) {
        duo::CacheArgs none{};   // no lengths, no caches: every sequence starts at position 0
        none.status = status;    // device conditions (a wait that ran out) are reported here
        const duo::EpiArgs mix{duo::EPI_MIX, alpha, nullptr, nullptr, 0.f};
        cudaError_t e = duo::launch_prefill_tc(as, none, q, k, v, N, out, nullptr, 0, (cudaStream_t)stream);
        if (e == cudaSuccess)
            e = duo::launch_prefill_tc(ac, none, q, k, v, N, out, nullptr, 0, (cudaStream_t)stream, &mix);
        return e == cudaSuccess ? ok() : cuda_fail(e, "duo_gated_mix");
    }
    const cudaError_t e = duo::launch_simt_attention(a, nullptr, alpha, q, k, v, N, out, 1, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_gated_mix");
}

duo_status duo_gated_mix_grad_alpha(const duo_layer_desc* desc, const void* q, const void* k, const void* v,
                                    int32_t N, const void* dout, float* dalpha, int32_t* status,
                                    duo_stream_t stream) {
    duo_status s = check_desc(desc);
    if (s != DUO_OK) return s;
    if (!q || !k || !v || !dout || !dalpha || !status)
        return fail(DUO_ERR_INVALID_ARG, "duo_gated_mix_grad_alpha: NULL argument");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout))
        return fail(DUO_ERR_INVALID_ARG, "duo_gated_mix_grad_alpha tensors must be 16-byte aligned");
    if (N < 0) return fail(DUO_ERR_SHAPE, "N must be >= 0 (got %d)", N);
    cudaError_t e = cudaMemsetAsync(dalpha, 0, sizeof(float) * desc->n_kv_heads, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "duo_gated_mix_grad_alpha");
    if (N == 0) return ok();
    duo::LayerArgs a;
    fill_args(desc, a);
    for (int i = 0; i < a.Hkv; ++i) {   // model head order, as for duo_gated_mix
        a.kv_head[i] = i;
        a.q_head0[i] = i * a.G;
        a.slot_of[i] = i;
    }
    // bf16, d 128: the mix is linear in alpha, so dalpha = <dout, causal> -
    // <dout, streaming>; each term is one launch of the tensor-core kernel
    // whose epilogue adds its rows' dot products into dalpha (no attention
    // is stored, so no scratch is needed)
    duo::LayerArgs as = a, ac = a;
    as.R = 0;
    as.S = a.Hkv;
    ac.R = a.Hkv;
    ac.S = 0;
    for (duo::LayerArgs* x : {&as, &ac}) {
        x->page_size = 0;
        x->capacity = 0;
        x->stream_chunk = 0;
        x->kv_bits = 0;
    }
    if (duo::prefill_tc_supported(as) && duo::prefill_tc_supported(ac)) {
        duo::CacheArgs none{};
        none.status = status;
        const duo::EpiArgs minus{duo::EPI_DOT, nullptr, dout, dalpha, -1.f};
        const duo::EpiArgs plus{duo::EPI_DOT, nullptr, dout, dalpha, 1.f};
        e = duo::launch_prefill_tc(as, none, q, k, v, N, nullptr, nullptr, 0, (cudaStream_t)stream, &minus);
        if (e == cudaSuccess)
            e = duo::launch_prefill_tc(ac, none, q, k, v, N, nullptr, nullptr, 0, (cudaStream_t)stream, &plus);
        return e == cudaSuccess ? ok() : cuda_fail(e, "duo_gated_mix_grad_alpha");
    }
    e = duo::launch_simt_attention(a, nullptr, nullptr, q, k, v, N, nullptr, 2, (cudaStream_t)stream, dout, dalpha);
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_gated_mix_grad_alpha");
}

duo_status duo_exp2_fma_probe(const float* x, float* y, int64_t n, duo_stream_t stream) {
    if (n < 0) return fail(DUO_ERR_INVALID_ARG, "duo_exp2_fma_probe: n must be >= 0 (got %lld)", (long long)n);
    if (n > 0 && (!x || !y)) return fail(DUO_ERR_INVALID_ARG, "duo_exp2_fma_probe: NULL argument");
    cudaError_t e = duo::launch_exp2_fma_probe(x, y, n, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_exp2_fma_probe");
}

duo_status duo_wait_probe(int32_t* status, uint32_t limit_us, duo_stream_t stream) {
    if (!status) return fail(DUO_ERR_INVALID_ARG, "duo_wait_probe: status is NULL");
    if (limit_us < 1 || limit_us > 1000000u)
        return fail(DUO_ERR_INVALID_ARG, "duo_wait_probe: limit_us must be in 1..1000000 (got %u)", limit_us);
    const cudaError_t e = duo::launch_wait_probe(status, (uint64_t)limit_us * 1000ull, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_wait_probe");
}

duo_status duo_check_status(const duo_kv_state* st, int32_t* host_status, duo_stream_t stream) {
    if (!st || !st->status || !host_status) return fail(DUO_ERR_INVALID_ARG, "duo_check_status: NULL argument");
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, st->status, sizeof v, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "duo_check_status");
    *host_status = v;
    if (v) return fail(DUO_ERR_DEVICE, "device status bits 0x%x", v);
    return ok();
}

}  // extern "C"

// ===========================================================================
// duo_decode_attn_noalloc: decode with library-owned scratch for callers that
// cannot allocate device memory themselves (see include/duo.h).
// ===========================================================================
namespace {

// Split-K partials and ticket words of duo_decode_attn_noalloc.  In host code
// this name is only a stand-in for the symbol: the device address comes from
// cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DUO_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
// the array's device address per device ordinal, and the context it was
// looked up in: a device reset makes a new context, which loads the module
// again and may place the array elsewhere
void* g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    }
    return fn;
}

}  // namespace

extern "C" duo_status duo_decode_attn_noalloc(const duo_layer_desc* desc, const duo_kv_state* st, const void* q,
                                              void* out, duo_stream_t stream) {
    duo_status s = check_desc(desc);
    if (s != DUO_OK) return s;
    duo::LayerArgs a;
    duo::CacheArgs c;
    fill_args(desc, a);
    if ((s = check_state(desc, st, a, c)) != DUO_OK) return s;
    if (!q || !out) return fail(DUO_ERR_INVALID_ARG, "q / out is NULL");
    if (!aligned16(q) || !aligned16(out)) return fail(DUO_ERR_INVALID_ARG, "q / out not 16-byte aligned");
    const duo::DecodePlan plan = duo::decode_plan(a);
    if (plan.bytes > DUO_NOALLOC_SCRATCH_BYTES)
        return fail(DUO_ERR_CAPACITY,
                    "duo_decode_attn_noalloc: this layer needs %zu bytes of split-K scratch, the built-in array "
                    "holds %u; call duo_decode_attn with a workspace instead",
                    plan.bytes, (unsigned)DUO_NOALLOC_SCRATCH_BYTES);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "duo_decode_attn_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(DUO_ERR_UNSUPPORTED, "device ordinal %d above %d", dev, kMaxDevices);
    // the device's current context (cudaGetDevice above made the runtime's
    // context current)
    CUcontext ctx = nullptr;
    const CtxGetCurrentFn get_ctx = ctx_get_current();
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS || !ctx)
        return fail(DUO_ERR_CUDA, "duo_decode_attn_noalloc: cannot read the current CUDA context");
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_ptr[dev] || g_noalloc_ctx[dev] != ctx) {
            // once per device (and again after a reset gave it a new
            // context), with that device current
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess) return cuda_fail(e, "duo_decode_attn_noalloc: cudaGetSymbolAddress");
            g_noalloc_ptr[dev] = p;
            g_noalloc_ctx[dev] = ctx;
        }
        scratch = g_noalloc_ptr[dev];
    }
    // the ticket words must start at zero; the array keeps the previous call's contents
    const size_t ticket_bytes = plan.bytes - plan.ticket_offset;
    e = cudaMemsetAsync(static_cast<unsigned char*>(scratch) + plan.ticket_offset, 0, ticket_bytes,
                        (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "duo_decode_attn_noalloc: clearing the ticket words");
    e = duo::launch_decode(a, c, plan, q, out, scratch, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "duo_decode_attn_noalloc");
}
