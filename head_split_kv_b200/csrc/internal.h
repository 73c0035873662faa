// internal.h -- launch parameters shared between the C-ABI layer (duo_abi.cu)
// and the kernels.  Not part of the public ABI.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "duo.h"

namespace duo {

// Raises `kernel`'s dynamic shared memory limit to `bytes` once per device:
// function attributes belong to a device's context, so a process that
// launches on several devices sets them on each.  `done` holds a bit per
// device (ordinal < 64; higher ordinals set the attribute on every call).
template <typename K>
inline cudaError_t smem_limit_once(K* kernel, int bytes, std::atomic<unsigned long long>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

// Flattened, validated view of a layer descriptor plus state, passed by
// value to every kernel.
struct LayerArgs {
    int B, Hq, Hkv, G, D, R, S, sink, recent, W;
    int dtype, page_size, capacity, max_pages, n_pages;
    int stream_chunk;  // pre-fill: streaming heads see the whole chunk (DUO_STREAM_CHUNK)
    int kv_bits;       // the full cache holds 8- or 4-bit codes + scales (DUO_KV_INT8 / DUO_KV_INT4); 0: plain
    float scale;       // softmax scale
    // For block slot i (0..Hkv-1): index of its first query head and of its
    // KV head in the caller's q / k / v / out tensors (model or block order).
    int q_head0[DUO_MAX_KV_HEADS];
    int kv_head[DUO_MAX_KV_HEADS];
    // Inverse of kv_head: block slot of the caller's KV head h.
    int slot_of[DUO_MAX_KV_HEADS];
};

struct CacheArgs {
    void* k_full;
    void* v_full;
    const int32_t* page_table;
    void* k_ring;
    void* v_ring;
    int32_t* ring_pos;
    int32_t* seq_len;
    uint32_t* counters;
    int32_t* status;
    float* k_scale;    // 8- / 4-bit full cache: per-row scales [B][R][capacity]
    float* v_scale;
};

// Split-K plan of a decode call: number of splits per (sequence, retrieval
// head) and the workspace carve-up.
struct DecodePlan {
    int nsplit;
    size_t partial_floats;  // B * R * nsplit * G * (D + 2)
    size_t ticket_offset;   // bytes from workspace start to the ticket words
    size_t counter_offset;  // ... to the tile counters (one per pair, after the tickets)
    size_t bytes;           // total workspace bytes
};

DecodePlan decode_plan(const LayerArgs& a);

cudaError_t launch_append(const LayerArgs& a, const CacheArgs& c, const void* k_new, const void* v_new, int T,
                          cudaStream_t s);
// k_new / v_new non-NULL: append the new token first (duo_decode_step).
cudaError_t launch_decode(const LayerArgs& a, const CacheArgs& c, const DecodePlan& plan, const void* q, void* out,
                          void* workspace, cudaStream_t s, const void* k_new = nullptr,
                          const void* v_new = nullptr);
// CUDA-core attention: chunked pre-fill (mode 0), gated mix (mode 1) or the
// gated mix's gate gradient (mode 2: dout in, dalpha accumulated).
cudaError_t launch_simt_attention(const LayerArgs& a, const CacheArgs* c, const float* alpha, const void* q,
                                  const void* k, const void* v, int n_tokens, void* out, int mode, cudaStream_t s,
                                  const void* dout = nullptr, float* dalpha = nullptr);
// tcgen05 pre-fill for bf16, d = 128; returns cudaErrorNotSupported when it
// cannot take the call.
// Key-range split plan of the tensor-core pre-fill (see prefill_tc.cu).
struct PrefillPlan {
    int ns;                 // CTAs per retrieval unit
    size_t ticket_offset;   // bytes from workspace start to the ticket words
    size_t bytes;           // workspace bytes the plan needs (256 when ns == 1)
};
int sm_count();
PrefillPlan prefill_plan(const LayerArgs& a, int C, int n_sms);
size_t prefill_workspace_bytes(const LayerArgs& a, int max_chunk);
// Epilogues of the tensor-core attention kernel: the pre-fill's store, and
// the gated mix's two (no key-range splits):
//   EPI_MIX: out is read back as the streaming attention and overwritten
//            with alpha[kv] * result + (1 - alpha[kv]) * out;
//   EPI_DOT: nothing is stored; sign * <dout row, result row> summed over
//            the rows is added into dalpha[kv] (atomics).
enum { EPI_STORE = 0, EPI_MIX = 1, EPI_DOT = 2 };
struct EpiArgs {
    int mode;
    const float* alpha;   // EPI_MIX: [Hkv] gates
    const void* dout;     // EPI_DOT: [B][C][Hq][d] bf16
    float* dalpha;        // EPI_DOT: [Hkv] accumulated
    float sign;           // EPI_DOT: +1 or -1
};
// qscale non-NULL: the full cache holds 8- or 4-bit codes (as bf16 values)
// and qscale [B][R][capacity][4] fp32 the (k scale, v scale, -, -) of each
// row, applied to the scores and to p.
cudaError_t launch_prefill_tc(const LayerArgs& a, const CacheArgs& c, const void* q, const void* k_chunk,
                              const void* v_chunk, int C, void* out, void* workspace, size_t ws_bytes,
                              cudaStream_t s, const EpiArgs* epi = nullptr, const float* qscale = nullptr);
cudaError_t launch_exp2_fma_probe(const float* x, float* y, int64_t n, cudaStream_t s);
// An 8- or 4-bit layer's cached rows (below seq_len) staged for the
// tensor-core pre-fill: the codes as bf16 values (exact) in a contiguous
// [B][R][capacity][128] K area, the same for V, then [B][R][capacity][4]
// fp32 (k scale, v scale, 0, 0).
size_t dequant_staging_bytes(const LayerArgs& a);
cudaError_t launch_dequant(const LayerArgs& a, const CacheArgs& c, void* staging, cudaStream_t s);
// One warp waits on an mbarrier that never completes, with the given limit.
cudaError_t launch_wait_probe(int32_t* status, uint64_t limit_ns, cudaStream_t s);

bool prefill_tc_supported(const LayerArgs& a);
// bf16 tensor map of `rank` dims (innermost first), 64-element-wide boxes with
// the 128-byte swizzle, out-of-range elements read as zero; encodings are
// cached per (base, dims, strides, box).  False if the driver refuses.
bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box);
// Any element type (a CUtensorMapDataType) and a 32/64/128-byte swizzle (0: none).
bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                 const uint32_t* box, int dtype, int swizzle_bytes);

cudaError_t launch_permute(const void* x, void* y, int64_t rows, int hkv, const int* perm, int heads_per_kv,
                           int64_t head_elems, int elem_bytes, int direction, cudaStream_t s);

}  // namespace duo
