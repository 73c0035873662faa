// permute.cu -- duo_permute_heads: move head blocks between the model's
// order and the contiguous [retrieval | streaming] block order
// [Review S3 "Deployment optimisation": the output channels of the Q/K/V
// projections are reordered so that each head type forms one block].
//
// A gather over rows of [Hkv * heads_per_kv] head blocks of head_elems
// elements.  Head blocks whose byte length is a multiple of 16 are moved in
// 16-byte pieces, others byte by byte.
#include "common.cuh"
#include "internal.h"

namespace duo {
namespace {

struct PermArgs {
    int perm[DUO_MAX_KV_HEADS];
};

template <typename V>
__global__ void __launch_bounds__(256) permute_kernel(const V* __restrict__ x, V* __restrict__ y, const long rows,
                                                      const int hkv, const PermArgs pa, const int hpk,
                                                      const long vec_per_head, const int direction) {
    const long heads = (long)hkv * hpk;
    const long total = rows * heads * vec_per_head;
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
        const long e = i % vec_per_head;
        const long rh = i / vec_per_head;
        const int hy = (int)(rh % heads);       // destination head block
        const long r = rh / heads;
        const int slot = hy / hpk, g = hy % hpk;
        int hx;
        if (direction == DUO_MODEL_TO_BLOCK) {
            hx = pa.perm[slot] * hpk + g;        // y in block order
        } else {
            // y in model order: model KV head `slot` sits at block slot inv(slot)
            int inv = 0;
            for (int k = 0; k < hkv; ++k)
                if (pa.perm[k] == slot) inv = k;
            hx = inv * hpk + g;
        }
        y[(r * heads + hy) * vec_per_head + e] = x[(r * heads + hx) * vec_per_head + e];
    }
}

}  // namespace

cudaError_t launch_permute(const void* x, void* y, int64_t rows, int hkv, const int* perm, int heads_per_kv,
                           int64_t head_elems, int elem_bytes, int direction, cudaStream_t s) {
    PermArgs pa{};
    for (int i = 0; i < hkv; ++i) pa.perm[i] = perm[i];
    const long head_bytes = head_elems * elem_bytes;
    const bool vec = (head_bytes % 16 == 0) && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) % 16 == 0);
    const long vph = vec ? head_bytes / 16 : head_bytes;
    const long total = rows * hkv * heads_per_kv * vph;
    long blocks = (total + 255) / 256;
    if (blocks > 148L * 16) blocks = 148L * 16;
    if (blocks < 1) blocks = 1;
    if (vec)
        permute_kernel<uint4><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4*>(x), static_cast<uint4*>(y),
                                                               rows, hkv, pa, heads_per_kv, vph, direction);
    else
        permute_kernel<uint8_t><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint8_t*>(x),
                                                                 static_cast<uint8_t*>(y), rows, hkv, pa,
                                                                 heads_per_kv, vph, direction);
    return cudaGetLastError();
}

}  // namespace duo
