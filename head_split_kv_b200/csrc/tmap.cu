// tmap.cu -- host-side encoding of TMA tensor maps (cuTensorMapEncodeTiled,
// reached through cudaGetDriverEntryPoint so the library needs no link
// against libcuda), plus a small cache so repeated calls on the same buffers
// encode nothing.
#include <cstring>
#include <mutex>

#include "internal.h"

namespace duo {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

struct Entry {
    bool used;
    const void* base;
    int rank, dtype, swizzle;
    uint64_t dims[5], strides[4];
    uint32_t box[5];
    CUtensorMap map;
};
constexpr int kEntries = 64;
Entry g_cache[kEntries];
int g_next = 0;
std::mutex g_mu;

}  // namespace

bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box) {
    return encode_tmap(map, base, rank, dims, strides_bytes, box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128);
}

bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                 const uint32_t* box, int dtype, int swizzle_bytes) {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < kEntries; ++i) {
        const Entry& e = g_cache[i];
        if (e.used && e.base == base && e.rank == rank && e.dtype == dtype && e.swizzle == swizzle_bytes &&
            !memcmp(e.dims, dims, rank * sizeof(uint64_t)) &&
            !memcmp(e.strides, strides_bytes, (rank - 1) * sizeof(uint64_t)) &&
            !memcmp(e.box, box, rank * sizeof(uint32_t))) {
            *map = e.map;
            return true;
        }
    }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
    const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swizzle_bytes == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : swizzle_bytes == 32  ? CU_TENSOR_MAP_SWIZZLE_32B
                                                         : CU_TENSOR_MAP_SWIZZLE_NONE;
    const CUresult r = fn(map, (CUtensorMapDataType)dtype, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bx, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    Entry& e = g_cache[g_next];
    g_next = (g_next + 1) % kEntries;
    e.used = true;
    e.base = base;
    e.rank = rank;
    e.dtype = dtype;
    e.swizzle = swizzle_bytes;
    memcpy(e.dims, dims, rank * sizeof(uint64_t));
    memcpy(e.strides, strides_bytes, (rank - 1) * sizeof(uint64_t));
    memcpy(e.box, box, rank * sizeof(uint32_t));
    e.map = *map;
    return true;
}

}  // namespace duo
