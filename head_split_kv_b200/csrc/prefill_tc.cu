// prefill_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) chunked pre-fill.
#include "common.cuh"
#include "internal.h"

namespace duo {

bool prefill_tc_supported(const LayerArgs& a) { (void)a; return false; }

cudaError_t launch_prefill_tc(const LayerArgs& a, const CacheArgs& c, const void* q, const void* k_chunk,
                              const void* v_chunk, int C, void* out, cudaStream_t s) {
    (void)a; (void)c; (void)q; (void)k_chunk; (void)v_chunk; (void)C; (void)out; (void)s;
    return cudaErrorNotSupported;
}

}  // namespace duo
