// common.cuh -- device helpers shared by the libduo kernels (sm_100a).
//
// mbarrier, bulk-copy and timer wrappers in inline PTX, bf16 <-> fp32
// conversion, and the bounded-wait policy: every spin on an mbarrier gives up
// after DUO_WAIT_TIMEOUT_NS of wall time, ORs DUO_DEV_WAIT_TIMEOUT into the
// state's status word and returns false, so a kernel never hangs the GPU.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "duo.h"

#ifndef DUO_WAIT_TIMEOUT_NS
#define DUO_WAIT_TIMEOUT_NS 2000000000ull  // 2 s
#endif

namespace duo {

constexpr float kLog2e = 1.4426950408889634f;
// Finite stand-in for -inf in running maxima: exp2 of (sentinel - finite) is 0
// and (sentinel - sentinel) is 0, so no NaN can arise.
constexpr float kNegBig = -1.0e30f;

// Index checks of the debug build (compiled with -DDUO_DEBUG_BOUNDS into
// libduo_debug.so): a check that fails ORs DUO_DEV_BOUNDS into the status word
// and the caller skips the access it guards -- never a trap.  In the release
// build every check is the constant true and compiles away.  The checks sit
// at the writes whose addresses come from computed indices (outputs, cache
// rows, ring slots, split records) and at the untiled bulk reads; tensor-map
// copies are bounds-checked by the TMA unit itself.
__device__ __forceinline__ bool bounds_ok(bool ok, int32_t* status) {
#ifdef DUO_DEBUG_BOUNDS
    if (!ok && status != nullptr) atomicOr(status, (int32_t)DUO_DEV_BOUNDS);
    return ok;
#else
    (void)ok;
    (void)status;
    return true;
#endif
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async (TMA / tensor) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy accesses (tcgen05.mma reading operands written by threads).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One potentially blocking test of the phase: the thread may sleep until the
// phase completes or about `hint_ns` pass, so waiting warps do not spin.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns = 20000) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete: gives up
// after `limit_ns` of wall time, ORs DUO_DEV_WAIT_TIMEOUT into *status (when
// given) and returns false.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, int32_t* status, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            if (status) atomicOr(status, DUO_DEV_WAIT_TIMEOUT);
            return false;
        }
    }
}

// The kernels' wait: the same, with the library's limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* status) {
    return mbar_wait_for(bar, parity, status, DUO_WAIT_TIMEOUT_NS);
}

// ------------------------------------------------------------- bulk copies

// Contiguous global -> shared copy on the TMA engine, completing `bytes`
// transaction bytes on `bar`.  src, dst 16-byte aligned; bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------- packed fp32 arithmetic

// Two fp32 fused multiply-adds in one instruction (sm_100 f32x2 forms).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(*reinterpret_cast<unsigned long long*>(&d))
        : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)),
          "l"(*reinterpret_cast<unsigned long long*>(&c)));
    return d;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(*reinterpret_cast<unsigned long long*>(&d))
        : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)));
    return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("add.rn.f32x2 %0, %1, %2;"
        : "=l"(*reinterpret_cast<unsigned long long*>(&d))
        : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)));
    return d;
}

// max(a, b, c) in one instruction (sm_100 three-input form)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// ------------------------------------------------- tiled TMA copies

// Tiled global -> shared copy of one box of a tensor map (coordinates
// innermost first), completing the box's bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

// Asks the bulk-copy engine to bring a contiguous global range into L2 (a
// hint: nothing is written to shared memory, nothing to wait for).  The
// address is 16-byte aligned and `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// A relaxed, device-scope load: well defined even while another grid
// updates the word with atomics (it returns the old or the new value).
__device__ __forceinline__ int ld_relaxed_gpu(const int32_t* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------ conversions

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static constexpr int kDtype = DUO_BF16;
    __device__ static __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ static __forceinline__ __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};

template <>
struct Elem<float> {
    static constexpr int kBytes = 4;
    static constexpr int kDtype = DUO_FP32;
    __device__ static __forceinline__ float to_f32(float x) { return x; }
    __device__ static __forceinline__ float from_f32(float x) { return x; }
};

// Loads N consecutive elements starting at p (16-byte aligned for N*bytes >= 16)
// and widens them to fp32.
template <typename T, int N>
__device__ __forceinline__ void load_row_f32(const T* p, float (&out)[N]);

template <>
__device__ __forceinline__ void load_row_f32<__nv_bfloat16, 8>(const __nv_bfloat16* p, float (&o)[8]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    o[0] = bf16_lo(w.x); o[1] = bf16_hi(w.x); o[2] = bf16_lo(w.y); o[3] = bf16_hi(w.y);
    o[4] = bf16_lo(w.z); o[5] = bf16_hi(w.z); o[6] = bf16_lo(w.w); o[7] = bf16_hi(w.w);
}
template <>
__device__ __forceinline__ void load_row_f32<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&o)[4]) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    o[0] = bf16_lo(w.x); o[1] = bf16_hi(w.x); o[2] = bf16_lo(w.y); o[3] = bf16_hi(w.y);
}
template <>
__device__ __forceinline__ void load_row_f32<float, 8>(const float* p, float (&o)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
template <>
__device__ __forceinline__ void load_row_f32<float, 4>(const float* p, float (&o)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
}

// Loads 2*N consecutive elements as N fp32 pairs.
template <typename T, int N>
__device__ __forceinline__ void load_pairs_f32(const T* p, float2 (&out)[N]);

template <>
__device__ __forceinline__ void load_pairs_f32<__nv_bfloat16, 4>(const __nv_bfloat16* p, float2 (&o)[4]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    o[0] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
    o[1] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
    o[2] = make_float2(bf16_lo(w.z), bf16_hi(w.z));
    o[3] = make_float2(bf16_lo(w.w), bf16_hi(w.w));
}
template <>
__device__ __forceinline__ void load_pairs_f32<__nv_bfloat16, 2>(const __nv_bfloat16* p, float2 (&o)[2]) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    o[0] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
    o[1] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
}
template <>
__device__ __forceinline__ void load_pairs_f32<float, 4>(const float* p, float2 (&o)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    o[0] = make_float2(a.x, a.y);
    o[1] = make_float2(a.z, a.w);
    o[2] = make_float2(b.x, b.y);
    o[3] = make_float2(b.z, b.w);
}
template <>
__device__ __forceinline__ void load_pairs_f32<float, 2>(const float* p, float2 (&o)[2]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    o[0] = make_float2(a.x, a.y);
    o[1] = make_float2(a.z, a.w);
}

// Stores N fp32 values as N consecutive elements (rounded once for bf16).
template <typename T, int N>
__device__ __forceinline__ void store_row(T* p, const float (&v)[N]);

template <>
__device__ __forceinline__ void store_row<__nv_bfloat16, 8>(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 w;
    __nv_bfloat162 t;
    t = __floats2bfloat162_rn(v[0], v[1]); w.x = *reinterpret_cast<uint32_t*>(&t);
    t = __floats2bfloat162_rn(v[2], v[3]); w.y = *reinterpret_cast<uint32_t*>(&t);
    t = __floats2bfloat162_rn(v[4], v[5]); w.z = *reinterpret_cast<uint32_t*>(&t);
    t = __floats2bfloat162_rn(v[6], v[7]); w.w = *reinterpret_cast<uint32_t*>(&t);
    *reinterpret_cast<uint4*>(p) = w;
}
template <>
__device__ __forceinline__ void store_row<__nv_bfloat16, 4>(__nv_bfloat16* p, const float (&v)[4]) {
    uint2 w;
    __nv_bfloat162 t;
    t = __floats2bfloat162_rn(v[0], v[1]); w.x = *reinterpret_cast<uint32_t*>(&t);
    t = __floats2bfloat162_rn(v[2], v[3]); w.y = *reinterpret_cast<uint32_t*>(&t);
    *reinterpret_cast<uint2*>(p) = w;
}
template <>
__device__ __forceinline__ void store_row<float, 8>(float* p, const float (&v)[8]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
template <>
__device__ __forceinline__ void store_row<float, 4>(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// Ring slot of absolute position p: p itself for a sink token, else a
// rotating slot among the `recent` ones.
__host__ __device__ __forceinline__ int ring_slot(int p, int sink, int recent) {
    return p < sink ? p : sink + (p - sink) % recent;
}

}  // namespace duo
