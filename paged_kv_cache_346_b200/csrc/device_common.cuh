// Device-side helpers shared by the pagedkv kernels: element types, 16-byte
// vector conversions, mbarrier and bulk-copy (TMA) PTX wrappers, bounded
// waits and the device status word.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "pagedkv.h"

namespace pkv {

// Record PKV_DEV_* bits in the device status word (passed to every kernel).
__device__ __forceinline__ void flag(unsigned int* status, unsigned int bits) {
    atomicOr(status, bits);
}

// ~2 s at 2 GHz: no legitimate wait in these kernels comes near it.
constexpr long long kWaitCycles = 4000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of the barrier to complete, giving up after
// `limit` clock cycles; on giving up the status word gets PKV_DEV_TIMEOUT.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity,
                                                unsigned int* status, long long limit) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(a, parity)) {
        if (clock64() - t0 > limit) {
            flag(status, PKV_DEV_TIMEOUT);
            return false;
        }
    }
    return true;
}

// The kernels' waits: kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned int* status) {
    return mbar_wait_limit(bar, parity, status, kWaitCycles);
}

// After a wait gave up: wait again (bounded) for the copies of slices
// [from, to) of a ring of `stages` barriers, so none lands in shared memory
// after the CTA has left.  A copy that does not land even then could still
// write into a later CTA's shared memory on that SM: that is flagged
// PKV_DEV_DRAIN_TIMEOUT, beside the PKV_DEV_TIMEOUT of the waits themselves.
__device__ __forceinline__ void drain_ring(uint64_t* bars, int stages, int from, int to,
                                           unsigned int* status) {
    for (int k = from; k < to; ++k)
        if (!mbar_wait(bars + k % stages, (uint32_t)((k / stages) & 1), status))
            flag(status, PKV_DEV_DRAIN_TIMEOUT);
}

// 2^x by the hardware approximation (relative error about 2^-22; -inf -> 0,
// results below the smallest normal -> 0): softmax weights and rescale
// factors, which tolerate far more
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// L2 policy for data read exactly once (the K/V pages of a decode step).
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 1-D bulk copy global -> shared (TMA), completion counted on `bar` in bytes.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue / wait here until the previous kernel's memory is visible.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_primary() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---- element types --------------------------------------------------------

// FP8 E4M3 codes (one byte each), the storage of quantised pages.
struct E4M3 {
    uint8_t bits;
};

template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kPerVec = 4;  // elements per 16-byte vector
    static constexpr int kBytes = 4;
    __device__ __forceinline__ static void to_f32(const uint4& v, float* f) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static float from_f32(float x) { return x; }
    __device__ __forceinline__ static float load1(const float* p) { return *p; }
};

template <>
struct Elem<__half> {
    static constexpr int kPerVec = 8;
    static constexpr int kBytes = 2;
    __device__ __forceinline__ static void to_f32(const uint4& v, float* f) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
            float2 t = __half22float2(h);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
    __device__ __forceinline__ static __half from_f32(float x) { return __float2half_rn(x); }
    __device__ __forceinline__ static float load1(const __half* p) { return __half2float(*p); }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kPerVec = 8;
    static constexpr int kBytes = 2;
    __device__ __forceinline__ static void to_f32(const uint4& v, float* f) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // bf16 -> f32 is exact: the bf16 bits are the top half of the f32
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static __nv_bfloat16 from_f32(float x) {
        return __float2bfloat16_rn(x);
    }
    __device__ __forceinline__ static float load1(const __nv_bfloat16* p) {
        return __bfloat162float(*p);
    }
};

template <>
struct Elem<E4M3> {
    static constexpr int kPerVec = 16;
    static constexpr int kBytes = 1;
    // 16 codes -> 16 floats (exact: every E4M3 value is a binary16 value)
    __device__ __forceinline__ static void to_f32(const uint4& v, float* f) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(
                    (__nv_fp8x2_storage_t)((w[i] >> (16 * j)) & 0xffffu), __NV_E4M3);
                const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&r));
                f[4 * i + 2 * j] = t.x;
                f[4 * i + 2 * j + 1] = t.y;
            }
        }
    }
};

}  // namespace pkv
