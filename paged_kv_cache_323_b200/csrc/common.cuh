// common.cuh -- device helpers shared by the sm_100a kernels of libpagedkv:
// mbarrier and bulk-copy (TMA engine) wrappers in inline PTX, bounded waits,
// the device error word, and element conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pagedkv.h"

namespace pkv {

// A bounded wait gives up after this many nanoseconds of %globaltimer.  A
// legitimate wait in these kernels lasts microseconds.
constexpr unsigned long long kWaitTimeoutNs = 1000000000ull;

// Record the first device fault of the current run; later ones are dropped.
__device__ __forceinline__ void set_error(int* err, int code) {
    if (err != nullptr) atomicCAS(err, 0, code);
}

// Debug builds (-DPKV_DEBUG) check every index derived from the inputs
// (schedule entries, units, copy sources and destinations, workspace and
// output rows) right before its use: a failed check records
// PKV_ERR_DEVICE_BOUNDS in err[0] and the source line in err[1] (the first
// failure wins), and the caller skips the access, so the build reports a
// bad index where a release build would read or write out of bounds.  In
// release builds PKV_DCHECK is the constant true and compiles away.
#ifdef PKV_DEBUG
static __device__ __noinline__ void debug_fail(int* err, int line) {
    if (err != nullptr) {
        atomicCAS(err, 0, PKV_ERR_DEVICE_BOUNDS);
        atomicCAS(err + 1, 0, line);
    }
}
#define PKV_DCHECK(err, cond) ((cond) ? true : (::pkv::debug_fail((err), __LINE__), false))
#else
#define PKV_DCHECK(err, cond) true
#endif

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_addr(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Returns
// false (without completing) when *abort becomes non-zero or the wait passes
// kWaitTimeoutNs; the caller then records the fault and winds down.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  const volatile int* abort,
                                                  unsigned long long timeout_ns = kWaitTimeoutNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// ------------------------------------------------- bulk copy (TMA engine)
// One contiguous global -> shared copy of `bytes` (a multiple of 16; both
// addresses 16-byte aligned), completing on `bar` as transaction bytes.  No
// multicast: the destination is this CTA's own shared memory.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// ------------------------------------------------------- element types
template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kPer16B = 4;
    static constexpr pkv_dtype kCode = PKV_F32;
    // 16 bytes -> 4 floats
    static __device__ __forceinline__ void unpack(const uint4& r, float* f) {
        f[0] = __uint_as_float(r.x);
        f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z);
        f[3] = __uint_as_float(r.w);
    }
    static __device__ __forceinline__ void store(float* dst, float v) { *dst = v; }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kPer16B = 8;
    static constexpr pkv_dtype kCode = PKV_BF16;
    // 16 bytes -> 8 floats.  A bf16 is the top half of a binary32, so the
    // widening is a shift (low element) or a mask (high element), exactly.
    static __device__ __forceinline__ void unpack(const uint4& r, float* f) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* dst, float v) {
        *dst = __float2bfloat16_rn(v);
    }
};

// fp8 e4m3 cache elements (stored value = code * per-kv-head scale).
template <>
struct Elem<__nv_fp8_e4m3> {
    static constexpr int kPer16B = 16;
    // 16 bytes -> 16 floats, each code widened exactly (e4m3 -> f16 -> f32)
    static __device__ __forceinline__ void unpack(const uint4& r, float* f) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                    (__nv_fp8x2_storage_t)((w[i] >> (16 * h)) & 0xffffu), __NV_E4M3);
                const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&hr));
                f[4 * i + 2 * h] = f2.x;
                f[4 * i + 2 * h + 1] = f2.y;
            }
        }
    }
};

}  // namespace pkv
