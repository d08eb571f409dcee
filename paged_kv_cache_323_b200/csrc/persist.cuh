// persist.cuh -- what the persistent decode kernels share: the queue's
// unit order, a warp's zero rows, and the named barrier of the four softmax
// warps.
#pragma once

#include "decode_common.cuh"

namespace pkv {
namespace tc {

// Unit u of the queue: with a longest-first schedule (p.order) pair
// order[u / Hkv] and kv head u % Hkv, so the longest units go first and the
// empty ones last; without one, index order (B x Hkv x P, partition fastest).
// Returns false (debug builds) for a schedule entry out of range.
__device__ __forceinline__ bool queue_unit(const DecodeParams& p, int u, int& s, int& g, int& part) {
    const int P = p.num_partitions;
    if (p.order != nullptr) {
        const int2 e = p.order[u / p.num_kv_heads];
        g = u % p.num_kv_heads;
        s = e.x / P;
        part = e.x % P;
    } else {
        part = u % P;
        g = (u / P) % p.num_kv_heads;
        s = u / (P * p.num_kv_heads);
    }
    return PKV_DCHECK(p.err, s >= 0 && s < p.num_seqs && part >= 0 && part < P);
}

// A unit's index in index order (partition fastest), and back.
__device__ __forceinline__ int unit_index(const DecodeParams& p, int s, int g, int part) {
    return (s * p.num_kv_heads + g) * p.num_partitions + part;
}

__device__ __forceinline__ void index_unit(const DecodeParams& p, int idx, int& s, int& g, int& part) {
    const int P = p.num_partitions;
    part = idx % P;
    g = (idx / P) % p.num_kv_heads;
    s = idx / (P * p.num_kv_heads);
}

// Zero G output rows from row sh0 with the lanes of one warp.
template <int G>
__device__ __forceinline__ void zero_rows_warp(const DecodeParams& p, long long sh0, int lane) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + sh0 * 128;
    for (int i = lane; i < G * 128; i += 32) out[i] = __float2bfloat16_rn(0.f);
}

// Named barrier 1 over the four softmax warps (128 threads): a plain
// barrier, and one that also returns whether every thread passed true.
__device__ __forceinline__ void soft_bar_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ bool soft_bar_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

}  // namespace tc
}  // namespace pkv
