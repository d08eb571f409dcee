// decode_common.cuh -- what the decode kernels share: the launch parameters,
// the fused split-K merge and the zero-row writer.  The CUDA-core kernel
// (decode_attn.cuh) and the tensor-core kernels (decode_tc.cuh,
// decode_tc_fp8.cuh) all end a partition through fused_merge.
#pragma once

#include <math.h>

#include "common.cuh"

namespace pkv {

struct DecodeParams {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_o;    // [B][H][P][D] unnormalised partial outputs
    float2* ws_ml;  // [B][H][P] (running max in log2 units, running sum)
    int* counters;  // [B][Hkv] partitions finished, zero between launches
    const float* k_scales;  // fp8 caches: per-kv-head dequantisation scales (else null)
    const float* v_scales;
    int* err;
    int num_seqs;
    int num_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int num_blocks;
    int partition_tokens;
    int num_partitions;  // partitions per sequence in the grid
    float qscale;        // scale * log2(e)
};

// Split-K merge, fused into the decode kernels: called by every thread of a
// partition CTA after the CTA wrote its (m, l, o) for the group's G heads to
// the workspace.  The last partition CTA of (s, g) to arrive -- found with
// one atomicInc on the group's counter, which wraps back to 0 on that arrival
// so the counters are zero again after every complete launch -- merges all
// partitions in partition order:
//     M = max_i m_i,  L = sum_i 2^(m_i - M) l_i,  out = sum_i 2^(m_i - M) o_i / L.
// `scratch` is shared memory of at least merge_scratch_bytes<G, D, NTHREADS>().
template <int G, int D, int NTHREADS>
constexpr int merge_scratch_bytes() {
    return ((2 * G + 3) / 4) * 16 + (NTHREADS > G * D / 4 ? NTHREADS : G * D / 4) * 16;
}

template <typename T, int D, int G, int NTHREADS>
__device__ __forceinline__ void fused_merge(const DecodeParams& p, int s, int g, int nparts,
                                            long long sh0, float* scratch, int* last_flag) {
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int P = p.num_partitions;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned old = atomicInc(
            reinterpret_cast<unsigned*>(p.counters) + (long long)s * p.num_kv_heads + g,
            (unsigned)(nparts - 1));
        *last_flag = old == (unsigned)(nparts - 1);
    }
    __syncthreads();
    if (!*last_flag) return;
    __threadfence();

    // per head: M = max_i m_i, L = sum_i 2^(m_i - M) l_i (one warp per head)
    float* red = scratch;  // [G][2]
    for (int hg = warp; hg < G; hg += NTHREADS / 32) {
        const float2* ml = p.ws_ml + (sh0 + hg) * P;
        float M = -INFINITY;
        for (int i = lane; i < nparts; i += 32) M = fmaxf(M, __ldcg(&ml[i]).x);
#pragma unroll
        for (int msk = 16; msk; msk >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, msk));
        float L = 0.f;
        if (M != -INFINITY) {
            for (int i = lane; i < nparts; i += 32) {
                const float2 v = __ldcg(&ml[i]);
                L = fmaf(exp2f(v.x - M), v.y, L);
            }
        }
#pragma unroll
        for (int msk = 16; msk; msk >>= 1) L += __shfl_xor_sync(0xffffffffu, L, msk);
        if (lane == 0) {
            red[2 * hg] = M;
            red[2 * hg + 1] = L;
        }
    }
    __syncthreads();
    // out = sum_i 2^(m_i - M) o_i / L, partitions split over thread groups
    constexpr int COLS = D / 4;
    constexpr int UNITS = G * COLS;
    constexpr int GROUPS = NTHREADS / UNITS > 0 ? NTHREADS / UNITS : 1;
    float4* acc_s = reinterpret_cast<float4*>(scratch + ((2 * G + 3) / 4) * 4);  // [GROUPS][UNITS]
    for (int u = tid; u < GROUPS * UNITS; u += NTHREADS) {
        const int unit = u % UNITS;
        const int grp = u / UNITS;
        const int hg = unit / COLS;
        const int col = unit % COLS;
        const float M = red[2 * hg];
        const float2* ml = p.ws_ml + (sh0 + hg) * P;
        const float4* o = reinterpret_cast<const float4*>(p.ws_o + (sh0 + hg) * P * D) + col;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
#pragma unroll 8
            for (int i = grp; i < nparts; i += GROUPS) {
                const float w = exp2f(__ldcg(&ml[i]).x - M);
                const float4 v = __ldcg(o + (long long)i * COLS);
                a.x = fmaf(w, v.x, a.x);
                a.y = fmaf(w, v.y, a.y);
                a.z = fmaf(w, v.z, a.z);
                a.w = fmaf(w, v.w, a.w);
            }
        }
        acc_s[grp * UNITS + unit] = a;
    }
    __syncthreads();
    for (int unit = tid; unit < UNITS; unit += NTHREADS) {
        const int hg = unit / COLS;
        const int col = unit % COLS;
        float4 t = acc_s[unit];
        for (int grp = 1; grp < GROUPS; ++grp) {
            const float4 v = acc_s[grp * UNITS + unit];
            t.x += v.x;
            t.y += v.y;
            t.z += v.z;
            t.w += v.w;
        }
        const float L = red[2 * hg + 1];
        const float inv = L > 0.f ? 1.f / L : 0.f;
        T* dst = static_cast<T*>(p.out) + (sh0 + hg) * D + col * 4;
        Elem<T>::store(dst + 0, t.x * inv);
        Elem<T>::store(dst + 1, t.y * inv);
        Elem<T>::store(dst + 2, t.z * inv);
        Elem<T>::store(dst + 3, t.w * inv);
    }
}

template <typename T, int D, int G>
__device__ __forceinline__ void zero_rows(const DecodeParams& p, int s, int g) {
    T* out = static_cast<T*>(p.out) + ((long long)s * p.num_heads + (long long)g * G) * D;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) Elem<T>::store(out + i, 0.f);
}

}  // namespace pkv
