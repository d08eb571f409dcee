// decode_common.cuh -- what the decode kernels share: the launch parameters,
// the fused split-K merge and the zero-row writer.  The CUDA-core kernel
// (decode_attn.cuh) and the tensor-core kernels (decode_tc.cuh,
// decode_tc_fp8.cuh) all end a partition through fused_merge.
#pragma once

#include <math.h>

#include <utility>

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
    // persistent kernels' work queue: [0] next unit, [1] CTAs done; zero
    // between launches (the last CTA of a launch resets both)
    int* work;
    // longest-first schedule written by plan_kernel just before this launch
    // ([B * P] entries {s * P + part, context length of s}), or null for
    // index order
    const int2* order;
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
    // limit of the pipeline's bounded waits (ns of %globaltimer); the drain
    // after an abort always waits up to kWaitTimeoutNs
    unsigned long long wait_ns;
};

// Launch a decode kernel, as a programmatic dependent launch when `pdl`: its
// CTAs may start while the preceding grid (the planning grid, or the append
// of the same step, which releases its dependents at once) still runs, and
// wait for it (griddepcontrol.wait) before they read anything.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_decode_kernel(void (*kern)(KArgs...), unsigned grid, unsigned threads,
                                        size_t smem, cudaStream_t st, bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Which (sequence, kv head, partition) this CTA runs.  The CTA first waits
// for the grid its launch depends on (the planning grid or the step's
// append; a no-op when the launch depends on none), then, with a schedule
// (p.order), takes pair order[b / Hkv] and kv head b % Hkv.  Without one: partition fastest, or, when `partition_major` (the
// tensor-core kernels with at most 4 partitions per sequence), all first
// partitions, then all second ones, and so on.
struct Unit {
    int s, g, part, ctx;  // ctx: the sequence's context length
};

// `Hkv` is the number of head units per sequence: the kv heads, or the kv
// head pairs of the head_dim-64 tensor-core kernel (unit g = pair g).
__device__ __forceinline__ Unit decode_unit(const DecodeParams& p, bool partition_major, int Hkv) {
    const int P = p.num_partitions;
    const long long bid = blockIdx.x;
    Unit u;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (p.order != nullptr) {
        const int2 e = p.order[bid / Hkv];
        u.g = (int)(bid % Hkv);
        u.s = e.x / P;
        u.part = e.x % P;
        u.ctx = e.y;
    } else if (partition_major) {
        const long long units = (long long)p.num_seqs * Hkv;
        u.part = (int)(bid / units);
        u.g = (int)((bid % units) % Hkv);
        u.s = (int)((bid % units) / Hkv);
    } else {
        u.part = (int)(bid % P);
        u.g = (int)((bid / P) % Hkv);
        u.s = (int)(bid / ((long long)P * Hkv));
    }
    if (!PKV_DCHECK(p.err, u.s >= 0 && u.s < p.num_seqs && u.g >= 0 && u.g < Hkv && u.part >= 0 &&
                               u.part < P))
        u.s = -1;  // the CTA exits
    else if (p.order == nullptr)
        u.ctx = p.context_lens[u.s];
    return u;
}

__device__ __forceinline__ Unit decode_unit(const DecodeParams& p, bool partition_major) {
    return decode_unit(p, partition_major, p.num_kv_heads);
}

// Split-K merge, fused into the decode kernels: called by every thread of a
// partition CTA after the CTA wrote its (m, l, o) for the group's G heads to
// the workspace.  The last partition CTA of (s, g) to arrive -- found with
// one atomicInc on the group's counter, which wraps back to 0 on that arrival
// so the counters are zero again after every complete launch -- merges all
// partitions in partition order:
//     M = max_i m_i,  L = sum_i 2^(m_i - M) l_i,  out = sum_i 2^(m_i - M) o_i / L.
// `scratch` is shared memory of at least merge_scratch_bytes<G, D, NTHREADS>().
// The partitions are split over thread groups of a fixed 128-thread budget
// (kMergeLanes), whatever the caller's thread count, so every kernel -- one
// CTA per unit or persistent -- sums them in the same order and gives the
// same bits.
constexpr int kMergeLanes = 128;
template <int G, int D, int NTHREADS>
constexpr int merge_scratch_bytes() {
    return ((2 * G + 3) / 4) * 16 + (kMergeLanes > G * D / 4 ? kMergeLanes : G * D / 4) * 16;
}

// The merge itself, for the NTHREADS threads that call it: tid is the
// caller's index among them and sync() a barrier over exactly those threads,
// which returns false when it could not complete (a bounded wait that ran
// out); the merge then returns false too.
template <typename T, int D, int G, int NTHREADS, class Sync>
__device__ __forceinline__ bool fused_merge_with(const DecodeParams& p, int s, int g, int nparts,
                                                 long long sh0, float* scratch, int* last_flag,
                                                 int tid, Sync&& sync) {
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int P = p.num_partitions;
    __threadfence();
    if (!sync()) return false;
    if (tid == 0) {
        *last_flag = 0;
        if (PKV_DCHECK(p.err, nparts <= P && (long long)s * p.num_kv_heads + g <
                                                 (long long)p.num_seqs * p.num_kv_heads)) {
            const unsigned old = atomicInc(
                reinterpret_cast<unsigned*>(p.counters) + (long long)s * p.num_kv_heads + g,
                (unsigned)(nparts - 1));
            *last_flag = old == (unsigned)(nparts - 1);
        }
    }
    if (!sync()) return false;
    if (!*last_flag) return true;
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
    if (!sync()) return false;
    // out = sum_i 2^(m_i - M) o_i / L, partitions split over thread groups
    constexpr int COLS = D / 4;
    constexpr int UNITS = G * COLS;
    constexpr int GROUPS = kMergeLanes / UNITS > 0 ? kMergeLanes / UNITS : 1;
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
    if (!sync()) return false;
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
        if (!PKV_DCHECK(p.err, sh0 + hg < (long long)p.num_seqs * p.num_heads)) continue;
        T* dst = static_cast<T*>(p.out) + (sh0 + hg) * D + col * 4;
        Elem<T>::store(dst + 0, t.x * inv);
        Elem<T>::store(dst + 1, t.y * inv);
        Elem<T>::store(dst + 2, t.z * inv);
        Elem<T>::store(dst + 3, t.w * inv);
    }
    return true;
}

// The fused merge for a whole CTA (all NTHREADS threads, __syncthreads).
template <typename T, int D, int G, int NTHREADS>
__device__ __forceinline__ void fused_merge(const DecodeParams& p, int s, int g, int nparts,
                                            long long sh0, float* scratch, int* last_flag) {
    fused_merge_with<T, D, G, NTHREADS>(p, s, g, nparts, sh0, scratch, last_flag, (int)threadIdx.x,
                                        [] {
                                            __syncthreads();
                                            return true;
                                        });
}

// Zero the G output rows of D values from query head row sh0 (= s * H + the
// CTA's first query head) on.
template <typename T, int D, int G>
__device__ __forceinline__ void zero_rows(const DecodeParams& p, long long sh0) {
    T* out = static_cast<T*>(p.out) + sh0 * D;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) Elem<T>::store(out + i, 0.f);
}

// The end of a partition CTA whose bounded wait ran out (called by every
// thread, after the CTA's own copies and MMAs have landed).  It still takes
// its one turn on the (s, g) merge counter, so the counter wraps back to zero
// exactly as on a complete launch and the workspace stays valid for later
// calls: it posts an empty partial (m = -inf, l = 0, o = 0), which the merge
// weighs by zero, and if it arrives last it writes zero rows instead of
// merging.  A sequence with one partition has no counter; its rows are
// zeroed.  The outputs of a launch that timed out are not meaningful, but
// they are finite and the error word says PKV_ERR_TIMEOUT.
template <typename T, int D, int G>
__device__ __forceinline__ void abort_merge_turn(const DecodeParams& p, int s, int g, long long sh0,
                                                 int part, int nparts, int* last_flag) {
    if (nparts == 1) {
        zero_rows<T, D, G>(p, sh0);
        return;
    }
    const int P = p.num_partitions;
    if (!PKV_DCHECK(p.err, part < P && sh0 + G <= (long long)p.num_seqs * p.num_heads)) return;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x)
        p.ws_o[((sh0 + i / D) * P + part) * D + i % D] = 0.f;
    if (threadIdx.x < G) p.ws_ml[(sh0 + threadIdx.x) * P + part] = make_float2(-INFINITY, 0.f);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned old = atomicInc(
            reinterpret_cast<unsigned*>(p.counters) + (long long)s * p.num_kv_heads + g,
            (unsigned)(nparts - 1));
        *last_flag = old == (unsigned)(nparts - 1);
    }
    __syncthreads();
    if (*last_flag) zero_rows<T, D, G>(p, sh0);
}

}  // namespace pkv
