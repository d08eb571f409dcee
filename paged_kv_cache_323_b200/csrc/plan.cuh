// plan.cuh -- the longest-first schedule of a decode grid.
//
// A decode launch has one CTA per (sequence, kv head, partition), and the
// hardware hands CTAs to SMs in index order as slots free up.  With context
// lengths that vary (the pages' serving batches: "PagedAttention Explained:
// Virtual Memory for the KV Cache", section "The problem: the KV cache is big
// and unpredictable"), index order leaves the longest partitions wherever
// their sequences happen to sit, and the last of them run alone at the end of
// the launch while most of the GPU idles.  Handing out the longest work first
// removes that tail (list scheduling in decreasing order).
//
// plan_kernel sorts the launch's (sequence, partition) pairs by token count,
// longest first, into `order` (one entry {s * P + part, context length of s}
// per pair, P partitions per sequence in the grid); the decode kernel's CTA b
// then runs pair order[b / Hkv] for kv head b % Hkv, so the kv heads of a pair
// stay adjacent.  The entry carries the context length so that a CTA needs
// one dependent load, as without a schedule, before it reads its table.
// Counts are bucketed in kPlanQuantum-token steps (a counting sort); within a
// bucket the order is that of the atomics.  static_assert below: the bucket
// scan covers every bucket.  The schedule changes which SM runs
// a unit and when, never what it computes or the order of any reduction, so
// outputs are bit-identical under every schedule.  One CTA; it lets the
// decode grid launch at once (programmatic dependent launch), and the decode
// CTAs wait for it (griddepcontrol.wait) before they read the order.
#pragma once

#include "common.cuh"

namespace pkv {

constexpr int kPlanThreads = 1024;
constexpr int kPlanQuantum = 64;  // tokens per length bucket
constexpr int kPlanBuckets = 4096 / kPlanQuantum + 1;
constexpr int kPlanKept = 8;      // pairs per thread whose buckets stay in registers
static_assert(kPlanBuckets <= 3 * 32, "warp 0 scans three buckets per lane");

// Length bucket of pair `pair` (sequence pair / P, partition pair % P): its
// tokens in kPlanQuantum steps, 0 past the sequence's end and for a context
// length the decode kernel rejects.
__device__ __forceinline__ int plan_bucket(int ctx, long long pair, int P, int PT, int max_ctx) {
    const int part = (int)(pair % P);
    int len = (ctx < 0 || ctx > max_ctx) ? 0 : ctx - part * PT;
    len = len < 0 ? 0 : (len > PT ? PT : len);
    return (len + kPlanQuantum - 1) / kPlanQuantum;
}

__global__ void __launch_bounds__(kPlanThreads)
    plan_kernel(const int32_t* context_lens, int num_seqs, int P, int PT, int max_ctx, int2* order,
                int* err) {
    // the decode grid may launch now; its CTAs wait for this grid to finish
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int count[kPlanBuckets];
    __shared__ int next[kPlanBuckets];
    const int tid = threadIdx.x;
    for (int b = tid; b < kPlanBuckets; b += kPlanThreads) count[b] = 0;
    __syncthreads();
    const long long n = (long long)num_seqs * P;
    // count: the first kPlanKept * 1024 pairs keep their buckets in registers
    // (their context lengths are loaded once, all in flight together)
    int kept[kPlanKept], kept_ctx[kPlanKept];
#pragma unroll
    for (int k = 0; k < kPlanKept; ++k) {
        const long long i = tid + (long long)k * kPlanThreads;
        kept_ctx[k] = i < n ? context_lens[i / P] : 0;
    }
#pragma unroll
    for (int k = 0; k < kPlanKept; ++k) {
        const long long i = tid + (long long)k * kPlanThreads;
        kept[k] = i < n ? plan_bucket(kept_ctx[k], i, P, PT, max_ctx) : -1;
        if (kept[k] >= 0) atomicAdd(&count[kept[k]], 1);
    }
    for (long long i = tid + (long long)kPlanKept * kPlanThreads; i < n; i += kPlanThreads)
        atomicAdd(&count[plan_bucket(context_lens[i / P], i, P, PT, max_ctx)], 1);
    __syncthreads();
    // first slot of each bucket, longest bucket first: warp 0 scans the
    // buckets in descending order, three per lane
    if (tid < 32) {
        int c[3], sum = 0;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int b = kPlanBuckets - 1 - (3 * tid + k);
            c[k] = b >= 0 ? count[b] : 0;
            sum += c[k];
        }
        int incl = sum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, d);
            if (tid >= d) incl += v;
        }
        int run = incl - sum;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int b = kPlanBuckets - 1 - (3 * tid + k);
            if (b >= 0) next[b] = run;
            run += c[k];
        }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kPlanKept; ++k) {
        if (kept[k] < 0) continue;
        const int pos = atomicAdd(&next[kept[k]], 1);
        if (PKV_DCHECK(err, pos >= 0 && pos < n))
            order[pos] = make_int2(tid + k * kPlanThreads, kept_ctx[k]);
    }
    for (long long i = tid + (long long)kPlanKept * kPlanThreads; i < n; i += kPlanThreads) {
        const int ctx = context_lens[i / P];
        const int pos = atomicAdd(&next[plan_bucket(ctx, i, P, PT, max_ctx)], 1);
        if (PKV_DCHECK(err, pos >= 0 && pos < n)) order[pos] = make_int2((int)i, ctx);
    }
}

}  // namespace pkv
