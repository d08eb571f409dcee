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
// longest first, into `order` (one entry s * P + part per pair, P partitions
// per sequence in the grid); the decode kernel's CTA b then runs pair
// order[b / Hkv] for kv head b % Hkv, so the kv heads of a pair stay adjacent.
// Counts are bucketed in kPlanQuantum-token steps (a counting sort); within a
// bucket the order is that of the atomics.  The schedule changes which SM runs
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

// Tokens of partition `part` of a sequence of `ctx` tokens (0 past its end,
// and 0 for a context length the decode kernel rejects).
__device__ __forceinline__ int plan_bucket(const int32_t* context_lens, long long pair, int P,
                                           int PT, int max_ctx) {
    const int s = (int)(pair / P), part = (int)(pair % P);
    const int ctx = context_lens[s];
    int len = (ctx < 0 || ctx > max_ctx) ? 0 : ctx - part * PT;
    len = len < 0 ? 0 : (len > PT ? PT : len);
    return (len + kPlanQuantum - 1) / kPlanQuantum;
}

__global__ void __launch_bounds__(kPlanThreads)
    plan_kernel(const int32_t* context_lens, int num_seqs, int P, int PT, int max_ctx, int* order,
                int* err) {
    // the decode grid may launch now; its CTAs wait for this grid to finish
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int count[kPlanBuckets];
    __shared__ int next[kPlanBuckets];
    for (int b = threadIdx.x; b < kPlanBuckets; b += blockDim.x) count[b] = 0;
    __syncthreads();
    const long long n = (long long)num_seqs * P;
    for (long long i = threadIdx.x; i < n; i += blockDim.x)
        atomicAdd(&count[plan_bucket(context_lens, i, P, PT, max_ctx)], 1);
    __syncthreads();
    if (threadIdx.x == 0) {  // first slot of each bucket, longest bucket first
        int run = 0;
        for (int b = kPlanBuckets - 1; b >= 0; --b) {
            next[b] = run;
            run += count[b];
        }
    }
    __syncthreads();
    for (long long i = threadIdx.x; i < n; i += blockDim.x) {
        const int b = plan_bucket(context_lens, i, P, PT, max_ctx);
        const int pos = atomicAdd(&next[b], 1);
        if (PKV_DCHECK(err, pos >= 0 && pos < n)) order[pos] = (int)i;
    }
}

}  // namespace pkv
