// kv_ops.cuh -- the two write kernels of the paged cache (sm_100a):
//
//  * append: "PagedAttention Explained: Virtual Memory for the KV Cache",
//    section "The problem: the KV cache is big and unpredictable" -- the cache
//    grows by one entry per new token.  New token i's K and V rows (every kv
//    head) are stored at physical slot slot_mapping[i] (block slot / bs,
//    offset slot % bs) of the [block][kv_head][slot][dim] pools.
//  * copy_blocks: same page, section "Sharing blocks between sequences" --
//    before a sequence writes into a shared block, the block is copied and
//    the writer's table is pointed at the copy (copy-on-write).
//
// Both are pure bandwidth kernels: 16-byte vector loads and stores, grid
// stride over 16-byte chunks, bit-exact.  Out-of-range slots or block indices
// set the device error word and are skipped.
#pragma once

#include "common.cuh"

namespace pkv {

struct AppendParams {
    void* k_cache;
    void* v_cache;
    const void* k;
    const void* v;
    const int64_t* slot_mapping;
    int* err;
    long long num_slots;  // num_blocks * block_size
    int num_tokens;
    int num_kv_heads;
    int block_size;
    int chunks_per_row;  // head_dim * elt / 16
};

// One thread per 16-byte chunk of one (token, kv head) row, K and V.
__global__ void __launch_bounds__(256) kv_append_kernel(const AppendParams p) {
    const long long per_token = (long long)p.num_kv_heads * p.chunks_per_row;
    const long long total = (long long)p.num_tokens * per_token;
    uint4* kc = static_cast<uint4*>(p.k_cache);
    uint4* vc = static_cast<uint4*>(p.v_cache);
    const uint4* kn = static_cast<const uint4*>(p.k);
    const uint4* vn = static_cast<const uint4*>(p.v);
    for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < total;
         x += (long long)gridDim.x * blockDim.x) {
        const long long i = x / per_token;
        const long long rem = x - i * per_token;  // g * chunks_per_row + chunk
        const long long slot = p.slot_mapping[i];
        if (slot < 0) continue;  // -1: nothing to write for this token
        if (slot >= p.num_slots) {
            if (rem == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            continue;
        }
        const long long blk = slot / p.block_size;
        const long long off = slot - blk * p.block_size;
        const long long g = rem / p.chunks_per_row;
        const long long ch = rem - g * p.chunks_per_row;
        const long long dst = ((blk * p.num_kv_heads + g) * p.block_size + off) * p.chunks_per_row + ch;
        kc[dst] = kn[x];
        vc[dst] = vn[x];
    }
}

struct CopyParams {
    void* k_cache;
    void* v_cache;
    const int64_t* pairs;
    int* err;
    long long chunks_per_block;  // num_kv_heads * block_size * head_dim * elt / 16
    int num_pairs;
    int num_blocks;
};

// gridDim.y = pairs; gridDim.x CTAs share one pair's block, 4 chunks per
// thread in flight for K and for V.
__global__ void __launch_bounds__(256) copy_blocks_kernel(const CopyParams p) {
    const int pair = blockIdx.y;
    const long long src = p.pairs[2 * pair];
    const long long dst = p.pairs[2 * pair + 1];
    if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
        return;
    }
    const uint4* ks = static_cast<const uint4*>(p.k_cache) + src * p.chunks_per_block;
    const uint4* vs = static_cast<const uint4*>(p.v_cache) + src * p.chunks_per_block;
    uint4* kd = static_cast<uint4*>(p.k_cache) + dst * p.chunks_per_block;
    uint4* vd = static_cast<uint4*>(p.v_cache) + dst * p.chunks_per_block;
    constexpr int U = 4;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long base = blockIdx.x * (long long)blockDim.x + threadIdx.x; base < p.chunks_per_block;
         base += stride * U) {
        uint4 kr[U], vr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long x = base + u * stride;
            if (x < p.chunks_per_block) {
                kr[u] = ks[x];
                vr[u] = vs[x];
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long x = base + u * stride;
            if (x < p.chunks_per_block) {
                kd[x] = kr[u];
                vd[x] = vr[u];
            }
        }
    }
}

}  // namespace pkv
