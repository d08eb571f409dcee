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

// A CTA of 256 threads covers 256 / chunks_per_row whole (token, kv head)
// rows, one thread per 16-byte chunk.  The new token's K and V chunks are
// loaded before the slot is known, so the only dependent step is the store.
__global__ void __launch_bounds__(256) kv_append_kernel(const AppendParams p) {
    // a decode launched next as a programmatic dependent may start now; it
    // waits for this grid to finish before it reads the pools
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int cpr = p.chunks_per_row;
    const int rows_per_cta = blockDim.x / cpr;
    const int r_in = threadIdx.x / cpr;
    const int ch = threadIdx.x - r_in * cpr;
    if (r_in >= rows_per_cta) return;
    const long long nrows = (long long)p.num_tokens * p.num_kv_heads;
    uint4* kc = static_cast<uint4*>(p.k_cache);
    uint4* vc = static_cast<uint4*>(p.v_cache);
    const uint4* kn = static_cast<const uint4*>(p.k);
    const uint4* vn = static_cast<const uint4*>(p.v);
    for (long long row = (long long)blockIdx.x * rows_per_cta + r_in; row < nrows;
         row += (long long)gridDim.x * rows_per_cta) {
        const long long x = row * cpr + ch;
        const uint4 kv = kn[x];
        const uint4 vv = vn[x];
        const long long i = row / p.num_kv_heads;
        const long long g = row - i * p.num_kv_heads;
        const long long slot = p.slot_mapping[i];
        if (slot < 0) continue;  // -1: nothing to write for this token
        if (slot >= p.num_slots) {
            if (ch == 0 && g == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            continue;
        }
        const long long blk = slot / p.block_size;
        const long long off = slot - blk * p.block_size;
        const long long dst = ((blk * p.num_kv_heads + g) * p.block_size + off) * cpr + ch;
        kc[dst] = kv;
        vc[dst] = vv;
    }
}

// Append with quantisation to fp8 e4m3 (per-kv-head scales): each thread
// writes one 16-byte chunk of codes (16 elements) of one (token, kv head)
// row from 32 bytes of bf16 input: code = e4m3(x / scale), the division
// correctly rounded in fp32, round-to-nearest-even and saturation to +-448
// in the conversion.
struct AppendFp8Params {
    void* k_cache;
    void* v_cache;
    const float* k_scales;
    const float* v_scales;
    const void* k;  // bf16 [T][Hkv][D]
    const void* v;
    const int64_t* slot_mapping;
    int* err;
    long long num_slots;
    int num_tokens;
    int num_kv_heads;
    int block_size;
    int chunks_per_row;  // head_dim / 16
};

__device__ __forceinline__ uint4 quantise16(const uint4 a, const uint4 b, float scale) {
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t packed = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t w = in[2 * i + h];  // two bf16 values
            const float x0 = __uint_as_float(w << 16);
            const float x1 = __uint_as_float(w & 0xffff0000u);
            const __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(
                make_float2(__fdiv_rn(x0, scale), __fdiv_rn(x1, scale)), __NV_SATFINITE, __NV_E4M3);
            packed |= (uint32_t)q << (16 * h);
        }
        out[i] = packed;
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void __launch_bounds__(256) kv_append_fp8_kernel(const AppendFp8Params p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // as in kv_append_kernel
    const int cpr = p.chunks_per_row;
    const int rows_per_cta = blockDim.x / cpr;
    const int r_in = threadIdx.x / cpr;
    const int ch = threadIdx.x - r_in * cpr;
    if (r_in >= rows_per_cta) return;
    const long long nrows = (long long)p.num_tokens * p.num_kv_heads;
    uint4* kc = static_cast<uint4*>(p.k_cache);
    uint4* vc = static_cast<uint4*>(p.v_cache);
    const uint4* kn = static_cast<const uint4*>(p.k);
    const uint4* vn = static_cast<const uint4*>(p.v);
    for (long long row = (long long)blockIdx.x * rows_per_cta + r_in; row < nrows;
         row += (long long)gridDim.x * rows_per_cta) {
        const long long x = (row * cpr + ch) * 2;  // two bf16 chunks per fp8 chunk
        const uint4 k0 = kn[x], k1 = kn[x + 1];
        const uint4 v0 = vn[x], v1 = vn[x + 1];
        const long long i = row / p.num_kv_heads;
        const long long g = row - i * p.num_kv_heads;
        const long long slot = p.slot_mapping[i];
        if (slot < 0) continue;  // -1: nothing to write for this token
        if (slot >= p.num_slots) {
            if (ch == 0 && g == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            continue;
        }
        const long long blk = slot / p.block_size;
        const long long off = slot - blk * p.block_size;
        const long long dst = ((blk * p.num_kv_heads + g) * p.block_size + off) * cpr + ch;
        kc[dst] = quantise16(k0, k1, p.k_scales[g]);
        vc[dst] = quantise16(v0, v1, p.v_scales[g]);
    }
}

struct CopyParams {
    void* dst_k;
    void* dst_v;
    const void* src_k;
    const void* src_v;
    const int64_t* pairs;
    int* err;
    long long chunks_per_block;  // num_kv_heads * block_size * head_dim * elt / 16
    int num_pairs;
    int num_src_blocks;
    int num_dst_blocks;
};

// One pair per gridDim.y row; gridDim.x CTAs share one pair's block, 4
// chunks per thread in flight for K and for V.  Serves copy-on-write (source
// and destination in the same device pool) and swapping (one side in a
// pinned host pool, reached through its device-mapped address).
__global__ void __launch_bounds__(256) copy_blocks_kernel(const CopyParams p) {
    const long long pair = blockIdx.x;  // blockIdx.y splits one pair's block
    const long long src = p.pairs[2 * pair];
    const long long dst = p.pairs[2 * pair + 1];
    if (src < 0 || src >= p.num_src_blocks || dst < 0 || dst >= p.num_dst_blocks) {
        if (blockIdx.y == 0 && threadIdx.x == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
        return;
    }
    const uint4* ks = static_cast<const uint4*>(p.src_k) + src * p.chunks_per_block;
    const uint4* vs = static_cast<const uint4*>(p.src_v) + src * p.chunks_per_block;
    uint4* kd = static_cast<uint4*>(p.dst_k) + dst * p.chunks_per_block;
    uint4* vd = static_cast<uint4*>(p.dst_v) + dst * p.chunks_per_block;
    constexpr int U = 4;
    const long long stride = (long long)gridDim.y * blockDim.x;
    for (long long base = blockIdx.y * (long long)blockDim.x + threadIdx.x; base < p.chunks_per_block;
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

// Self-test of the failure path: one warp waits, with the same bounded wait
// the kernels use, on an mbarrier that nothing ever arrives at.  The wait
// gives up after timeout_ns, records PKV_ERR_TIMEOUT and the kernel returns;
// no trap, and the context stays usable.
__global__ void bounded_wait_selftest_kernel(int* err, unsigned long long timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    const bool ok = mbar_wait_bounded(&bar, 0, &abort_flag, timeout_ns);
    if (!__all_sync(0xffffffffu, ok) && threadIdx.x == 0) set_error(err, PKV_ERR_TIMEOUT);
}

}  // namespace pkv
