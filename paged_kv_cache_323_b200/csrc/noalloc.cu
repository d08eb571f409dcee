// noalloc.cu -- paged_attention_decode_noalloc: decode attention for callers
// that cannot allocate device memory.
//
// Who needs it: a serving engine usually sizes its KV-block pool to take all
// of the device memory left after the model weights, so nothing is free for a
// split-K workspace; some host frameworks only allow allocations through
// their own allocator, so that their memory accounting stays exact; and
// cudaMalloc / cudaFree may synchronise the device, which a latency-bound
// decode loop cannot afford.  This entry point takes the same inputs and
// outputs as paged_attention_decode_ex but keeps its split-K scratch (partial
// outputs, partial softmax sums and the merge counters) in one fixed-size
// array in device memory that is part of the library image: every GPU that
// loads the library holds PKV_NOALLOC_SCRATCH_BYTES for it until the process
// exits.  No call here allocates or frees memory.
//
// The host never uses the array's name as an address (in host code it is
// only a stand-in symbol): every call looks up the device address with
// cudaGetSymbolAddress, with the caller's device current.  The lookup
// allocates nothing, and doing it per call keeps the address right if the
// device is reset and a new context replaces the old one.  Every call shares
// the array and it keeps the previous call's contents, so each call clears
// the merge counters (the only part that must start at zero) with
// cudaMemsetAsync on its stream before the kernel runs.
// Two calls whose kernels overlap on the GPU -- on different streams, or on
// different host threads -- race on the array and corrupt each other's
// results; callers must order them.
#include <cuda_runtime.h>

#include <climits>

#include "../../include/pagedkv.h"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

// The device address of the scratch array on the current device.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return PKV_ERR_CUDA;
    }
    *out = p;
    return PKV_OK;
}

}  // namespace

// Defined in api.cu, not exported: the workspace size and the place of the
// merge counters for the partition size paged_attention_decode_ex picks.
extern "C" void pkv_internal_decode_scratch(int num_seqs, int num_heads, int num_kv_heads,
                                            int head_dim, int block_size, int max_blocks_per_seq,
                                            int dtype, int partition_tokens, size_t* total,
                                            size_t* cnt_off, size_t* cnt_bytes);

extern "C" PKV_API int paged_attention_decode_noalloc(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, float scale,
    int num_blocks, int dtype, int partition_tokens, void* stream) {
    if (num_seqs < 0) return PKV_ERR_INVALID;
    if (num_seqs == 0) return PKV_OK;
    if (num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        max_blocks_per_seq <= 0 || partition_tokens < 0)
        return PKV_ERR_INVALID;
    const long long max_ctx = (long long)max_blocks_per_seq * block_size;
    if (max_ctx > INT_MAX) return PKV_ERR_INVALID;
    size_t need = 0, cnt_off = 0, cnt_bytes = 0;
    pkv_internal_decode_scratch(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                max_blocks_per_seq, dtype, partition_tokens, &need, &cnt_off,
                                &cnt_bytes);
    // a batch whose split-K scratch exceeds the fixed array is refused, never truncated
    if (need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        const int rc = scratch_address(&scratch);
        if (rc != PKV_OK) return rc;
        if (cudaMemsetAsync(static_cast<char*>(scratch) + cnt_off, 0, cnt_bytes,
                            static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return PKV_ERR_CUDA;
    }
    return paged_attention_decode_ex(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                                     num_heads, num_kv_heads, head_dim, block_size,
                                     max_blocks_per_seq, scale, num_blocks, dtype, partition_tokens,
                                     scratch, need, stream);
}
