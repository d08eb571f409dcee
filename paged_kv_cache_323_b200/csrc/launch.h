// launch.h -- host-side entry points of the per-dtype decode translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "decode_common.cuh"

namespace pkv {

cudaError_t launch_decode_partition_f32(const DecodeParams& p, int D, int BS, int G, long long grid,
                                        cudaStream_t st);
cudaError_t launch_decode_partition_bf16(const DecodeParams& p, int D, int BS, int G,
                                         long long grid, cudaStream_t st);
// fp8 (e4m3) caches, bf16 q and out, per-kv-head scales in p.k_scales / p.v_scales
cudaError_t launch_decode_partition_fp8(const DecodeParams& p, int D, int BS, int G,
                                        long long grid, cudaStream_t st);

// bf16 MHA over 8-token blocks, head_dim 128: K and V streamed through
// registers with plain loads instead of staged copies
bool decode_reg_supported(int kv_dtype, int D, int BS, int G);
cudaError_t launch_decode_reg(const DecodeParams& p, int D, int BS, int G, long long grid, cudaStream_t st);

// Tensor-core (tcgen05) kernels, partitions a multiple of 128 tokens: bf16
// caches with head_dim 128 and groups of 2, 4 or 8 query heads; fp8 (e4m3)
// caches with head_dim 128 and groups of 1, 2, 4 or 8, or head_dim 64, an
// even number of kv heads (one CTA per pair) and groups of 1, 2 or 4.
bool decode_tc_supported(int kv_dtype, int D, int BS, int G, int Hkv, int partition_tokens);
// persistent: the fp8 kernel that takes its units from the work queue in
// p.work, in the order of the schedule p.order when there is one (needs a
// workspace and decode_tc_fp8_persistent_supported: 1, 2 or 4 query heads per
// kv head, partitions of at most decode_tc_fp8_persistent_max_tokens(BS))
cudaError_t launch_decode_tc(const DecodeParams& p, int kv_dtype, int D, int BS, int G, long long grid,
                             bool persistent, cudaStream_t st);
bool decode_tc_fp8_persistent_supported(int BS, int G, int partition_tokens);
int decode_tc_fp8_persistent_max_tokens(int BS);
// internal to the tensor-core translation units
void* tc_tensor_map_encoder();  // cuTensorMapEncodeTiled, or null
cudaError_t launch_decode_tc_fp8_d64(const DecodeParams& p, int BS, int G, cudaStream_t st);
cudaError_t make_tc_pool_map(CUtensorMap* map, const void* pool, int Hkv, int BS, int num_blocks,
                             int elem_bytes);
cudaError_t launch_decode_tc_fp8(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                                 int BS, int G, long long grid, cudaStream_t st);
cudaError_t launch_decode_tc_fp8_persistent(const DecodeParams& p, const CUtensorMap& mk,
                                            const CUtensorMap& mv, int BS, int G, long long units,
                                            cudaStream_t st);

}  // namespace pkv
