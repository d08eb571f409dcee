// launch.h -- host-side entry points of the per-dtype decode translation units.
#pragma once

#include <cuda_runtime.h>

#include "decode_attn.cuh"

namespace pkv {

cudaError_t launch_decode_partition_f32(const DecodeParams& p, int D, int BS, int G, long long grid,
                                        cudaStream_t st);
cudaError_t launch_decode_partition_bf16(const DecodeParams& p, int D, int BS, int G,
                                         long long grid, cudaStream_t st);
// fp8 (e4m3) caches, bf16 q and out, per-kv-head scales in p.k_scales / p.v_scales
cudaError_t launch_decode_partition_fp8(const DecodeParams& p, int D, int BS, int G,
                                        long long grid, cudaStream_t st);

// Tensor-core (tcgen05) kernel for grouped-query heads: bf16, head_dim 128,
// groups of 2, 4 or 8, partitions a multiple of 128 tokens.
bool decode_tc_supported(int dtype, int D, int BS, int G, int partition_tokens);
cudaError_t launch_decode_tc(const DecodeParams& p, int BS, int G, long long grid, cudaStream_t st);

}  // namespace pkv
