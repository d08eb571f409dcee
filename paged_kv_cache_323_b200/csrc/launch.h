// launch.h -- host-side entry points of the per-dtype decode translation units.
#pragma once

#include <cuda_runtime.h>

#include "decode_attn.cuh"

namespace pkv {

cudaError_t launch_decode_partition_f32(const DecodeParams& p, int D, int BS, int G, long long grid,
                                        cudaStream_t st);
cudaError_t launch_decode_partition_bf16(const DecodeParams& p, int D, int BS, int G,
                                         long long grid, cudaStream_t st);

}  // namespace pkv
