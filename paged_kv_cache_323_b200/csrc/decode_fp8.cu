// decode_fp8.cu -- instantiations of the CUDA-core decode kernel for fp8
// (e4m3) K/V caches with bf16 q and out.
#include "decode_launch.cuh"
#include "launch.h"

namespace pkv {

cudaError_t launch_decode_partition_fp8(const DecodeParams& p, int D, int BS, int G,
                                        long long grid, cudaStream_t st) {
    return dispatch_partition<__nv_bfloat16, __nv_fp8_e4m3>(p, D, BS, G, grid, st);
}

}  // namespace pkv
