// decode_bf16.cu -- bf16 instantiations of the paged decode kernels.
#include "decode_launch.cuh"
#include "launch.h"

namespace pkv {

cudaError_t launch_decode_partition_bf16(const DecodeParams& p, int D, int BS, int G,
                                         long long grid, cudaStream_t st) {
    return dispatch_partition<__nv_bfloat16>(p, D, BS, G, grid, st);
}

}  // namespace pkv
