// decode_f32.cu -- fp32 instantiations of the paged decode kernels.
#include "decode_launch.cuh"
#include "launch.h"

namespace pkv {

cudaError_t launch_decode_partition_f32(const DecodeParams& p, int D, int BS, int G, long long grid,
                                        cudaStream_t st) {
    return dispatch_partition<float>(p, D, BS, G, grid, st);
}

}  // namespace pkv
