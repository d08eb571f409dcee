// decode_reg.cu -- launch of the register-streamed decode kernel
// (decode_reg.cuh): bf16 caches, head_dim 128, one query head per kv head.
#include "decode_reg.cuh"
#include "launch.h"

namespace pkv {

namespace {
constexpr int kRegWarps = 4;      // warps per CTA
constexpr int kRegMinBlocks = 4;  // CTAs per SM the registers are budgeted for
}  // namespace

bool decode_reg_supported(int kv_dtype, int D, int BS, int G) {
    return kv_dtype == PKV_BF16 && D == 128 && (BS == 8 || BS == 16 || BS == 32) && G == 1;
}

cudaError_t launch_decode_reg(const DecodeParams& p, int D, int BS, int G, long long grid, cudaStream_t st) {
    if (D != 128 || G != 1) return cudaErrorInvalidValue;
    void (*kern)(const DecodeParams) = nullptr;
    switch (BS) {
        case 8: kern = decode_reg_kernel<128, 8, kRegWarps, kRegMinBlocks>; break;
        case 16: kern = decode_reg_kernel<128, 16, kRegWarps, kRegMinBlocks>; break;
        case 32: kern = decode_reg_kernel<128, 32, kRegWarps, kRegMinBlocks>; break;
        default: return cudaErrorInvalidValue;
    }
    // every CTA waits for the preceding grid in decode_unit
    return launch_decode_kernel(kern, static_cast<unsigned>(grid), kRegWarps * 32, 0, st, true, p);
}

}  // namespace pkv
