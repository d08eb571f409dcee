// decode_reg.cu -- launch of the register-streamed decode kernel
// (decode_reg.cuh): bf16 caches, head_dim 64 or 128, one query head per kv
// head.
#include "decode_reg.cuh"
#include "launch.h"

namespace pkv {

namespace {
constexpr int kRegWarps = 4;  // warps per CTA
// CTAs per SM the registers are budgeted for: a chunk of 2 KB of K and V
// holds 4 x 16 bytes of each per lane (about 126 registers, 4 CTAs); the
// 1 KB chunks of head_dim 64 at block size 8 hold half that (80 registers,
// 6 CTAs), so more warps keep them in flight
template <int D, int BS>
constexpr int reg_min_blocks() {
    return RegCfg<D, BS, kRegWarps>::RPL >= 4 ? 4 : 6;
}

template <int D>
void (*reg_kernel(int BS))(const DecodeParams) {
    switch (BS) {
        case 8: return decode_reg_kernel<D, 8, kRegWarps, reg_min_blocks<D, 8>()>;
        case 16: return decode_reg_kernel<D, 16, kRegWarps, reg_min_blocks<D, 16>()>;
        case 32: return decode_reg_kernel<D, 32, kRegWarps, reg_min_blocks<D, 32>()>;
        default: return nullptr;
    }
}
}  // namespace

bool decode_reg_supported(int kv_dtype, int D, int BS, int G) {
    return kv_dtype == PKV_BF16 && (D == 64 || D == 128) && (BS == 8 || BS == 16 || BS == 32) && G == 1;
}

cudaError_t launch_decode_reg(const DecodeParams& p, int D, int BS, int G, long long grid, cudaStream_t st) {
    if (G != 1) return cudaErrorInvalidValue;
    void (*kern)(const DecodeParams) = D == 128 ? reg_kernel<128>(BS) : D == 64 ? reg_kernel<64>(BS) : nullptr;
    if (kern == nullptr) return cudaErrorInvalidValue;
    // every CTA waits for the preceding grid in decode_unit
    return launch_decode_kernel(kern, static_cast<unsigned>(grid), kRegWarps * 32, 0, st, true, p);
}

}  // namespace pkv
