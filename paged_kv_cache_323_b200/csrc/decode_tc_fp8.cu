// decode_tc_fp8.cu -- launches of the tensor-core decode kernel over fp8
// (e4m3) pools, dispatched over (block_size, group size).
#include <atomic>

#include "decode_tc_fp8.cuh"
#include "launch.h"

namespace pkv {
namespace {

template <int BS, int G>
cudaError_t launch_inst(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                        long long grid, cudaStream_t st) {
    using C = tc::TcFp8Cfg<BS, G>;
    auto kern = tc::decode_tc_fp8_kernel<BS, G>;
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit);
    }
    // one CTA per unit: every CTA waits for the preceding grid in decode_unit
    return launch_decode_kernel(kern, static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, st, true, p,
                                mk, mv);
}

template <int BS>
cudaError_t launch_group(const DecodeParams& p, int G, const CUtensorMap& mk, const CUtensorMap& mv,
                         long long grid, cudaStream_t st) {
    switch (G) {
        case 1: return launch_inst<BS, 1>(p, mk, mv, grid, st);
        case 2: return launch_inst<BS, 2>(p, mk, mv, grid, st);
        case 4: return launch_inst<BS, 4>(p, mk, mv, grid, st);
        case 8: return launch_inst<BS, 8>(p, mk, mv, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode_tc_fp8(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                                 int BS, int G, long long grid, cudaStream_t st) {
    switch (BS) {
        case 8: return launch_group<8>(p, G, mk, mv, grid, st);
        case 16: return launch_group<16>(p, G, mk, mv, grid, st);
        case 32: return launch_group<32>(p, G, mk, mv, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkv
