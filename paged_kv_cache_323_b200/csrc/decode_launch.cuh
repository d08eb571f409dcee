// decode_launch.cuh -- compile-time dispatch of the decode kernels over
// (head_dim, block_size, query-group size).  Included by one .cu file per
// element type so the instantiations compile in parallel.
#pragma once

#include <atomic>

#include "decode_attn.cuh"

namespace pkv {

template <typename T, typename TKV, int D, int BS, int G>
cudaError_t launch_partition_inst(const DecodeParams& p, long long grid, cudaStream_t st) {
    using C = DecodeCfg<T, TKV, D, BS, G>;
    auto kern = decode_partition_kernel<T, TKV, D, BS, G>;
    static std::atomic<unsigned long long> configured{0};  // one bit per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit);
    }
    // every CTA waits for the preceding grid in decode_unit
    return launch_decode_kernel(kern, static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, st, true, p);
}

template <typename T, typename TKV, int D, int BS>
cudaError_t dispatch_group(const DecodeParams& p, int G, long long grid, cudaStream_t st) {
    switch (G) {
        case 1: return launch_partition_inst<T, TKV, D, BS, 1>(p, grid, st);
        case 2: return launch_partition_inst<T, TKV, D, BS, 2>(p, grid, st);
        case 4: return launch_partition_inst<T, TKV, D, BS, 4>(p, grid, st);
        case 8: return launch_partition_inst<T, TKV, D, BS, 8>(p, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, typename TKV, int D>
cudaError_t dispatch_block_size(const DecodeParams& p, int BS, int G, long long grid,
                                cudaStream_t st) {
    switch (BS) {
        case 8: return dispatch_group<T, TKV, D, 8>(p, G, grid, st);
        case 16: return dispatch_group<T, TKV, D, 16>(p, G, grid, st);
        case 32: return dispatch_group<T, TKV, D, 32>(p, G, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

// q / out of type T, cached K / V of type TKV
template <typename T, typename TKV = T>
cudaError_t dispatch_partition(const DecodeParams& p, int D, int BS, int G, long long grid,
                               cudaStream_t st) {
    switch (D) {
        case 64: return dispatch_block_size<T, TKV, 64>(p, BS, G, grid, st);
        case 128: return dispatch_block_size<T, TKV, 128>(p, BS, G, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkv
