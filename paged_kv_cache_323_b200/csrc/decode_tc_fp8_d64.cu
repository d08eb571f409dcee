// decode_tc_fp8_d64.cu -- host side of the head_dim-64 fp8 tensor-core decode
// kernel: the 5-D tensor maps that land a block of two kv heads as 8-token
// groups of the two heads' rows, and dispatch over (block_size, group size).
#include <atomic>

#include "decode_tc_fp8_d64.cuh"
#include "launch.h"

namespace pkv {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The pool [num_blocks][Hkv][bs][64] (one byte per code) as a 5-D tensor,
// dims innermost first: code (64), slot within a group of 8 (8, stride 64 B),
// kv head (Hkv, stride bs x 64 B), group of 8 slots (bs / 8, stride 512 B),
// block (stride Hkv x bs x 64 B).  A box (64, 8, 2, bs / 8, 1) at kv head g0
// lands, per group of 8 tokens, 8 rows of head g0 then 8 rows of head g0 + 1,
// 64-byte rows under the 64-byte swizzle.
cudaError_t make_pair_map(CUtensorMap* map, const void* pool, int Hkv, int BS, int num_blocks) {
    EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(tc_tensor_map_encoder());
    if (fn == nullptr) return cudaErrorNotSupported;
    const cuuint64_t row = 64;
    const cuuint64_t dims[5] = {64, 8, (cuuint64_t)Hkv, (cuuint64_t)(BS / 8), (cuuint64_t)num_blocks};
    const cuuint64_t strides[4] = {row, (cuuint64_t)BS * row, 8 * row, (cuuint64_t)Hkv * BS * row};
    const cuuint32_t box[5] = {64, 8, 2, (cuuint32_t)(BS / 8), 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(pool), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int BS, int G>
cudaError_t launch_inst(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                        long long grid, cudaStream_t st) {
    using C = tc::TcFp8D64Cfg<BS, G>;
    auto kern = tc::decode_tc_fp8_d64_kernel<BS, G>;
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
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode_tc_fp8_d64(const DecodeParams& p, int BS, int G, cudaStream_t st) {
    if (p.num_kv_heads % 2 != 0) return cudaErrorInvalidValue;
    CUtensorMap mk, mv;
    cudaError_t e = make_pair_map(&mk, p.k_cache, p.num_kv_heads, BS, p.num_blocks);
    if (e != cudaSuccess) return e;
    e = make_pair_map(&mv, p.v_cache, p.num_kv_heads, BS, p.num_blocks);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)p.num_seqs * (p.num_kv_heads / 2) * p.num_partitions;
    switch (BS) {
        case 8: return launch_group<8>(p, G, mk, mv, grid, st);
        case 16: return launch_group<16>(p, G, mk, mv, grid, st);
        case 32: return launch_group<32>(p, G, mk, mv, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkv
