// decode_tc.cu -- host side of the tensor-core GQA decode kernel: TMA tensor
// maps over the K and V pools, and dispatch over (block_size, group size).
#include <atomic>
#include <mutex>

#include "decode_tc.cuh"
#include "launch.h"

namespace pkv {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

}  // namespace

void* tc_tensor_map_encoder() { return reinterpret_cast<void*>(encoder()); }

// The pool [num_blocks][Hkv][bs][128] as a 4-D tensor (dims innermost first:
// dim, slot, kv head, block); boxes of one 128-byte row span (64 bf16 dims or
// 128 e4m3 codes) x bs slots of one (block, kv head), 128-byte swizzle.
cudaError_t make_tc_pool_map(CUtensorMap* map, const void* pool, int Hkv, int BS, int num_blocks,
                             int elem_bytes) {
    EncodeTiledFn fn = encoder();
    if (fn == nullptr) return cudaErrorNotSupported;
    if (elem_bytes == 2 && BS == 8) {
        // bf16, block size 8: one box per block, both 64-dim halves: dims
        // (64 values, 8 slots at 256 B, 2 halves at 128 B, kv head, block),
        // box (64, 8, 2, 1, 1) -> the block's 8 rows of the first half, then
        // its 8 rows of the second
        const cuuint64_t dims[5] = {64, 8, 2, (cuuint64_t)Hkv, (cuuint64_t)num_blocks};
        const cuuint64_t strides[4] = {256, 128, 8 * 256, (cuuint64_t)Hkv * 8 * 256};
        const cuuint32_t box[5] = {64, 8, 2, 1, 1};
        const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
        const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(pool), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
    }
    const cuuint64_t eb = (cuuint64_t)elem_bytes;
    const cuuint64_t dims[4] = {128, (cuuint64_t)BS, (cuuint64_t)Hkv, (cuuint64_t)num_blocks};
    const cuuint64_t strides[3] = {128 * eb, (cuuint64_t)BS * 128 * eb, (cuuint64_t)Hkv * BS * 128 * eb};
    const cuuint32_t box[4] = {(cuuint32_t)(128 / elem_bytes), (cuuint32_t)BS, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                          4, const_cast<void*>(pool), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

template <int BS, int G>
cudaError_t launch_inst(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                        long long grid, cudaStream_t st) {
    using C = tc::TcCfg<BS, G>;
    auto kern = tc::decode_tc_kernel<BS, G>;
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
        case 2: return launch_inst<BS, 2>(p, mk, mv, grid, st);
        case 4: return launch_inst<BS, 4>(p, mk, mv, grid, st);
        case 8: return launch_inst<BS, 8>(p, mk, mv, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool decode_tc_supported(int kv_dtype, int D, int BS, int G, int Hkv, int partition_tokens) {
    const bool bs = (BS == 8 || BS == 16 || BS == 32) && partition_tokens % 128 == 0;
    if (kv_dtype == PKV_BF16) return bs && D == 128 && (G == 2 || G == 4 || G == 8);
    if (kv_dtype == PKV_FP8_E4M3) {
        if (D == 64) return bs && Hkv % 2 == 0 && (G == 1 || G == 2 || G == 4);  // kv head pairs
        return bs && D == 128 && (G == 1 || G == 2 || G == 4 || G == 8);
    }
    return false;
}

cudaError_t launch_decode_tc(const DecodeParams& p, int kv_dtype, int D, int BS, int G, long long grid,
                             bool persistent, cudaStream_t st) {
    if (kv_dtype == PKV_FP8_E4M3 && D == 64) return launch_decode_tc_fp8_d64(p, BS, G, st);
    const int eb = kv_dtype == PKV_FP8_E4M3 ? 1 : 2;
    CUtensorMap mk, mv;
    cudaError_t e = make_tc_pool_map(&mk, p.k_cache, p.num_kv_heads, BS, p.num_blocks, eb);
    if (e != cudaSuccess) return e;
    e = make_tc_pool_map(&mv, p.v_cache, p.num_kv_heads, BS, p.num_blocks, eb);
    if (e != cudaSuccess) return e;
    if (kv_dtype == PKV_FP8_E4M3)
        return persistent ? launch_decode_tc_fp8_persistent(p, mk, mv, BS, G, grid, st)
                          : launch_decode_tc_fp8(p, mk, mv, BS, G, grid, st);
    switch (BS) {
        case 8: return launch_group<8>(p, G, mk, mv, grid, st);
        case 16: return launch_group<16>(p, G, mk, mv, grid, st);
        case 32: return launch_group<32>(p, G, mk, mv, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkv
