// decode_tc_fp8p.cu -- launches of the persistent fp8 (e4m3) tensor-core
// decode kernel: one CTA per resident slot (SMs x CTAs per SM, never more
// than there are units), dispatched over (block_size, group size).
#include <atomic>

#include "decode_tc_fp8p.cuh"
#include "launch.h"

namespace pkv {
namespace {

template <int BS, int G, bool FW>
cudaError_t launch_fw(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                      long long units, cudaStream_t st) {
    using C = tc::TcFp8PCfg<BS, G>;
    auto kern = tc::decode_tc_fp8_persistent_kernel<BS, G, FW>;
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
    // CTAS_PER_SM is what registers (launch bounds), shared memory and TMEM
    // admit; a CTA that finds no slot free starts late and finds less work
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long slots = (long long)sms * C::CTAS_PER_SM;
    const long long grid = units < slots ? units : slots;
    return launch_decode_kernel(kern, static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, st,
                                p.order != nullptr, p, mk, mv);
}

// Launches whose sequences each fit one partition start a first wave in
// index order without waiting for the schedule (decode_tc_fp8p.cuh).
template <int BS, int G>
cudaError_t launch_inst(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                        long long units, cudaStream_t st) {
    return p.num_partitions == 1 ? launch_fw<BS, G, true>(p, mk, mv, units, st)
                                 : launch_fw<BS, G, false>(p, mk, mv, units, st);
}

template <int BS>
cudaError_t launch_group(const DecodeParams& p, int G, const CUtensorMap& mk, const CUtensorMap& mv,
                         long long units, cudaStream_t st) {
    switch (G) {
        case 1: return launch_inst<BS, 1>(p, mk, mv, units, st);
        case 2: return launch_inst<BS, 2>(p, mk, mv, units, st);
        case 4: return launch_inst<BS, 4>(p, mk, mv, units, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool decode_tc_fp8_persistent_supported(int BS, int G, int partition_tokens) {
    return (G == 1 || G == 2 || G == 4) && (BS == 8 || BS == 16 || BS == 32) &&
           partition_tokens <= decode_tc_fp8_persistent_max_tokens(BS);
}

int decode_tc_fp8_persistent_max_tokens(int BS) { return tc::TcFp8PCfg<16, 1>::MAX_PART_BLOCKS * BS; }

cudaError_t launch_decode_tc_fp8_persistent(const DecodeParams& p, const CUtensorMap& mk,
                                            const CUtensorMap& mv, int BS, int G, long long units,
                                            cudaStream_t st) {
    if (p.work == nullptr || !decode_tc_fp8_persistent_supported(BS, G, p.partition_tokens))
        return cudaErrorInvalidValue;
    switch (BS) {
        case 8: return launch_group<8>(p, G, mk, mv, units, st);
        case 16: return launch_group<16>(p, G, mk, mv, units, st);
        case 32: return launch_group<32>(p, G, mk, mv, units, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkv
