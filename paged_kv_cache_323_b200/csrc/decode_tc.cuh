// decode_tc.cuh -- tensor-core (tcgen05 + TMEM) paged decode attention for
// grouped-query heads on sm_100a: bf16 caches, head_dim 128, groups of 2, 4
// or 8 query heads per kv head.
//
// Same computation as decode_attn.cuh ("PagedAttention Explained: Virtual
// Memory for the KV Cache", section "How PagedAttention works", item 5: the
// attention follows the block table and gathers K and V from non-contiguous
// blocks), with the query-group x block contraction on the tensor cores.
// With G query heads sharing one kv head ("Trade-offs and related
// techniques": grouped-query attention), QK^T and PV are small matrix
// products; on CUDA cores their issue cost, not HBM, bounds the kernel.
//
// One CTA per (sequence, kv head, partition), 192 threads in three roles:
//  * warp 0, lane 0 -- producer: walks the partition's block-table entries
//    (loaded once, range-checked) and, for each 128-token chunk, brings the
//    chunk's K tile and then its V tile into a ring of three 32 KB shared
//    memory slots with 4-D TMA tensor copies (one box of 64 dims x bs slots
//    per block and half of the head dimension, 128-byte swizzle, no
//    multicast), completing on mbarriers.  Rows of a tile are tokens.
//  * warp 1 -- owns the TMEM allocation (64 columns); lane 0 issues the
//    MMAs: S^T[128 tokens x 16] = K_tile . Q^T (M=128, N=16, K=128 in eight
//    K=16 steps, both operands K-major) into one of two S buffers, then
//    O^T[128 dims x 16] = V_tile^T . P^T (A MN-major: the V tile read as
//    V^T) into one of two O buffers.  Query heads are padded to N=16 with
//    zero rows of Q; padded columns are never read.
//  * warps 2-5 -- softmax: thread r owns TMEM lane r, i.e. token r of the S
//    tile and head dimension r of the O tile.  Per chunk: read S, mask,
//    chunk max per head (warp shuffles, then the four warps through shared
//    memory and an mbarrier), base-2 probabilities, bf16 P^T into shared
//    memory (swizzled K-major), and the running sums; then fold the previous
//    chunk's O into fp32 registers with the rescaling factor of that chunk.
//    S, P and O are double-buffered, so the softmax of chunk c overlaps the
//    PV product of chunk c-1.  Rows past the context or in skipped blocks are
//    masked, and their V rows are zeroed before PV (they may hold NaN).
// The partition's (m, l, o) then go through the same output / fused split-K
// merge as the CUDA-core kernel.  Every wait is bounded; on timeout the CTA
// records the error, lets its copies and MMAs land, frees TMEM and returns.
#pragma once

#include <cuda.h>

#include "decode_common.cuh"

namespace pkv {
namespace tc {

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            int c3, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            int c3, int c4, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
        "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] . B[smem desc], 16-bit inputs (bf16 or f16, as
// the instruction descriptor says), fp32 accumulator.
__device__ __forceinline__ void mma_kind_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same with 8-bit inputs (e4m3 here), K = 32 per instruction.
__device__ __forceinline__ void mma_kind_f8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Make this thread's generic-proxy shared-memory writes visible to the
// async proxy (the tensor cores read P, Q and the zeroed V rows through it).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: start
// address, leading and stride byte offsets in 16-byte units, version 1,
// layout type 2 = SWIZZLE_128B).  All tiles start on 1024-byte boundaries.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

// Instruction descriptor: fp32 D (bit 4), A and B formats (bits 7-9 and
// 10-12: for kind::f16 0 = f16, 1 = bf16; for kind::f8f6f4 0 = e4m3), A and
// B major-ness (bits 15, 16: 1 = MN-major), N / 8 (bits 17-22), M / 16
// (bits 24-28).
constexpr uint32_t idesc_make(int M, int N, uint32_t ab_format, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (ab_format << 7) | (ab_format << 10) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return idesc_make(M, N, 1u, a_mn_major, b_mn_major);
}

template <int BS, int G>
struct TcCfg {
    static constexpr int D = 128;
    static constexpr int TILE = 128;         // tokens per chunk (MMA M of QK^T)
    static constexpr int BPT = TILE / BS;    // blocks per chunk
    static constexpr int NPAD = 16;          // query heads padded to the MMA N
    static constexpr int ROW = 128;          // bytes of one swizzled row (64 bf16)
    static constexpr int HALF = TILE * ROW;  // one 64-dim half of a K or V tile
    static constexpr int SLOT = 2 * HALF;    // one K or V tile (32 KB)
    // Tile layout.  Block sizes 16 and 32: the first 64-dim half of all 128
    // tokens, then the second (two copies per block, one per half).  Block
    // size 8: one copy per block lands its 8 rows of the first half and then
    // its 8 rows of the second (2 KB), so a chunk is 16 such pairs -- half
    // the copies, which at 1 KB each had set the pace (~45 SM cycles per
    // copy).  Either way token r's half h sits at
    // (r / 8) * GSTRIDE + h * HSTEP + (r % 8) * ROW.
    static constexpr bool IL = BS == 8;
    static constexpr int HSTEP = IL ? 8 * ROW : HALF;        // offset of the second half
    static constexpr int GSTRIDE = IL ? 16 * ROW : 8 * ROW;  // stride of 8-token groups
    static constexpr int NSLOT = 3;
    static constexpr int QB = 2 * NPAD * ROW;  // Q operand: 2 dim halves x 16 rows
    static constexpr int PB = 2 * NPAD * ROW;  // one P operand: 2 token halves x 16 rows
    static constexpr int MAX_PART_BLOCKS = 4096 / BS;
    static constexpr int THREADS = 192;
    static constexpr int NSOFT = 128;  // softmax threads
    static constexpr uint32_t TMEM_COLS = 64;
    static constexpr uint32_t S_COL = 0;   // two S buffers at columns 0 and 16
    static constexpr uint32_t O_COL = 32;  // two O buffers at columns 32 and 48
    // shared-memory map, offsets from a 1024-byte aligned base
    static constexpr int Q_OFF = NSLOT * SLOT;
    static constexpr int P_OFF = Q_OFF + QB;
    static constexpr int BAR_OFF = P_OFF + 2 * PB;
    // full[3] empty[3] s_full[2] s_free[2] p_full[2] o_full[2] o_free[2] red[2] mma_done
    static constexpr int NBARS = 2 * NSLOT + 13;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;  // tmem address, abort, last flag
    static constexpr int RED_OFF = MISC_OFF + 16;         // [2][4][16] chunk maxima, [4][16] sums
    static constexpr int PHYS_OFF = RED_OFF + (2 * 4 * NPAD + 4 * NPAD) * 4;
    static constexpr int SMEM_BYTES = PHYS_OFF + MAX_PART_BLOCKS * 4 + 1024;
    static constexpr uint32_t IDESC_QK = idesc_bf16(128, NPAD, false, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16(128, NPAD, true, false);

    static_assert(TILE % BS == 0 && (BS * ROW) % 1024 == 0, "blocks stack on swizzle atoms");
    static_assert(G <= NPAD, "query group fits the MMA N");
    static_assert(merge_scratch_bytes<G, D, THREADS>() <= NSLOT * SLOT, "merge scratch reuses the ring");
    static_assert(SMEM_BYTES <= 113 * 1024, "two CTAs per SM");
};

template <int BS, int G>
__global__ void __launch_bounds__(192, 2)
    decode_tc_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv) {
    using C = TcCfg<BS, G>;
    using T = __nv_bfloat16;
    constexpr int D = C::D;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

    const int P = p.num_partitions;
    // Launch order: the longest-first schedule when there is one.  Without
    // it, with a few partitions per sequence (the grid is sized for the
    // longest, so many CTAs lie past a shorter sequence's end)
    // partition-major, so the CTAs that exit at once come last instead of
    // taking SM slots between real work; with many (long contexts)
    // partition-fastest, so that a unit's partitions finish together.
    const Unit unit = decode_unit(p, P <= 4);
    if (unit.s < 0) return;  // a schedule entry out of range (debug builds)
    const int part = unit.part, g = unit.g, s = unit.s;
    const int ctx = unit.ctx;
    const int max_ctx = p.max_blocks_per_seq * BS;
    if (ctx < 0 || ctx > max_ctx) {
        if (part == 0) {
            if (threadIdx.x == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            zero_rows<T, D, G>(p, (long long)s * p.num_heads + (long long)g * G);
        }
        return;
    }
    const int PT = p.partition_tokens;
    const int nparts = (ctx + PT - 1) / PT;
    if (part >= nparts) {
        if (ctx == 0 && part == 0) zero_rows<T, D, G>(p, (long long)s * p.num_heads + (long long)g * G);
        return;
    }
    const int tok0 = part * PT;
    const int tok1 = min(ctx, tok0 + PT);
    const int nblk = (tok1 - tok0 + BS - 1) / BS;
    const int blk0 = tok0 / BS;
    const int nchunks = (tok1 - tok0 + C::TILE - 1) / C::TILE;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::NSLOT;
    uint64_t* s_full = bars + 2 * C::NSLOT;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* o_full = p_full + 2;
    uint64_t* o_free = o_full + 2;
    uint64_t* red_bar = o_free + 2;
    uint64_t* mma_done = red_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
    int* last_flag = reinterpret_cast<int*>(smem + C::MISC_OFF + 8);
    float* red_max = reinterpret_cast<float*>(smem + C::RED_OFF);  // [2][4][16]
    float* red_sum = red_max + 2 * 4 * C::NPAD;                   // [4][16]
    int* phys = reinterpret_cast<int*>(smem + C::PHYS_OFF);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < C::NSLOT; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 4);
            mbar_init(&p_full[b], 4);
            mbar_init(&o_full[b], 1);
            mbar_init(&o_free[b], 4);
            mbar_init(&red_bar[b], 4);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    const int32_t* bt = p.block_tables + (long long)s * p.max_blocks_per_seq + blk0;
    for (int j = tid; j < nblk; j += C::THREADS) {
        int e = bt[j];
        if (e < 0 || e >= p.num_blocks) {
            set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            e = -1;
        }
        phys[j] = e;
    }
    if (warp >= 2) {
        // Q operand: row h = query head g*G+h (zero for padded rows), 128-byte
        // swizzled rows, one region per 64-dim half; P buffers start at zero.
        const int t = tid - 64;
        for (int u = t; u < C::NPAD * 16; u += C::NSOFT) {
            const int h = u / 16;
            const int c16 = u % 16;  // 16-byte chunk of the 128 dims
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (h < G)
                val = reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) +
                                                     ((long long)s * p.num_heads + g * G + h) * D)[c16];
            const int half = c16 / 8, c = c16 % 8;
            *reinterpret_cast<uint4*>(smem + C::Q_OFF + half * (C::NPAD * C::ROW) + h * C::ROW +
                                      ((c ^ (h & 7)) * 16)) = val;
        }
        for (int u = t; u < 2 * C::PB / 16; u += C::NSOFT)
            reinterpret_cast<uint4*>(smem + C::P_OFF)[u] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int issued = 0;  // producer: loads issued
    int mma_issued = 0;
    // softmax state (warps 2-5)
    float m_run[G], l_run[G], acc[G], alpha_prev[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.f;
        acc[h] = 0.f;
        alpha_prev[h] = 1.f;
    }

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The whole warp: lane j issues the copies of block j of the chunk, so
        // the (up to 16) TMA issues of a chunk do not serialise on one thread.
        for (int li = 0; li < 2 * nchunks; ++li) {
            const int c = li >> 1;
            const CUtensorMap* map = (li & 1) ? &tmv : &tmk;
            const int st = li % C::NSLOT;
            if (li >= C::NSLOT) {
                const bool ready = mbar_wait_bounded(&empty[st], ((li / C::NSLOT) - 1) & 1, abort_flag, p.wait_ns);
                if (!__all_sync(0xffffffffu, ready)) {
                    if (lane == 0) {
                        set_error(p.err, PKV_ERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    break;
                }
            }
            const int jb0 = c * C::BPT;
            const int j = jb0 + lane;
            const int e = (lane < C::BPT && j < nblk) ? phys[j] : -1;
            const bool load = e >= 0 && PKV_DCHECK(p.err, e < p.num_blocks && g < p.num_kv_heads &&
                                                              st < C::NSLOT &&
                                                              (lane + 1) * BS * C::ROW <= C::HALF);
            const int nload = __popc(__ballot_sync(0xffffffffu, load));
            if (lane == 0) {
                if (nload > 0)
                    mbar_arrive_expect_tx(&full[st], (uint32_t)(nload * BS * 2 * C::ROW));
                else
                    mbar_arrive(&full[st]);
            }
            __syncwarp();  // the expected byte count is registered before any copy lands
            if (load) {
                if constexpr (C::IL) {
                    tma_load_5d(smem + st * C::SLOT + lane * 2 * BS * C::ROW, map, 0, 0, 0, g, e, &full[st]);
                } else {
                    unsigned char* dst = smem + st * C::SLOT + lane * BS * C::ROW;
                    tma_load_4d(dst, map, 0, 0, g, e, &full[st]);
                    tma_load_4d(dst + C::HALF, map, 64, 0, g, e, &full[st]);
                }
            }
            issued = li + 1;
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t q_base = smem_addr(smem + C::Q_OFF);
            auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) -> bool {
                if (mbar_wait_bounded(bar, parity, abort_flag, p.wait_ns)) return true;
                set_error(p.err, PKV_ERR_TIMEOUT);
                *abort_flag = 1;
                return false;
            };
            auto issue_qk = [&](int c) -> bool {
                const int li = 2 * c, st = li % C::NSLOT;
                if (!wait_or_abort(&full[st], (li / C::NSLOT) & 1)) return false;
                if (c >= 2 && !wait_or_abort(&s_free[c & 1], ((c >> 1) - 1) & 1)) return false;
                tc_fence_after();
                const uint32_t k_base = smem_addr(smem + st * C::SLOT);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = sw128_desc(k_base + (kk >> 2) * C::HSTEP + (kk & 3) * 32, 16, C::GSTRIDE);
                    const uint64_t b = sw128_desc(q_base + (kk >> 2) * (C::NPAD * C::ROW) + (kk & 3) * 32, 16, 1024);
                    mma_kind_f16(tmem + C::S_COL + (c & 1) * 16, a, b, C::IDESC_QK, kk > 0);
                }
                mma_commit(&s_full[c & 1]);
                mma_commit(&empty[st]);
                ++mma_issued;
                return true;
            };
            auto issue_pv = [&](int c) -> bool {
                const int li = 2 * c + 1, st = li % C::NSLOT;
                if (!wait_or_abort(&full[st], (li / C::NSLOT) & 1)) return false;
                if (!wait_or_abort(&p_full[c & 1], (c >> 1) & 1)) return false;
                if (c >= 2 && !wait_or_abort(&o_free[c & 1], ((c >> 1) - 1) & 1)) return false;
                tc_fence_after();
                const uint32_t v_base = smem_addr(smem + st * C::SLOT);
                const uint32_t p_base = smem_addr(smem + C::P_OFF + (c & 1) * C::PB);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // A = V^T, MN-major: 64-dim halves HSTEP apart, 8-token groups
                    // GSTRIDE apart, 16 tokens (two groups) per step
                    const uint64_t a = sw128_desc(v_base + kk * 2 * C::GSTRIDE, C::HSTEP, C::GSTRIDE);
                    const uint64_t b = sw128_desc(p_base + (kk >> 2) * (C::NPAD * C::ROW) + (kk & 3) * 32, 16, 1024);
                    mma_kind_f16(tmem + C::O_COL + (c & 1) * 16, a, b, C::IDESC_PV, kk > 0);
                }
                mma_commit(&o_full[c & 1]);
                mma_commit(&empty[st]);
                ++mma_issued;
                return true;
            };
            bool ok = issue_qk(0);
            for (int c = 0; ok && c < nchunks; ++c) {
                if (c + 1 < nchunks) ok = issue_qk(c + 1);
                if (ok) ok = issue_pv(c);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int q4 = warp & 3;            // TMEM lane quadrant of this warp
        const int r = q4 * 32 + lane;       // token row of S, dimension row of O
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
            const bool ok = mbar_wait_bounded(bar, parity, abort_flag, p.wait_ns);
            if (__all_sync(0xffffffffu, ok)) return true;
            if (lane == 0) {
                set_error(p.err, PKV_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            return false;
        };
        auto fold = [&](int cc, const float* alpha) -> bool {
            if (!wait_all(&o_full[cc & 1], (cc >> 1) & 1)) return false;
            tc_fence_after();
            float ov[16];
            tmem_ld16(lane_addr + C::O_COL + (cc & 1) * 16, ov);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[cc & 1]);
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = fmaf(acc[h], alpha[h], ov[h]);
            return true;
        };
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            if (!wait_all(&s_full[c & 1], (c >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[16];
            tmem_ld16(lane_addr + C::S_COL + (c & 1) * 16, sv);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[c & 1]);

            const int rel = c * C::TILE + r;  // token index within the partition
            const bool valid = tok0 + rel < tok1 && phys[rel / BS] >= 0;
            float x[G];
#pragma unroll
            for (int h = 0; h < G; ++h) x[h] = valid ? sv[h] * p.qscale : -INFINITY;
            // chunk maximum per head: within the warp, then across the four warps
            float* rm = red_max + (c & 1) * 4 * C::NPAD;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float v = x[h];
#pragma unroll
                for (int msk = 16; msk; msk >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, msk));
                if (lane == 0) rm[q4 * C::NPAD + h] = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_bar[c & 1]);
            if (!wait_all(&red_bar[c & 1], (c >> 1) & 1)) {
                ok = false;
                break;
            }
            float alpha[G];
            unsigned char* pbuf = smem + C::P_OFF + (c & 1) * C::PB;
            const int th = r / 64, tr = r % 64;  // token half and row within it
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float mc = fmaxf(fmaxf(rm[h], rm[C::NPAD + h]), fmaxf(rm[2 * C::NPAD + h], rm[3 * C::NPAD + h]));
                const float m_new = fmaxf(m_run[h], mc);
                alpha[h] = m_new == -INFINITY ? 1.f : exp2f(m_run[h] - m_new);
                m_run[h] = m_new;
                const float pr = valid ? exp2f(x[h] - m_new) : 0.f;
                const __nv_bfloat16 pb = __float2bfloat16_rn(pr);
                l_run[h] = fmaf(l_run[h], alpha[h], __bfloat162float(pb));
                *reinterpret_cast<__nv_bfloat16*>(pbuf + th * (C::NPAD * C::ROW) + h * C::ROW +
                                                  ((((tr >> 3) ^ (h & 7)) << 4)) + (tr & 7) * 2) = pb;
            }
            // rows that are not valid tokens: zero their V rows (they may hold NaN)
            bool any_invalid = tok1 - (tok0 + c * C::TILE) < C::TILE;
            for (int j = c * C::BPT; j < min((c + 1) * C::BPT, nblk); ++j) any_invalid |= phys[j] < 0;
            if (any_invalid) {
                const int li = 2 * c + 1, st = li % C::NSLOT;
                if (!wait_all(&full[st], (li / C::NSLOT) & 1)) {
                    ok = false;
                    break;
                }
                if (!valid) {
                    unsigned char* row = smem + st * C::SLOT + (r >> 3) * C::GSTRIDE + (r & 7) * C::ROW;
                    uint4* row0 = reinterpret_cast<uint4*>(row);
                    uint4* row1 = reinterpret_cast<uint4*>(row + C::HSTEP);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        row0[k] = make_uint4(0u, 0u, 0u, 0u);
                        row1[k] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[c & 1]);
            if (c >= 1 && !fold(c - 1, alpha_prev)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int h = 0; h < G; ++h) alpha_prev[h] = alpha[h];
        }
        if (ok && nchunks > 0) ok = fold(nchunks - 1, alpha_prev);
        if (ok) {
            // totals of the running sums over the 128 softmax threads
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float v = l_run[h];
#pragma unroll
                for (int msk = 16; msk; msk >>= 1) v += __shfl_xor_sync(0xffffffffu, v, msk);
                if (lane == 0) red_sum[q4 * C::NPAD + h] = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_bar[nchunks & 1]);
            if (wait_all(&red_bar[nchunks & 1], (nchunks >> 1) & 1)) {
                const int H = p.num_heads;
                const long long sh0 = (long long)s * H + (long long)g * G;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    if (!PKV_DCHECK(p.err, sh0 + h < (long long)p.num_seqs * H && part < P)) continue;
                    const float L = (red_sum[h] + red_sum[C::NPAD + h]) +
                                    (red_sum[2 * C::NPAD + h] + red_sum[3 * C::NPAD + h]);
                    if (nparts == 1) {
                        Elem<T>::store(static_cast<T*>(p.out) + (sh0 + h) * D + r,
                                       L > 0.f ? acc[h] / L : 0.f);
                    } else {
                        p.ws_o[((sh0 + h) * P + part) * D + r] = acc[h];
                        if (r == 0) p.ws_ml[(sh0 + h) * P + part] = make_float2(m_run[h], L);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == 0 && lane == 0) {
            for (int li = issued - C::NSLOT > 0 ? issued - C::NSLOT : 0; li < issued; ++li) {
                const int st = li % C::NSLOT;
                const unsigned long long t0 = globaltimer_ns();
                while (!mbar_try_wait(&full[st], (li / C::NSLOT) & 1))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            }
        }
        if (warp == 1 && lane == 0 && mma_issued > 0) {
            mma_commit(mma_done);
            const unsigned long long t0 = globaltimer_ns();
            while (!mbar_try_wait(mma_done, 0))
                if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
        abort_merge_turn<T, D, G>(p, s, g, (long long)s * p.num_heads + (long long)g * G, part, nparts, last_flag);
        return;
    }
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
    if (nparts == 1) return;
    fused_merge<T, D, G, C::THREADS>(p, s, g, nparts, (long long)s * p.num_heads + (long long)g * G,
                                      reinterpret_cast<float*>(smem), last_flag);
}

}  // namespace tc
}  // namespace pkv
