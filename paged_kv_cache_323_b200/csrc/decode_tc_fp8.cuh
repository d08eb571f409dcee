// decode_tc_fp8.cuh -- tensor-core (tcgen05 + TMEM) paged decode attention
// over fp8 (OCP e4m3) K and V pools with one dequantisation scale per kv
// head: head_dim 128, 1, 2, 4 or 8 query heads per kv head, bf16 q and out.
//
// Same computation as decode_attn.cuh ("PagedAttention Explained: Virtual
// Memory for the KV Cache", section "How PagedAttention works", item 5: the
// attention follows the block table and gathers K and V from non-contiguous
// blocks) over a quantised cache (section "Sharing requires more than
// allocation": supported cache quantization), stored value = code x scale.
//
// Why the tensor cores: an e4m3 code costs the CUDA-core kernel a widening
// (e4m3 -> f16 -> f32) before each FMA, so per byte it issues twice the
// instructions of a bf16 cache, and with grouped query heads every code feeds
// G FMAs.  Here both products run on kind::f8f6f4 and read the codes as the
// TMA lands them (128-byte swizzle, one 128-byte row of 128 codes per token):
//  * S^T = K . Q^T: the K tile is the K-major A operand.  q is made e4m3
//    without losing its bf16 value: each head is scaled by a power of two so
//    that its largest |q| lies in [128, 256), then split as q = hi + lo / 16,
//    hi the nearest e4m3 of q and lo the nearest e4m3 of 16 (q - hi).  A bf16
//    value has 8 significant bits; after rounding to hi's 4 the remainder has
//    at most 4, so lo holds it exactly unless it falls below e4m3's subnormal
//    quantum -- elements under 2^-13 of the head's largest, which then err by
//    at most 2^-21 of it.  S column 2h is K.hi_h, column 2h+1 is K.lo_h, and
//    the logit is (S_2h + S_2h+1 / 16) times the logit scale, the K scale and
//    the inverse power of two.
//  * O^T = V^T . P^T: the V tile is the A operand read MN-major (dims are
//    contiguous in a token's row).  The probabilities p in [0, 1] are split
//    the same way at scale 256: 256 p = hi + lo / 16, so every p keeps 8
//    significant bits (as a bf16 P would) down to 2^-14, and errs by under
//    2^-22 below that.  P^T holds both terms as rows (2h: hi, 2h + 1: lo), so
//    one PV product gives O_hi and O_lo in columns 2h and 2h + 1, combined as
//    O_hi + O_lo / 16 when the chunk is folded; the running sums add the same
//    represented values.  V rows that are not tokens of the
//    partition are zeroed before PV (they may hold NaN codes).
//
// One CTA per (sequence, kv head, partition), 192 threads:
//  * warp 0 -- producer: per 128-token chunk, one TMA copy per block of the K
//    tile, then of the V tile, into a ring of 16 KB slots, K tiles in the
//    even slots and V tiles in the odd ones; no multicast.  Up to 4 query
//    heads per CTA: two slots, so that five (up to 2 heads) or four CTAs
//    share an SM and their per-chunk chains overlap.  8 query heads need
//    more registers (two CTAs per SM): six slots.
//  * warp 1 -- TMEM owner (64 columns) and, lane 0, MMA issuer: QK^T (M=128,
//    N=16, four K=32 steps) and PV (M=128, N=16, four K=32 steps, both p
//    terms at once), each issued as soon as its operands are ready (the
//    issuer polls both, so neither waits behind the other).
//  * warps 2-5 -- softmax, as in the bf16 kernel: thread r owns TMEM lane r
//    (token r of S, dimension r of O); S, P and O are double-buffered.
// Every wait is bounded; on timeout the CTA records the error, lets its copies
// and MMAs land, frees TMEM and returns.

#pragma once

#include "decode_tc.cuh"

namespace pkv {
namespace tc {

template <int BS, int G>
struct TcFp8Cfg {
    static constexpr int D = 128;
    static constexpr int TILE = 128;          // tokens per chunk
    static constexpr int BPT = TILE / BS;     // blocks per chunk
    static constexpr int NPAD = 16;           // MMA N: 2GT columns used by QK, G by PV
    static constexpr int ROW = 128;           // bytes of a swizzled row: 128 codes
    static constexpr int SLOT = TILE * ROW;   // one K or V tile (16 KB)
    // CTAs per SM: more CTAs overlap more per-chunk chains (2 -> 3 -> 4 on
    // batch-64 MHA: 122.5 / 115.0 / 112.0 us); up to 2 query heads fit the
    // 64 registers of 5, 4 heads the 80 of 4, 8 heads need 2.
    static constexpr int CTAS_PER_SM = G >= 8 ? 2 : (G >= 4 ? 4 : 5);
    static constexpr int NSLOT = CTAS_PER_SM == 2 ? 6 : 2;
    // tile li (K of chunk li/2 when even, V when odd) sits in slot li % NSLOT
    static constexpr int QB = NPAD * ROW;     // Q operand (hi and lo rows): 16 rows of 128 codes
    // one P buffer: P^T rows 2h (hi term) and 2h + 1 (lo term) of query head
    // h, 128 token codes each; one PV product yields both O terms
    static constexpr int PB = NPAD * ROW;
    static constexpr int MAX_PART_BLOCKS = 4096 / BS;
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 64;
    static constexpr uint32_t S_COL = 0;      // two S buffers at columns 0 and 16
    static constexpr uint32_t O_COL = 32;     // two O buffers at 32 and 48: column 2h hi, 2h + 1 lo
    // shared-memory map, offsets from a 1024-byte aligned base
    static constexpr int Q_OFF = NSLOT * SLOT;
    static constexpr int P_OFF = Q_OFF + QB;
    static constexpr int BAR_OFF = P_OFF + 2 * PB;
    // full[NSLOT] empty[NSLOT] s_full[2] s_free[2] p_full[2] o_full[2] o_free[2] red[2] mma_done
    static constexpr int NBARS = 2 * NSLOT + 13;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;   // tmem address, abort, last flag
    static constexpr int KQ_OFF = MISC_OFF + 16;           // per-head logit factor (float)
    static constexpr int RED_OFF = KQ_OFF + 8 * 4;         // [2][4][16] chunk maxima, [4][16] sums
    static constexpr int PHYS_OFF = RED_OFF + (2 * 4 * NPAD + 4 * NPAD) * 4;
    static constexpr int SMEM_BYTES = PHYS_OFF + MAX_PART_BLOCKS * 4 + 1024;
    // e4m3 x e4m3: QK with both operands K-major, PV with A (V^T) MN-major
    static constexpr uint32_t IDESC_QK = idesc_make(128, NPAD, 0u, false, false);
    static constexpr uint32_t IDESC_PV = idesc_make(128, NPAD, 0u, true, false);

    static_assert(TILE % BS == 0 && (BS * ROW) % 1024 == 0, "blocks stack on swizzle atoms");
    static_assert(2 * G <= NPAD && G <= 8, "hi and lo columns of every head fit the MMA N");
    static_assert(Q_OFF % 1024 == 0 && P_OFF % 1024 == 0 && PB % 1024 == 0, "operand alignment");
    static_assert(merge_scratch_bytes<G, D, THREADS>() <= NSLOT * SLOT, "merge scratch reuses the ring");
    static_assert(CTAS_PER_SM * (SMEM_BYTES + 1024) <= 228 * 1024, "CTAs per SM by shared memory");
    static_assert(CTAS_PER_SM * TMEM_COLS <= 512, "CTAs per SM by TMEM");
    // An even ring keeps K tiles and V tiles in slots of their own, so a
    // tile's slot was last used by the same product's previous tile, whose
    // wait came first.  With an odd ring, K of chunk c would take the slot
    // V of chunk c-2 held, and the issuer's parity test could not tell that
    // barrier's awaited phase from the phase before it.
    static_assert(NSLOT % 2 == 0, "K and V tiles in slots of their own");
};

// Two floats to two e4m3 codes (low byte first), round to nearest even,
// saturating to +-448.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

// Two e4m3 codes (low byte first) back to floats, exactly.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t two_codes) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two_codes & 0xffffu), __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Whether the phase of `bar` with the given parity has completed (no wait).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Maximum of v over the warp.
__device__ __forceinline__ float warp_max(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

// The first N columns of this thread's TMEM lane from taddr, waited for
// (N = 2, 4, 8 or 16).
template <int N>
__device__ __forceinline__ void tmem_ld_first(uint32_t taddr, float (&v)[N]) {
    static_assert(N == 2 || N == 4 || N == 8 || N == 16, "load shape");
    if constexpr (N == 16) {
        tmem_ld16(taddr, v);
    } else {
        uint32_t r[N];
        if constexpr (N == 2) {
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];\n\t"
                "tcgen05.wait::ld.sync.aligned;"
                : "=r"(r[0]), "=r"(r[1])
                : "r"(taddr)
                : "memory");
        } else if constexpr (N == 4) {
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];\n\t"
                "tcgen05.wait::ld.sync.aligned;"
                : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                : "r"(taddr)
                : "memory");
        } else if constexpr (N == 8) {
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
                "tcgen05.wait::ld.sync.aligned;"
                : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                  "=r"(r[6]), "=r"(r[7])
                : "r"(taddr)
                : "memory");
        }
#pragma unroll
        for (int i = 0; i < N; ++i) v[i] = __uint_as_float(r[i]);
    }
}

template <int BS, int G>
__global__ void __launch_bounds__(192, TcFp8Cfg<BS, G>::CTAS_PER_SM)
    decode_tc_fp8_kernel(const __grid_constant__ DecodeParams p,
                         const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv) {
    using C = TcFp8Cfg<BS, G>;
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
    const int PTOK = p.partition_tokens;
    const int nparts = (ctx + PTOK - 1) / PTOK;
    if (part >= nparts) {
        if (ctx == 0 && part == 0) zero_rows<T, D, G>(p, (long long)s * p.num_heads + (long long)g * G);
        return;
    }
    const int tok0 = part * PTOK;
    const int tok1 = min(ctx, tok0 + PTOK);
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
    float* qsk = reinterpret_cast<float*>(smem + C::KQ_OFF);  // [G]
    float* red_max = reinterpret_cast<float*>(smem + C::RED_OFF);  // [2][4][16]
    float* red_sum = red_max + 2 * 4 * C::NPAD;                   // [4][16]
    int* phys = reinterpret_cast<int*>(smem + C::PHYS_OFF);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < C::NSLOT; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);  // freed by the MMA that read the slot
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
        // Q operand: row n = 2h + term (hi, 16 x lo) of query head g*G+h, zero
        // rows past 2G; thread t writes 16 codes (dims 16j .. 16j+15) of row t / 8.
        const int t = tid - 64;
        const int n = t >> 3, j = t & 7;
        const int hq = n >> 1;  // query head within the group
        float qv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) qv[e] = 0.f;
        if (n < 2 * G) {
            const uint4* qrow = reinterpret_cast<const uint4*>(
                static_cast<const T*>(p.q) + ((long long)s * p.num_heads + g * G + hq) * D + j * 16);
            Elem<T>::unpack(qrow[0], qv);
            Elem<T>::unpack(qrow[1], qv + 8);
        }
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(qv[e]));
#pragma unroll
        for (int msk = 1; msk < 8; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
        // largest |q| of the head into [128, 256)
        int kexp = mx > 0.f ? 7 - ((int)((__float_as_uint(mx) >> 23) & 0xffu) - 127) : 0;
        kexp = kexp < -120 ? -120 : (kexp > 120 ? 120 : kexp);
        const float up = __uint_as_float((uint32_t)(127 + kexp) << 23);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t hw = 0, lw = 0;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const float a = qv[4 * i + 2 * h2] * up, b = qv[4 * i + 2 * h2 + 1] * up;
                const uint32_t hc = f32x2_to_e4m3x2(a, b);
                const float2 hv = e4m3x2_to_f32x2(hc);
                const uint32_t lc = f32x2_to_e4m3x2((a - hv.x) * 16.f, (b - hv.y) * 16.f);
                hw |= hc << (16 * h2);
                lw |= lc << (16 * h2);
            }
            w[i] = (n & 1) ? lw : hw;
        }
        uint4 val = make_uint4(w[0], w[1], w[2], w[3]);
        if (n >= 2 * G) val = make_uint4(0u, 0u, 0u, 0u);
        if (!(mx <= 3.402823466e38f)) val = make_uint4(0x7f7f7f7fu, 0x7f7f7f7fu, 0x7f7f7f7fu, 0x7f7f7f7fu);  // inf / NaN in q: NaN codes
        *reinterpret_cast<uint4*>(smem + C::Q_OFF + n * C::ROW + ((j ^ (n & 7)) * 16)) = val;
        // the logit of head n/2 is its S columns' sum times scale, k_scale and 2^-k
        if (n < 2 * G && (n & 1) == 0 && j == 0)
            qsk[hq] = p.qscale * p.k_scales[g] * __uint_as_float((uint32_t)(127 - kexp) << 23);
        for (int u = t; u < 2 * C::PB / 16; u += 128)
            reinterpret_cast<uint4*>(smem + C::P_OFF)[u] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // a bounded wait taken by a whole warp; the warp leaves together if any lane gave up
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        const bool ok = mbar_wait_bounded(bar, parity, abort_flag, p.wait_ns);
        if (__all_sync(0xffffffffu, ok)) return true;
        if (lane == 0) {
            set_error(p.err, PKV_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        return false;
    };

    int issued = 0;  // producer: loads issued
    int mma_issued = 0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        for (int li = 0; li < 2 * nchunks; ++li) {
            const int c = li >> 1;
            const CUtensorMap* map = (li & 1) ? &tmv : &tmk;
            const int st = li % C::NSLOT;
            if (li >= C::NSLOT && !wait_all(&empty[st], ((li / C::NSLOT) - 1) & 1)) break;
            const int j = c * C::BPT + lane;
            const int e = (lane < C::BPT && j < nblk) ? phys[j] : -1;
            const bool load = e >= 0 && PKV_DCHECK(p.err, e < p.num_blocks && g < p.num_kv_heads &&
                                                              st < C::NSLOT &&
                                                              (lane + 1) * BS * C::ROW <= C::SLOT);
            const int nload = __popc(__ballot_sync(0xffffffffu, load));
            if (lane == 0) {
                if (nload > 0)
                    mbar_arrive_expect_tx(&full[st], (uint32_t)(nload * BS * C::ROW));
                else
                    mbar_arrive(&full[st]);
            }
            __syncwarp();  // the expected byte count is registered before any copy lands
            if (load) tma_load_4d(smem + st * C::SLOT + lane * BS * C::ROW, map, 0, 0, g, e, &full[st]);
            issued = li + 1;
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t q_base = smem_addr(smem + C::Q_OFF);
            int nq = 0, np = 0;  // next chunk for QK^T, for PV
            unsigned long long t_last = globaltimer_ns();
            while (np < nchunks) {
                bool progressed = false;
                if (nq < nchunks) {
                    const int li = 2 * nq, st = li % C::NSLOT;
                    if (mbar_test(&full[st], (li / C::NSLOT) & 1) &&
                        (nq < 2 || mbar_test(&s_free[nq & 1], ((nq >> 1) - 1) & 1))) {
                        tc_fence_after();
                        const uint32_t k_base = smem_addr(smem + st * C::SLOT);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {  // 32 codes (bytes) per step
                            const uint64_t a = sw128_desc(k_base + kk * 32, 16, 1024);
                            const uint64_t b = sw128_desc(q_base + kk * 32, 16, 1024);
                            mma_kind_f8f6f4(tmem + C::S_COL + (nq & 1) * 16, a, b, C::IDESC_QK, kk > 0);
                        }
                        mma_commit(&s_full[nq & 1]);
                        mma_commit(&empty[st]);
                        ++nq;
                        ++mma_issued;
                        progressed = true;
                    }
                }
                if (np < nq) {
                    const int li = 2 * np + 1, st = li % C::NSLOT;
                    if (mbar_test(&full[st], (li / C::NSLOT) & 1) &&
                        mbar_test(&p_full[np & 1], (np >> 1) & 1) &&
                        (np < 2 || mbar_test(&o_free[np & 1], ((np >> 1) - 1) & 1))) {
                        tc_fence_after();
                        const uint32_t v_base = smem_addr(smem + st * C::SLOT);
                        const uint32_t p_base = smem_addr(smem + C::P_OFF + (np & 1) * C::PB);
                        const uint32_t o_col = tmem + C::O_COL + (np & 1) * 16;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            // A = V^T, MN-major: the 128 dims of a token are one swizzled
                            // row; 32 tokens per step, 8-token groups 1024 B apart.
                            // B = P^T, both terms of every head (N = 16).
                            const uint64_t a = sw128_desc(v_base + kk * 32 * C::ROW, 16, 1024);
                            const uint64_t b = sw128_desc(p_base + kk * 32, 16, 1024);
                            mma_kind_f8f6f4(o_col, a, b, C::IDESC_PV, kk > 0);
                        }
                        mma_commit(&o_full[np & 1]);
                        mma_commit(&empty[st]);
                        ++np;
                        ++mma_issued;
                        progressed = true;
                    }
                }
                if (progressed) {
                    t_last = globaltimer_ns();
                } else {
                    if (*abort_flag) break;
                    if (globaltimer_ns() - t_last > p.wait_ns) {
                        set_error(p.err, PKV_ERR_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int q4 = warp & 3;            // TMEM lane quadrant of this warp
        const int r = q4 * 32 + lane;       // token row of S, dimension row of O
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        float m_run[G], l_run[G], acc[G], alpha_prev[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m_run[h] = -INFINITY;
            l_run[h] = 0.f;
            alpha_prev[h] = 1.f;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = 0.f;
        auto fold = [&](int cc, const float* alpha) -> bool {
            if (!wait_all(&o_full[cc & 1], (cc >> 1) & 1)) return false;
            tc_fence_after();
            float ov[2 * G], oh[G], ol[G];
            tmem_ld_first<2 * G>(lane_addr + C::O_COL + (cc & 1) * 16, ov);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                oh[h] = ov[2 * h];
                ol[h] = ov[2 * h + 1];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[cc & 1]);
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = fmaf(acc[h], alpha[h], fmaf(ol[h], 0.0625f, oh[h]));
            return true;
        };
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            if (!wait_all(&s_full[c & 1], (c >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[2 * G];
            tmem_ld_first<2 * G>(lane_addr + C::S_COL + (c & 1) * 16, sv);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[c & 1]);

            const int rel = c * C::TILE + r;
            const bool valid = tok0 + rel < tok1 && phys[rel / BS] >= 0;
            float x[G];
#pragma unroll
            for (int h = 0; h < G; ++h)
                x[h] = valid ? fmaf(sv[2 * h + 1], 0.0625f, sv[2 * h]) * qsk[h] : -INFINITY;
            float* rm = red_max + (c & 1) * 4 * C::NPAD;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float v = warp_max(x[h]);
                if (lane == 0) rm[q4 * C::NPAD + h] = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_bar[c & 1]);
            if (!wait_all(&red_bar[c & 1], (c >> 1) & 1)) {
                ok = false;
                break;
            }
            constexpr int GP = G + (G & 1);  // heads rounded up to pairs
            float alpha[G], pr[GP];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float mc = fmaxf(fmaxf(rm[h], rm[C::NPAD + h]), fmaxf(rm[2 * C::NPAD + h], rm[3 * C::NPAD + h]));
                const float m_new = fmaxf(m_run[h], mc);
                alpha[h] = m_new == -INFINITY ? 1.f : exp2f(m_run[h] - m_new);
                m_run[h] = m_new;
                pr[h] = valid ? exp2f(x[h] - m_new) * 256.f : 0.f;
            }
            if constexpr (GP > G) pr[G] = 0.f;
            // 256 p = hi + lo / 16, both e4m3; P^T rows 2h, 2h + 1, K-major over tokens
            unsigned char* pbuf = smem + C::P_OFF + (c & 1) * C::PB;
#pragma unroll
            for (int h = 0; h < GP; h += 2) {
                const uint32_t hc = f32x2_to_e4m3x2(pr[h], pr[h + 1]);
                const float2 hv = e4m3x2_to_f32x2(hc);
                const uint32_t lc = f32x2_to_e4m3x2((pr[h] - hv.x) * 16.f, (pr[h + 1] - hv.y) * 16.f);
                const float2 lv = e4m3x2_to_f32x2(lc);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int hh = h + u;
                    if (hh >= G) break;
                    const float rep = (u ? fmaf(lv.y, 0.0625f, hv.y) : fmaf(lv.x, 0.0625f, hv.x)) * 0.00390625f;
                    l_run[hh] = fmaf(l_run[hh], alpha[hh], rep);
                    const int rh = 2 * hh, rl = 2 * hh + 1;  // P^T rows of the two terms
                    pbuf[rh * C::ROW + (((r >> 4) ^ (rh & 7)) << 4) + (r & 15)] = (unsigned char)(hc >> (8 * u));
                    pbuf[rl * C::ROW + (((r >> 4) ^ (rl & 7)) << 4) + (r & 15)] = (unsigned char)(lc >> (8 * u));
                }
            }
            // the V tile must have landed; rows that are not valid tokens get
            // zero codes (they may hold NaN ones)
            {
                const int li = 2 * c + 1, st = li % C::NSLOT;
                if (!wait_all(&full[st], (li / C::NSLOT) & 1)) {
                    ok = false;
                    break;
                }
                if (!valid) {
                    uint4* row = reinterpret_cast<uint4*>(smem + st * C::SLOT + r * C::ROW);
#pragma unroll
                    for (int k = 0; k < 8; ++k) row[k] = make_uint4(0u, 0u, 0u, 0u);
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
                // O accumulated 256 p; the V scale and 1/256 go on here
                const float vsc = p.v_scales[g] * 0.00390625f;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    if (!PKV_DCHECK(p.err, sh0 + h < (long long)p.num_seqs * H && part < P)) continue;
                    const float L = (red_sum[h] + red_sum[C::NPAD + h]) +
                                    (red_sum[2 * C::NPAD + h] + red_sum[3 * C::NPAD + h]);
                    const float O = acc[h] * vsc;
                    if (nparts == 1) {
                        Elem<T>::store(static_cast<T*>(p.out) + (sh0 + h) * D + r, L > 0.f ? O / L : 0.f);
                    } else {
                        p.ws_o[((sh0 + h) * P + part) * D + r] = O;
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
        abort_merge_turn<T, D, G>(p, s, g, (long long)s * p.num_heads + (long long)g * G, part,
                                   nparts, last_flag);
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
