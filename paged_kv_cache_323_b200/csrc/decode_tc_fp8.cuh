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
// G FMAs.  Here the codes are read by the tensor cores:
//  * QK^T on kind::f8f6f4.  The K tile lands from the pool by TMA (128-byte
//    swizzle, one 128-byte row of 128 codes per token) and is the A operand
//    as it is.  q is made e4m3 without losing its bf16 value: each head is
//    scaled by a power of two so that its largest |q| lies in [128, 256),
//    then split as q = hi + lo, hi the nearest e4m3 of q and lo the nearest
//    e4m3 of the remainder.  The remainder of a bf16 value (8 significant
//    bits) after rounding to 4 has at most 4 significant bits, so the split
//    is exact for every element whose remainder is above e4m3's subnormal
//    quantum -- all elements within 2^-9 of the head's largest; smaller ones
//    err by at most 2^-18 of it.  Column 2h of the S tile is K.hi_h^T, column
//    2h+1 is K.lo_h^T, and the logit is their sum times the logit scale, the
//    K scale and the inverse power of two.
//  * PV on kind::f16.  Four widening warps turn each V tile's codes into f16
//    (exact) in a shared-memory operand laid out as the bf16 kernel's TMA lays
//    out a bf16 V tile (128-byte swizzle, tokens as rows), and write zeros for
//    rows that are not tokens of the partition; P is f16 (11 significant
//    bits).  The V scale multiplies the partition's output.
//
// One CTA per (sequence, kv head, partition), 320 threads:
//  * warp 0 -- producer: per 128-token chunk, one TMA copy per block of the K
//    tile, then of the V tile, into a ring of four 16 KB slots (K tiles in
//    slots 0 and 2, V tiles in 1 and 3); no multicast.
//  * warp 1 -- TMEM owner (64 columns) and, lane 0, MMA issuer: S^T[128 x 16]
//    = K_tile . Qs^T (M=128, N=16, K=128 in four K=32 steps), then O^T[128 x
//    16] = V16^T . P^T (A MN-major, eight K=16 steps).
//  * warps 2-5 -- softmax, as in the bf16 kernel: thread r owns TMEM lane r
//    (token r of S, dimension r of O); S, P and O are double-buffered.
//  * warps 6-9 -- V widening: thread r widens row r of each V tile.
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
    static constexpr int NPAD = 16;           // MMA N: 2G columns used by QK, G by PV
    static constexpr int ROW = 128;           // bytes of a swizzled row (128 codes or 64 f16)
    static constexpr int SLOT = TILE * ROW;   // one fp8 K or V tile (16 KB)
    static constexpr int NSLOT = 4;           // K in slots 0, 2; V in 1, 3
    static constexpr int HALF16 = TILE * ROW; // one 64-dim half of the f16 V operand
    static constexpr int QB = NPAD * ROW;     // Q operand: 16 rows of 128 codes
    static constexpr int PB = 2 * NPAD * ROW; // one f16 P operand: 2 token halves x 16 rows
    static constexpr int MAX_PART_BLOCKS = 4096 / BS;
    static constexpr int THREADS = 320;
    static constexpr uint32_t TMEM_COLS = 64;
    static constexpr uint32_t S_COL = 0;      // two S buffers at columns 0 and 16
    static constexpr uint32_t O_COL = 32;     // two O buffers at columns 32 and 48
    // shared-memory map, offsets from a 1024-byte aligned base
    static constexpr int Q_OFF = NSLOT * SLOT;
    static constexpr int V16_OFF = Q_OFF + QB;
    static constexpr int P_OFF = V16_OFF + 2 * HALF16;
    static constexpr int BAR_OFF = P_OFF + 2 * PB;
    // full[4] empty[4] s_full[2] s_free[2] p_full[2] o_full[2] o_free[2] red[2]
    // mma_done v16_full v16_free
    static constexpr int NBARS = 2 * NSLOT + 15;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;   // tmem address, abort, last flag
    static constexpr int KQ_OFF = MISC_OFF + 16;           // per-head power of two of q
    static constexpr int RED_OFF = KQ_OFF + 8 * 4;         // [2][4][16] chunk maxima, [4][16] sums
    static constexpr int PHYS_OFF = RED_OFF + (2 * 4 * NPAD + 4 * NPAD) * 4;
    static constexpr int SMEM_BYTES = PHYS_OFF + MAX_PART_BLOCKS * 4 + 1024;
    static constexpr uint32_t IDESC_QK = idesc_make(128, NPAD, 0u, false, false);  // e4m3 x e4m3
    static constexpr uint32_t IDESC_PV = idesc_make(128, NPAD, 0u, true, false);   // f16 x f16

    static_assert(TILE % BS == 0 && (BS * ROW) % 1024 == 0, "blocks stack on swizzle atoms");
    static_assert(2 * G <= NPAD && G <= 8, "hi and lo columns of every head fit the MMA N");
    static_assert(Q_OFF % 1024 == 0 && V16_OFF % 1024 == 0 && P_OFF % 1024 == 0, "operand alignment");
    static_assert(merge_scratch_bytes<G, D, THREADS>() <= NSLOT * SLOT, "merge scratch reuses the ring");
    static_assert(SMEM_BYTES <= 113 * 1024, "two CTAs per SM");
};

// Four e4m3 codes (low byte first) widened exactly to two f16 pairs.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t codes, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 c01, c23;\n\t"
        "mov.b32 {c01, c23}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, c01;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, c23;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(codes));
}

// Maximum of v over the warp.
__device__ __forceinline__ float warp_max(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

template <int BS, int G>
__global__ void __launch_bounds__(320, 2)
    decode_tc_fp8_kernel(const __grid_constant__ DecodeParams p,
                         const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv) {
    using C = TcFp8Cfg<BS, G>;
    using T = __nv_bfloat16;
    constexpr int D = C::D;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

    const int P = p.num_partitions;
    const int Hkv = p.num_kv_heads;
    const long long bid = blockIdx.x;
    const int part = (int)(bid % P);
    const int g = (int)((bid / P) % Hkv);
    const int s = (int)(bid / ((long long)P * Hkv));
    const int ctx = p.context_lens[s];
    const int max_ctx = p.max_blocks_per_seq * BS;
    if (ctx < 0 || ctx > max_ctx) {
        if (part == 0) {
            if (threadIdx.x == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            zero_rows<T, D, G>(p, s, g);
        }
        return;
    }
    const int PT = p.partition_tokens;
    const int nparts = (ctx + PT - 1) / PT;
    if (part >= nparts) {
        if (ctx == 0 && part == 0) zero_rows<T, D, G>(p, s, g);
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
    uint64_t* v16_full = mma_done + 1;
    uint64_t* v16_free = v16_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
    int* last_flag = reinterpret_cast<int*>(smem + C::MISC_OFF + 8);
    int* kq = reinterpret_cast<int*>(smem + C::KQ_OFF);
    float* red_max = reinterpret_cast<float*>(smem + C::RED_OFF);  // [2][4][16]
    float* red_sum = red_max + 2 * 4 * C::NPAD;                   // [4][16]
    int* phys = reinterpret_cast<int*>(smem + C::PHYS_OFF);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < C::NSLOT; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], (i & 1) ? 4 : 1);  // V slots: the four widening warps
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
        mbar_init(v16_full, 4);
        mbar_init(v16_free, 1);
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
    if (warp >= 2 && warp < 6) {
        // Q operand: row n = 2h + term (hi, lo) of query head g*G+h, zero rows
        // past 2G; thread t writes 16 codes (dims 16j .. 16j+15) of row t / 8.
        const int t = tid - 64;
        const int n = t >> 3, j = t & 7;
        float qv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) qv[e] = 0.f;
        if (n < 2 * G) {
            const uint4* qrow = reinterpret_cast<const uint4*>(
                static_cast<const T*>(p.q) + ((long long)s * p.num_heads + g * G + (n >> 1)) * D + j * 16);
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
                const __nv_fp8x2_storage_t hc =
                    __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
                const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(hc, __NV_E4M3);
                const float2 hv = __half22float2(*reinterpret_cast<const __half2*>(&hr));
                const __nv_fp8x2_storage_t lc =
                    __nv_cvt_float2_to_fp8x2(make_float2(a - hv.x, b - hv.y), __NV_SATFINITE, __NV_E4M3);
                hw |= (uint32_t)hc << (16 * h2);
                lw |= (uint32_t)lc << (16 * h2);
            }
            w[i] = (n & 1) ? lw : hw;
        }
        uint4 val = make_uint4(w[0], w[1], w[2], w[3]);
        if (n >= 2 * G) val = make_uint4(0u, 0u, 0u, 0u);
        if (!(mx <= 3.402823466e38f)) val = make_uint4(0x7f7f7f7fu, 0x7f7f7f7fu, 0x7f7f7f7fu, 0x7f7f7f7fu);  // inf / NaN in q: NaN codes
        *reinterpret_cast<uint4*>(smem + C::Q_OFF + n * C::ROW + ((j ^ (n & 7)) * 16)) = val;
        if (n < 2 * G && (n & 1) == 0 && j == 0) kq[n >> 1] = kexp;
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
        const bool ok = mbar_wait_bounded(bar, parity, abort_flag);
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
            const int nload = __popc(__ballot_sync(0xffffffffu, e >= 0));
            if (lane == 0) {
                if (nload > 0)
                    mbar_arrive_expect_tx(&full[st], (uint32_t)(nload * BS * C::ROW));
                else
                    mbar_arrive(&full[st]);
            }
            __syncwarp();  // the expected byte count is registered before any copy lands
            if (e >= 0) tma_load_4d(smem + st * C::SLOT + lane * BS * C::ROW, map, 0, 0, g, e, &full[st]);
            issued = li + 1;
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t q_base = smem_addr(smem + C::Q_OFF);
            const uint32_t v16_base = smem_addr(smem + C::V16_OFF);
            auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) -> bool {
                if (mbar_wait_bounded(bar, parity, abort_flag)) return true;
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
                for (int kk = 0; kk < 4; ++kk) {  // 32 codes (bytes) per step
                    const uint64_t a = sw128_desc(k_base + kk * 32, 16, 1024);
                    const uint64_t b = sw128_desc(q_base + kk * 32, 16, 1024);
                    mma_kind_f8f6f4(tmem + C::S_COL + (c & 1) * 16, a, b, C::IDESC_QK, kk > 0);
                }
                mma_commit(&s_full[c & 1]);
                mma_commit(&empty[st]);
                ++mma_issued;
                return true;
            };
            auto issue_pv = [&](int c) -> bool {
                if (!wait_or_abort(v16_full, c & 1)) return false;
                if (!wait_or_abort(&p_full[c & 1], (c >> 1) & 1)) return false;
                if (c >= 2 && !wait_or_abort(&o_free[c & 1], ((c >> 1) - 1) & 1)) return false;
                tc_fence_after();
                const uint32_t p_base = smem_addr(smem + C::P_OFF + (c & 1) * C::PB);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // A = V16^T, MN-major: 64-dim halves HALF16 apart, 8-token groups 1024 B apart
                    const uint64_t a = sw128_desc(v16_base + kk * 16 * C::ROW, C::HALF16, 1024);
                    const uint64_t b = sw128_desc(p_base + (kk >> 2) * (C::NPAD * C::ROW) + (kk & 3) * 32, 16, 1024);
                    mma_kind_f16(tmem + C::O_COL + (c & 1) * 16, a, b, C::IDESC_PV, kk > 0);
                }
                mma_commit(&o_full[c & 1]);
                mma_commit(v16_free);
                ++mma_issued;
                return true;
            };
            bool ok = issue_qk(0);
            for (int c = 0; ok && c < nchunks; ++c) {
                if (c + 1 < nchunks) ok = issue_qk(c + 1);
                if (ok) ok = issue_pv(c);
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------- V widening
        const int r = tid - 192;  // token row of the tile
        for (int c = 0; c < nchunks; ++c) {
            const int li = 2 * c + 1, st = li % C::NSLOT;
            if (!wait_all(&full[st], (li / C::NSLOT) & 1)) break;
            if (c >= 1 && !wait_all(v16_free, (c - 1) & 1)) break;
            const int rel = c * C::TILE + r;
            const bool valid = tok0 + rel < tok1 && phys[rel / BS] >= 0;
            const unsigned char* src = smem + st * C::SLOT + r * C::ROW;
            unsigned char* dst = smem + C::V16_OFF + r * C::ROW;
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // codes 16j .. 16j+15 (swizzled chunk j of the row)
                uint4 raw = make_uint4(0u, 0u, 0u, 0u);
                if (valid) raw = *reinterpret_cast<const uint4*>(src + ((j ^ (r & 7)) * 16));
                uint4 lo, hi;
                e4m3x4_to_f16x4(raw.x, lo.x, lo.y);
                e4m3x4_to_f16x4(raw.y, lo.z, lo.w);
                e4m3x4_to_f16x4(raw.z, hi.x, hi.y);
                e4m3x4_to_f16x4(raw.w, hi.z, hi.w);
                // f16 dims 16j .. 16j+7 and 16j+8 .. 16j+15: half j / 4, chunks 2(j % 4) and 2(j % 4) + 1
                unsigned char* half = dst + (j >> 2) * C::HALF16;
                const int c0 = 2 * (j & 3);
                *reinterpret_cast<uint4*>(half + ((c0 ^ (r & 7)) * 16)) = lo;
                *reinterpret_cast<uint4*>(half + (((c0 + 1) ^ (r & 7)) * 16)) = hi;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&empty[st]);
                mbar_arrive(v16_full);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int q4 = warp & 3;            // TMEM lane quadrant of this warp
        const int r = q4 * 32 + lane;       // token row of S, dimension row of O
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        float m_run[G], l_run[G], acc[G], alpha_prev[G], qsk[G];
        const float kscale = p.qscale * p.k_scales[g];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m_run[h] = -INFINITY;
            l_run[h] = 0.f;
            acc[h] = 0.f;
            alpha_prev[h] = 1.f;
            qsk[h] = kscale * __uint_as_float((uint32_t)(127 - kq[h]) << 23);
        }
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

            const int rel = c * C::TILE + r;
            const bool valid = tok0 + rel < tok1 && phys[rel / BS] >= 0;
            float x[G];
#pragma unroll
            for (int h = 0; h < G; ++h) x[h] = valid ? (sv[2 * h] + sv[2 * h + 1]) * qsk[h] : -INFINITY;
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
                const __half ph = __float2half_rn(pr);
                l_run[h] = fmaf(l_run[h], alpha[h], __half2float(ph));
                *reinterpret_cast<__half*>(pbuf + th * (C::NPAD * C::ROW) + h * C::ROW +
                                           ((((tr >> 3) ^ (h & 7)) << 4)) + (tr & 7) * 2) = ph;
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
                const float vsc = p.v_scales[g];
#pragma unroll
                for (int h = 0; h < G; ++h) {
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
