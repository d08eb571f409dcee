// decode_tc_fp8_d64.cuh -- tensor-core (tcgen05 + TMEM) paged decode attention
// over fp8 (e4m3) K and V pools with head_dim 64: one CTA per (sequence, pair
// of kv heads, partition), 1, 2 or 4 query heads per kv head, bf16 q and out.
//
// Same computation and arithmetic as decode_tc_fp8.cuh ("PagedAttention
// Explained: Virtual Memory for the KV Cache", section "How PagedAttention
// works", item 5, over a quantised cache: "What does PagedAttention change in
// LLM KV allocation?", section "Sharing requires more than allocation"): q and
// the probabilities each as two e4m3 terms, both products on kind::f8f6f4,
// fp32 online softmax in base 2, the fused split-K merge in partition order.
//
// Why pairs.  The PV product reads the V tile as its MN-major A operand with
// M = 128 rows of O, and one head has only 64 dims; two kv heads of the same
// sequence (the same tokens, the same block table) fill the 128 rows.  A
// token's two 64-code rows need not sit side by side: each head's rows form
// their own 64-byte swizzled tile, and the operand's descriptor steps from
// one head's rows to the other's.
//  * Tile layout.  One copy per block: a 5-D tensor map over the pool
//    (64 codes, 8 slots, kv head, group of 8 slots, block) whose box (64, 8,
//    2, bs / 8, 1) lands, for each group of 8 tokens, 8 rows of the first
//    head and then 8 rows of the second (64-byte rows, 64-byte swizzle):
//    group q of the chunk at 1024 q, head h at + 512 h, token row i at + 64 i.
//  * S^T = K . Q^T over both heads at once: the reduction runs over 128
//    "dims", the first head's 64 and then the second's (each K step of 32
//    codes starts in one head's tile), and Q^T is block structured: the
//    columns of a head of the first kv head hold its q in the first 64 dims
//    and zeros in the rest, those of the second the other way round.  So
//    column 2h' + t of S is the first head's logit term for h' < G and the
//    second's for h' >= G: one softmax over 2G heads, exactly as the
//    head_dim-128 kernel runs it over G.
//  * O^T = V^T . P^T: rows 0-63 of O are the first head's dims, rows 64-127
//    the second's; columns 2h' + t hold every head's P term.  A thread of O
//    row r reads only the columns of its own head (r < 64: heads h' < G).
//    The other products (a head's V against the other head's P) are computed
//    and never read.
// Roles, rings, waits, the abort path and the merge are those of
// decode_tc_fp8_kernel.
#pragma once

#include "decode_tc_fp8.cuh"

namespace pkv {
namespace tc {

template <int BS, int G>
struct TcFp8D64Cfg {
    static constexpr int D = 64;
    static constexpr int GP = 2 * G;          // query heads of the pair
    static constexpr int TILE = 128;          // tokens per chunk
    static constexpr int BPT = TILE / BS;     // blocks per chunk
    static constexpr int NPAD = 16;           // MMA N: 2 GP columns used
    static constexpr int ROW = 64;            // bytes of one head's token row
    static constexpr int GROUP = 2 * 8 * ROW; // 8 tokens of both heads (1024 B)
    static constexpr int SLOT = TILE * 2 * ROW;  // one K or V pair tile (16 KB)
    static constexpr int BLOCK_BYTES = BS * 2 * ROW;
    // registers: up to 2 heads in the softmax 5 CTAs per SM, 4 heads 4, 8 heads 2
    static constexpr int CTAS_PER_SM = GP >= 8 ? 2 : (GP >= 4 ? 4 : 5);
    static constexpr int NSLOT = CTAS_PER_SM == 2 ? 6 : 2;
    static constexpr int QPART = NPAD * ROW;  // Q^T dims of one head of the pair: 16 rows x 64 codes
    static constexpr int QB = 2 * QPART;
    static constexpr int PROW = 128;          // P^T rows: 128 token codes, 128-byte swizzle
    static constexpr int PB = NPAD * PROW;
    static constexpr int MAX_PART_BLOCKS = 4096 / BS;
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 64;
    static constexpr uint32_t S_COL = 0;      // two S buffers at columns 0 and 16
    static constexpr uint32_t O_COL = 32;     // two O buffers at 32 and 48
    static constexpr int Q_OFF = NSLOT * SLOT;
    static constexpr int P_OFF = Q_OFF + QB;
    static constexpr int BAR_OFF = P_OFF + 2 * PB;
    // full[NSLOT] empty[NSLOT] s_full[2] s_free[2] p_full[2] o_full[2] o_free[2] red[2] mma_done
    static constexpr int NBARS = 2 * NSLOT + 13;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;   // tmem address, abort, last flag
    static constexpr int KQ_OFF = MISC_OFF + 16;           // per-head logit factor (float)
    static constexpr int RED_OFF = KQ_OFF + 8 * 4;         // [2][4][8] chunk maxima, [4][8] sums
    static constexpr int RS = 8;
    static constexpr int PHYS_OFF = RED_OFF + (2 * 4 * RS + 4 * RS) * 4;
    static constexpr int SMEM_BYTES = PHYS_OFF + MAX_PART_BLOCKS * 4 + 1024;
    static constexpr uint32_t IDESC_QK = idesc_make(128, NPAD, 0u, false, false);
    static constexpr uint32_t IDESC_PV = idesc_make(128, NPAD, 0u, true, false);

    static_assert(BS % 8 == 0 && TILE % BS == 0, "blocks are whole groups of 8 tokens");
    static_assert(2 * GP <= NPAD && GP <= RS, "hi and lo columns of every head fit the MMA N");
    static_assert(Q_OFF % 1024 == 0 && P_OFF % 1024 == 0 && PB % 1024 == 0 && QPART % 512 == 0,
                  "operand alignment");
    static_assert(merge_scratch_bytes<GP, D, THREADS>() <= NSLOT * SLOT, "merge scratch reuses the ring");
    static_assert(CTAS_PER_SM * (SMEM_BYTES + 1024) <= 228 * 1024, "CTAs per SM by shared memory");
    static_assert(CTAS_PER_SM * TMEM_COLS <= 512, "CTAs per SM by TMEM");
    static_assert(NSLOT % 2 == 0, "K and V tiles in slots of their own");
};

// Shared-memory matrix descriptor with the 64-byte swizzle (layout type 4).
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= 4ull << 61;
    return d;
}

template <int BS, int G>
__global__ void __launch_bounds__(192, TcFp8D64Cfg<BS, G>::CTAS_PER_SM)
    decode_tc_fp8_d64_kernel(const __grid_constant__ DecodeParams p,
                             const __grid_constant__ CUtensorMap tmk,
                             const __grid_constant__ CUtensorMap tmv) {
    using C = TcFp8D64Cfg<BS, G>;
    using T = __nv_bfloat16;
    constexpr int D = C::D;
    constexpr int GP = C::GP;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

    const int P = p.num_partitions;
    const int npairs = p.num_kv_heads / 2;
    const Unit unit = decode_unit(p, P <= 4, npairs);
    if (unit.s < 0) return;
    const int part = unit.part, s = unit.s;
    const int g0 = 2 * unit.g;  // first kv head of the pair
    const int ctx = unit.ctx;
    const int max_ctx = p.max_blocks_per_seq * BS;
    const long long sh0 = (long long)s * p.num_heads + (long long)g0 * G;
    if (ctx < 0 || ctx > max_ctx) {
        if (part == 0) {
            if (threadIdx.x == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            zero_rows<T, D, GP>(p, sh0);
        }
        return;
    }
    const int PTOK = p.partition_tokens;
    const int nparts = (ctx + PTOK - 1) / PTOK;
    if (part >= nparts) {
        if (ctx == 0 && part == 0) zero_rows<T, D, GP>(p, sh0);
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
    float* qsk = reinterpret_cast<float*>(smem + C::KQ_OFF);       // [GP]
    float* red_max = reinterpret_cast<float*>(smem + C::RED_OFF);  // [2][4][RS]
    float* red_sum = red_max + 2 * 4 * C::RS;                      // [4][RS]
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
        // Q^T operand, two 64-code parts (one per kv head of the pair), rows
        // n = 2h' + term of query head h' of the pair; a row holds its head's
        // q in the part of its own kv head and zeros in the other.  Thread t
        // writes 16 codes: part t / 64, row (t / 4) % 16, codes 16 (t % 4)...
        const int t = tid - 64;
        const int part_k = t >> 6, n = (t >> 2) & 15, c = t & 3;
        const int hq = n >> 1;                    // query head within the pair
        const bool mine = n < 2 * GP && hq / G == part_k;
        float qv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) qv[e] = 0.f;
        if (mine) {
            const uint4* qrow = reinterpret_cast<const uint4*>(
                static_cast<const T*>(p.q) + (sh0 + hq) * D + c * 16);
            Elem<T>::unpack(qrow[0], qv);
            Elem<T>::unpack(qrow[1], qv + 8);
        }
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(qv[e]));
#pragma unroll
        for (int msk = 1; msk < 4; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
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
        if (!mine) val = make_uint4(0u, 0u, 0u, 0u);
        if (mine && !(mx <= 3.402823466e38f)) val = make_uint4(0x7f7f7f7fu, 0x7f7f7f7fu, 0x7f7f7f7fu, 0x7f7f7f7fu);
        // 64-byte swizzle: 16-byte chunk c of row n at chunk c ^ ((n / 2) % 4)
        *reinterpret_cast<uint4*>(smem + C::Q_OFF + part_k * C::QPART + n * C::ROW +
                                  ((c ^ ((n >> 1) & 3)) * 16)) = val;
        if (mine && (n & 1) == 0 && c == 0)
            qsk[hq] = p.qscale * p.k_scales[g0 + part_k] * __uint_as_float((uint32_t)(127 - kexp) << 23);
        for (int u = t; u < 2 * C::PB / 16; u += 128)
            reinterpret_cast<uint4*>(smem + C::P_OFF)[u] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        const bool ok = mbar_wait_bounded(bar, parity, abort_flag, p.wait_ns);
        if (__all_sync(0xffffffffu, ok)) return true;
        if (lane == 0) {
            set_error(p.err, PKV_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        return false;
    };

    int issued = 0;
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
            const bool load = e >= 0 && PKV_DCHECK(p.err, e < p.num_blocks && g0 + 1 < p.num_kv_heads &&
                                                              st < C::NSLOT &&
                                                              (lane + 1) * C::BLOCK_BYTES <= C::SLOT);
            const int nload = __popc(__ballot_sync(0xffffffffu, load));
            if (lane == 0) {
                if (nload > 0)
                    mbar_arrive_expect_tx(&full[st], (uint32_t)(nload * C::BLOCK_BYTES));
                else
                    mbar_arrive(&full[st]);
            }
            __syncwarp();
            if (load) tma_load_5d(smem + st * C::SLOT + lane * C::BLOCK_BYTES, map, 0, 0, g0, 0, e, &full[st]);
            issued = li + 1;
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t q_base = smem_addr(smem + C::Q_OFF);
            int nq = 0, np = 0;
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
                        for (int kk = 0; kk < 4; ++kk) {
                            // 32 codes per step: steps 0, 1 in the first head's rows, 2, 3 in the second's
                            const int h = kk >> 1, off = (kk & 1) * 32;
                            const uint64_t a = sw64_desc(k_base + h * 512 + off, 16, C::GROUP);
                            const uint64_t b = sw64_desc(q_base + h * C::QPART + off, 16, 512);
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
                            // A = V^T, MN-major: the two heads' 64 dims are the two
                            // 64-byte atoms along M (512 B apart), 8-token groups
                            // 1024 B apart, 32 tokens per step
                            const uint64_t a = sw64_desc(v_base + kk * 4 * C::GROUP, 512, C::GROUP);
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
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;       // token row of S; row of O: dim r % 64 of head r / 64
        const int hsel = r >> 6;            // kv head of the pair this thread's O row belongs to
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        float m_run[GP], l_run[GP], acc[G], alpha_prev[GP];
#pragma unroll
        for (int h = 0; h < GP; ++h) {
            m_run[h] = -INFINITY;
            l_run[h] = 0.f;
            alpha_prev[h] = 1.f;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = 0.f;
        auto fold = [&](int cc, const float* alpha) -> bool {
            if (!wait_all(&o_full[cc & 1], (cc >> 1) & 1)) return false;
            tc_fence_after();
            float ov[2 * GP];
            tmem_ld_first<2 * GP>(lane_addr + C::O_COL + (cc & 1) * 16, ov);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[cc & 1]);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float oh = hsel ? ov[2 * (G + h)] : ov[2 * h];
                const float ol = hsel ? ov[2 * (G + h) + 1] : ov[2 * h + 1];
                const float a = hsel ? alpha[G + h] : alpha[h];
                acc[h] = fmaf(acc[h], a, fmaf(ol, 0.0625f, oh));
            }
            return true;
        };
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            if (!wait_all(&s_full[c & 1], (c >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[2 * GP];
            tmem_ld_first<2 * GP>(lane_addr + C::S_COL + (c & 1) * 16, sv);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[c & 1]);

            const int rel = c * C::TILE + r;
            const bool valid = tok0 + rel < tok1 && phys[rel / BS] >= 0;
            float x[GP];
#pragma unroll
            for (int h = 0; h < GP; ++h)
                x[h] = valid ? fmaf(sv[2 * h + 1], 0.0625f, sv[2 * h]) * qsk[h] : -INFINITY;
            float* rm = red_max + (c & 1) * 4 * C::RS;
#pragma unroll
            for (int h = 0; h < GP; ++h) {
                const float v = warp_max(x[h]);
                if (lane == 0) rm[q4 * C::RS + h] = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_bar[c & 1]);
            if (!wait_all(&red_bar[c & 1], (c >> 1) & 1)) {
                ok = false;
                break;
            }
            float alpha[GP], pr[GP];
#pragma unroll
            for (int h = 0; h < GP; ++h) {
                const float mc = fmaxf(fmaxf(rm[h], rm[C::RS + h]), fmaxf(rm[2 * C::RS + h], rm[3 * C::RS + h]));
                const float m_new = fmaxf(m_run[h], mc);
                alpha[h] = m_new == -INFINITY ? 1.f : exp2f(m_run[h] - m_new);
                m_run[h] = m_new;
                pr[h] = valid ? exp2f(x[h] - m_new) * 256.f : 0.f;
            }
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
                    const float rep = (u ? fmaf(lv.y, 0.0625f, hv.y) : fmaf(lv.x, 0.0625f, hv.x)) * 0.00390625f;
                    l_run[hh] = fmaf(l_run[hh], alpha[hh], rep);
                    const int rh = 2 * hh, rl = 2 * hh + 1;
                    pbuf[rh * C::PROW + (((r >> 4) ^ (rh & 7)) << 4) + (r & 15)] = (unsigned char)(hc >> (8 * u));
                    pbuf[rl * C::PROW + (((r >> 4) ^ (rl & 7)) << 4) + (r & 15)] = (unsigned char)(lc >> (8 * u));
                }
            }
            {  // the V tile must have landed; both heads' rows of a token that is not valid get zero codes
                const int li = 2 * c + 1, st = li % C::NSLOT;
                if (!wait_all(&full[st], (li / C::NSLOT) & 1)) {
                    ok = false;
                    break;
                }
                if (!valid) {
                    unsigned char* row = smem + st * C::SLOT + (r >> 3) * C::GROUP + (r & 7) * C::ROW;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            reinterpret_cast<uint4*>(row + h * 512)[k] = make_uint4(0u, 0u, 0u, 0u);
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
            for (int h = 0; h < GP; ++h) alpha_prev[h] = alpha[h];
        }
        if (ok && nchunks > 0) ok = fold(nchunks - 1, alpha_prev);
        if (ok) {
#pragma unroll
            for (int h = 0; h < GP; ++h) {
                float v = l_run[h];
#pragma unroll
                for (int msk = 16; msk; msk >>= 1) v += __shfl_xor_sync(0xffffffffu, v, msk);
                if (lane == 0) red_sum[q4 * C::RS + h] = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_bar[nchunks & 1]);
            if (wait_all(&red_bar[nchunks & 1], (nchunks >> 1) & 1)) {
                const int H = p.num_heads;
                const float vsc = p.v_scales[g0 + hsel] * 0.00390625f;
                const int d = r & 63;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const int hh = hsel * G + h;  // query head within the pair
                    if (!PKV_DCHECK(p.err, sh0 + hh < (long long)p.num_seqs * H && part < P)) continue;
                    const float L = hsel ? (red_sum[G + h] + red_sum[C::RS + G + h]) +
                                               (red_sum[2 * C::RS + G + h] + red_sum[3 * C::RS + G + h])
                                         : (red_sum[h] + red_sum[C::RS + h]) +
                                               (red_sum[2 * C::RS + h] + red_sum[3 * C::RS + h]);
                    const float O = acc[h] * vsc;
                    if (nparts == 1) {
                        Elem<T>::store(static_cast<T*>(p.out) + (sh0 + hh) * D + d, L > 0.f ? O / L : 0.f);
                    } else {
                        p.ws_o[((sh0 + hh) * P + part) * D + d] = O;
                        if (d == 0) {
                            const float m = hsel ? m_run[G + h] : m_run[h];
                            p.ws_ml[(sh0 + hh) * P + part] = make_float2(m, L);
                        }
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
        abort_merge_turn<T, D, GP>(p, s, g0, sh0, part, nparts, last_flag);
        return;
    }
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
    if (nparts == 1) return;
    fused_merge<T, D, GP, C::THREADS>(p, s, g0, nparts, sh0, reinterpret_cast<float*>(smem), last_flag);
}

}  // namespace tc
}  // namespace pkv
