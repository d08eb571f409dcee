// decode_tc_fp8p.cuh -- the fp8 (e4m3) tensor-core decode kernel of
// decode_tc_fp8.cuh in persistent form: one CTA per slot (SMs x CTAs per SM),
// each running (sequence, kv head, partition) units one after another from a
// work queue in the workspace, so that a unit's start (table, q, first tiles)
// overlaps the previous unit's end.
//
// Same computation ("PagedAttention Explained: Virtual Memory for the KV
// Cache", section "How PagedAttention works", item 5; "What does
// PagedAttention change in LLM KV allocation?", section "Sharing requires
// more than allocation": supported cache quantization) and the same
// arithmetic as the one-CTA-per-unit kernel: q and the probabilities each as
// two e4m3 terms, QK^T and PV on kind::f8f6f4, fp32 online softmax in base 2,
// the fused split-K merge in partition order, so the outputs are the same
// bits.  Why persistent: with one CTA per unit the hardware hands out units
// in grid order as slots free up, and a long unit that starts late runs on
// while most slots idle; the longest-first grid order helps only as far as
// CTAs start in that order.  Here each CTA takes its next unit from a queue
// in the order of the longest-first schedule (one atomic per unit), so the
// last units handed out are the shortest, and a unit's start-up (queue
// entry, table, q) is hidden behind the running unit.  Parallel-sampling
// batch over an fp8 cache (256 sequences, groups of 4 query heads): 135.7 us
// with one CTA per unit, 124.1 us persistent.  Partitions hold at most 128
// blocks (the two unit records' tables).
//
// Roles (192 threads):
//  * warp 0, producer: takes the next unit with work from the queue, loads
//    its table entries and builds its Q operand (q as two e4m3 terms) into
//    one of two unit records, publishes the record (unit_full), then streams
//    the unit's K and V tiles into the slot ring; the ring and its phases
//    continue across units.
//  * warp 1, lane 0, MMA issuer: per published unit, QK^T and PV of each
//    chunk as their operands are ready; a tcgen05.commit releases the unit's
//    record once its MMAs are done.
//  * warps 2-5, softmax: per unit, the chunks' softmax (cross-warp max
//    through shared memory and an mbarrier), P, the fold of O; then, once
//    all four have come through the unit's bounded waits (one named-barrier
//    vote), the unit's output or partial and, for a split sequence, the
//    fused merge over the four warps on a named barrier; then they release
//    the record.
// Every wait is bounded.  A CTA whose wait runs out lets its copies and MMAs
// land, frees TMEM, and then keeps taking units from the queue without
// computing them, giving each its turn on its merge counter (an empty
// partial), so the merge counters and the queue end the launch at zero.  The
// last CTA to finish resets the queue.
#pragma once

#include "decode_tc_fp8.cuh"
#include "persist.cuh"

namespace pkv {
namespace tc {

// Up to four query heads per kv head (eight heads need more registers than
// a persistent CTA can spare next to four others; their one-CTA-per-unit
// kernel runs two CTAs per SM, where a unit's merge would stall the ring:
// 8-sequence 128K-token batch 332.9 us per unit, 336.7 us persistent).  Two
// slots (one K and one V tile in flight) at five CTAs per SM up to two query
// heads, four CTAs at four (registers).  On B200 more CTAs per SM beat
// deeper rings (batch-64 MHA: 2 slots x 5 CTAs 106.5 us, 2 x 4 110.2, 4 x 3
// 108.9 (index order), 6 x 2 120.3): the chain from a chunk's S to its PV,
// not the bytes in flight, limits a CTA.
template <int BS, int G>
struct TcFp8PCfg {
    static constexpr int D = 128;
    static constexpr int TILE = 128;
    static constexpr int BPT = TILE / BS;
    static constexpr int NPAD = 16;
    static constexpr int ROW = 128;
    static constexpr int SLOT = TILE * ROW;
    static constexpr int CTAS_PER_SM = G >= 4 ? 4 : 5;
    static constexpr int NSLOT = 2;
    static constexpr int QB = NPAD * ROW;      // one Q operand (two per CTA: one per unit record)
    static constexpr int PB = NPAD * ROW;      // one P buffer (rows 2h hi, 2h + 1 lo)
    static constexpr int MAX_PART_BLOCKS = 128;  // two tables per CTA
    static constexpr int MAX_PART_TOKENS = MAX_PART_BLOCKS * BS;
    static constexpr int THREADS = 192;
    static constexpr int NSOFT = 128;
    static constexpr uint32_t TMEM_COLS = 64;
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t O_COL = 32;
    static constexpr int RS = 8;               // stride of a warp's row in the reductions
    // The merge runs when both P buffers are idle (after the unit's last PV
    // completed, before the next unit's first P), so its scratch lies over
    // them when it fits: rows of P past 2G then hold leftovers, which only
    // reach the PV columns that are never read.
    static constexpr int MERGE_BYTES = (merge_scratch_bytes<G, D, NSOFT>() + 15) / 16 * 16;
    static constexpr bool MERGE_IN_P = MERGE_BYTES <= 2 * PB;
    // unit record: ints [0] end, [1] s, [2] g, [3] part, [4] nparts, [5] tok0,
    // [6] tok1, [7] nchunks, [8] nblk
    static constexpr int REC_INTS = 12;
    static constexpr int Q_OFF = NSLOT * SLOT;
    static constexpr int P_OFF = Q_OFF + 2 * QB;
    static constexpr int MRG_OFF = MERGE_IN_P ? P_OFF : P_OFF + 2 * PB;
    static constexpr int BAR_OFF = P_OFF + 2 * PB + (MERGE_IN_P ? 0 : MERGE_BYTES);
    // full[NSLOT] empty[NSLOT] s_full[2] s_free[2] p_full[2] o_full[2] o_free[2]
    // red[2] unit_full[2] unit_free[2] mma_done
    static constexpr int NBARS = 2 * NSLOT + 17;
    // tmem, abort, last flag, units done, units published, fetched unit, queue entry
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int KQ_OFF = MISC_OFF + 32;          // [2][8] per-head logit factors
    static constexpr int RED_OFF = KQ_OFF + 2 * 8 * 4;    // [2][4][RS] chunk maxima, [4][RS] sums
    static constexpr int REC_OFF = RED_OFF + (2 * 4 * RS + 4 * RS) * 4;
    static constexpr int PHYS_OFF = REC_OFF + 2 * REC_INTS * 4;
    static constexpr int SMEM_BYTES = PHYS_OFF + 2 * MAX_PART_BLOCKS * 4 + 1024;
    static constexpr uint32_t IDESC_QK = idesc_make(128, NPAD, 0u, false, false);
    static constexpr uint32_t IDESC_PV = idesc_make(128, NPAD, 0u, true, false);

    static_assert(TILE % BS == 0 && (BS * ROW) % 1024 == 0, "blocks stack on swizzle atoms");
    static_assert(G == 1 || G == 2 || G == 4, "one, two or four query heads per kv head");
    static_assert(Q_OFF % 1024 == 0 && QB % 1024 == 0 && P_OFF % 1024 == 0 && PB % 1024 == 0,
                  "operand alignment");
    static_assert(CTAS_PER_SM * (SMEM_BYTES + 1024) <= 228 * 1024, "CTAs per SM by shared memory");
    static_assert(CTAS_PER_SM * TMEM_COLS <= 512, "CTAs per SM by TMEM");
    static_assert(NSLOT % 2 == 0, "K and V tiles in slots of their own");
};

// Build the Q operand of (s, g) into q_op (16 rows of 128 codes, 128-byte
// swizzle) and the heads' logit factors into qsk, with the 32 lanes of one
// warp: lane l handles rows (l >> 3) + 4i, 16-code piece l & 7.  q is made
// e4m3 as in decode_tc_fp8_kernel: per head a power of two brings max |q|
// into [128, 256), then q = hi + lo / 16.
template <int G>
__device__ __forceinline__ void build_q_warp(const DecodeParams& p, int s, int g, unsigned char* q_op,
                                             float* qsk, int lane) {
    using T = __nv_bfloat16;
    constexpr int D = 128, ROW = 128;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int n = (lane >> 3) + 4 * i, j = lane & 7;
        const int hq = n >> 1;
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
        int kexp = mx > 0.f ? 7 - ((int)((__float_as_uint(mx) >> 23) & 0xffu) - 127) : 0;
        kexp = kexp < -120 ? -120 : (kexp > 120 ? 120 : kexp);
        const float up = __uint_as_float((uint32_t)(127 + kexp) << 23);
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t hw = 0, lw = 0;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const float a = qv[4 * k + 2 * h2] * up, b = qv[4 * k + 2 * h2 + 1] * up;
                const uint32_t hc = f32x2_to_e4m3x2(a, b);
                const float2 hv = e4m3x2_to_f32x2(hc);
                const uint32_t lc = f32x2_to_e4m3x2((a - hv.x) * 16.f, (b - hv.y) * 16.f);
                hw |= hc << (16 * h2);
                lw |= lc << (16 * h2);
            }
            w[k] = (n & 1) ? lw : hw;
        }
        uint4 val = make_uint4(w[0], w[1], w[2], w[3]);
        if (n >= 2 * G) val = make_uint4(0u, 0u, 0u, 0u);
        if (!(mx <= 3.402823466e38f)) val = make_uint4(0x7f7f7f7fu, 0x7f7f7f7fu, 0x7f7f7f7fu, 0x7f7f7f7fu);
        *reinterpret_cast<uint4*>(q_op + n * ROW + ((j ^ (n & 7)) * 16)) = val;
        if (n < 2 * G && (n & 1) == 0 && j == 0)
            qsk[hq] = p.qscale * p.k_scales[g] * __uint_as_float((uint32_t)(127 - kexp) << 23);
    }
}

// FIRST_WAVE: the launch's sequences each fit one partition (see the producer)
template <int BS, int G, bool FIRST_WAVE>
__global__ void __launch_bounds__(192, TcFp8PCfg<BS, G>::CTAS_PER_SM)
    decode_tc_fp8_persistent_kernel(const __grid_constant__ DecodeParams p,
                                    const __grid_constant__ CUtensorMap tmk,
                                    const __grid_constant__ CUtensorMap tmv) {
    using C = TcFp8PCfg<BS, G>;
    using T = __nv_bfloat16;
    constexpr int D = C::D;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

    const int P = p.num_partitions;
    const int PTOK = p.partition_tokens;
    const int max_ctx = p.max_blocks_per_seq * BS;
    const int num_units = p.num_seqs * p.num_kv_heads * P;
    constexpr bool first_wave = FIRST_WAVE;  // see the producer

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::NSLOT;
    uint64_t* s_full = bars + 2 * C::NSLOT;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* o_full = p_full + 2;
    uint64_t* o_free = o_full + 2;
    uint64_t* red_bar = o_free + 2;
    uint64_t* unit_full = red_bar + 2;
    uint64_t* unit_free = unit_full + 2;
    uint64_t* mma_done = unit_free + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
    int* last_flag = reinterpret_cast<int*>(smem + C::MISC_OFF + 8);
    volatile int* units_done = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 12);  // finished by softmax
    volatile int* units_published = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 16);
    volatile int* fetched_unit = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 20);  // taken, not published
    volatile int* queue_entry = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 24);
    float* red_max = reinterpret_cast<float*>(smem + C::RED_OFF);
    float* red_sum = red_max + 2 * 4 * C::RS;
    int* recs = reinterpret_cast<int*>(smem + C::REC_OFF);
    float* merge_scratch = reinterpret_cast<float*>(smem + C::MRG_OFF);

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
            mbar_init(&unit_full[b], 1);
            mbar_init(&unit_free[b], 5);  // the issuer's commit and the four softmax warps
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        *units_done = 0;
        *units_published = 0;
        *fetched_unit = -1;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp >= 2) {  // P buffers start at zero (rows past 2G are never written)
        for (int u = tid - 64; u < 2 * C::PB / 16; u += C::NSOFT)
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

    long long loads_issued = 0;  // producer: tiles issued over all units
    int mma_issued = 0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The first wave (launches where every sequence fits one partition):
        // CTA b's first unit is unit b in index order, taken at once.  Every
        // later unit comes from the queue, which follows the schedule the
        // planning grid writes (longest first) and skips the first wave's
        // units; so the plan runs while the first wave streams, and the units
        // handed out last are still the shortest (batch-64 MHA: 106.5 ->
        // 101.7 us).  With several partitions per sequence the index order
        // would start the short last partitions ahead of long ones (the
        // parallel-sampling batch lost 2 %): there every unit comes from the
        // queue.  Only this warp reads the schedule.
        bool first_pending = first_wave, plan_seen = false;
        for (int k = 0;; ++k) {
            const int rec = k & 1;
            // the next unit with work (its index-order id); units with nothing
            // to attend are settled here
            int u = -1, s = 0, g = 0, part = 0, ctx = 0, nparts = 0;
            for (;;) {
                int idx;
                if (first_pending) {
                    first_pending = false;
                    idx = (int)blockIdx.x;  // the grid never has more CTAs than units
                    index_unit(p, idx, s, g, part);
                } else {
                    if (!plan_seen) {
                        if (p.order != nullptr) asm volatile("griddepcontrol.wait;" ::: "memory");
                        plan_seen = true;
                    }
                    int cand = 0;
                    if (lane == 0) cand = atomicAdd(p.work, 1);
                    cand = __shfl_sync(0xffffffffu, cand, 0);
                    if (cand >= num_units) break;
                    if (!queue_unit(p, cand, s, g, part)) continue;
                    idx = unit_index(p, s, g, part);
                    if (first_wave && idx < (int)gridDim.x) continue;  // a first-wave unit: its CTA has it
                }
                ctx = p.context_lens[s];
                if (ctx < 0 || ctx > max_ctx) {
                    if (part == 0) {
                        if (lane == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
                        zero_rows_warp<G>(p, (long long)s * p.num_heads + (long long)g * G, lane);
                    }
                    continue;
                }
                nparts = (ctx + PTOK - 1) / PTOK;
                if (part >= nparts) {
                    if (ctx == 0 && part == 0)
                        zero_rows_warp<G>(p, (long long)s * p.num_heads + (long long)g * G, lane);
                    continue;
                }
                u = idx;
                break;
            }
            if (lane == 0) *fetched_unit = u;
            if (k >= 2 && !wait_all(&unit_free[rec], ((k >> 1) - 1) & 1)) break;
            int* R = recs + rec * C::REC_INTS;
            if (u < 0) {  // the queue is empty: tell the consumers
                if (lane == 0) {
                    R[0] = 1;
                    *fetched_unit = -1;
                    mbar_arrive(&unit_full[rec]);
                }
                break;
            }
            const int tok0 = part * PTOK;
            const int tok1 = min(ctx, tok0 + PTOK);
            const int nblk = (tok1 - tok0 + BS - 1) / BS;
            const int blk0 = tok0 / BS;
            const int nchunks = (tok1 - tok0 + C::TILE - 1) / C::TILE;
            int* phys = reinterpret_cast<int*>(smem + C::PHYS_OFF) + rec * C::MAX_PART_BLOCKS;
            const int32_t* bt = p.block_tables + (long long)s * p.max_blocks_per_seq + blk0;
            for (int j = lane; j < nblk; j += 32) {
                int e = bt[j];
                if (e < 0 || e >= p.num_blocks) {
                    set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
                    e = -1;
                }
                phys[j] = e;
            }
            build_q_warp<G>(p, s, g, smem + C::Q_OFF + rec * C::QB,
                            reinterpret_cast<float*>(smem + C::KQ_OFF) + rec * 8, lane);
            if (lane == 0) {
                R[0] = 0;
                R[1] = s;
                R[2] = g;
                R[3] = part;
                R[4] = nparts;
                R[5] = tok0;
                R[6] = tok1;
                R[7] = nchunks;
                R[8] = nblk;
            }
            fence_proxy_async_smem();  // the Q operand is read by the tensor cores
            __syncwarp();
            if (lane == 0) {
                *fetched_unit = -1;
                *units_published = k + 1;
                mbar_arrive(&unit_full[rec]);
            }
            // the unit's K and V tiles; the ring's phases continue across units
            bool ok = true;
            for (int li = 0; li < 2 * nchunks; ++li) {
                const long long L = loads_issued + li;
                const int c = li >> 1;
                const CUtensorMap* map = (li & 1) ? &tmv : &tmk;
                const int st = (int)(L % C::NSLOT);
                if (L >= C::NSLOT && !wait_all(&empty[st], (uint32_t)(((L / C::NSLOT) - 1) & 1))) {
                    ok = false;
                    loads_issued = L;
                    break;
                }
                const int j = c * C::BPT + lane;
                const int e = (lane < C::BPT && j < nblk) ? phys[j] : -1;
                const bool load = e >= 0 && PKV_DCHECK(p.err, e < p.num_blocks && st < C::NSLOT &&
                                                                  (lane + 1) * BS * C::ROW <= C::SLOT);
                const int nload = __popc(__ballot_sync(0xffffffffu, load));
                if (lane == 0) {
                    if (nload > 0)
                        mbar_arrive_expect_tx(&full[st], (uint32_t)(nload * BS * C::ROW));
                    else
                        mbar_arrive(&full[st]);
                }
                __syncwarp();
                if (load) tma_load_4d(smem + st * C::SLOT + lane * BS * C::ROW, map, 0, 0, g, e, &full[st]);
            }
            if (!ok) break;
            loads_issued += 2 * nchunks;
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            long long cbase = 0;  // chunks of the units before this one
            for (int k = 0;; ++k) {
                const int rec = k & 1;
                if (!mbar_wait_bounded(&unit_full[rec], (k >> 1) & 1, abort_flag, p.wait_ns)) {
                    set_error(p.err, PKV_ERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                const int* R = recs + rec * C::REC_INTS;
                if (R[0]) break;
                const int nchunks = R[7];
                const uint32_t q_base = smem_addr(smem + C::Q_OFF + rec * C::QB);
                int nq = 0, np = 0;
                bool ok = true;
                unsigned long long t_last = globaltimer_ns();
                while (np < nchunks) {
                    bool progressed = false;
                    if (nq < nchunks) {
                        const long long cq = cbase + nq;
                        const long long li = 2 * cq;
                        const int st = (int)(li % C::NSLOT);
                        if (mbar_test(&full[st], (uint32_t)((li / C::NSLOT) & 1)) &&
                            (cq < 2 || mbar_test(&s_free[cq & 1], (uint32_t)(((cq >> 1) - 1) & 1)))) {
                            tc_fence_after();
                            const uint32_t k_base = smem_addr(smem + st * C::SLOT);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t a = sw128_desc(k_base + kk * 32, 16, 1024);
                                const uint64_t b = sw128_desc(q_base + kk * 32, 16, 1024);
                                mma_kind_f8f6f4(tmem + C::S_COL + (cq & 1) * 16, a, b, C::IDESC_QK, kk > 0);
                            }
                            mma_commit(&s_full[cq & 1]);
                            mma_commit(&empty[st]);
                            ++nq;
                            ++mma_issued;
                            progressed = true;
                        }
                    }
                    if (np < nq) {
                        const long long cp = cbase + np;
                        const long long li = 2 * cp + 1;
                        const int st = (int)(li % C::NSLOT);
                        if (mbar_test(&full[st], (uint32_t)((li / C::NSLOT) & 1)) &&
                            mbar_test(&p_full[cp & 1], (uint32_t)((cp >> 1) & 1)) &&
                            (cp < 2 || mbar_test(&o_free[cp & 1], (uint32_t)(((cp >> 1) - 1) & 1)))) {
                            tc_fence_after();
                            const uint32_t v_base = smem_addr(smem + st * C::SLOT);
                            const uint32_t p_base = smem_addr(smem + C::P_OFF + (cp & 1) * C::PB);
                            const uint32_t o_col = tmem + C::O_COL + (cp & 1) * 16;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t a = sw128_desc(v_base + kk * 32 * C::ROW, 16, 1024);
                                const uint64_t b = sw128_desc(p_base + kk * 32, 16, 1024);
                                mma_kind_f8f6f4(o_col, a, b, C::IDESC_PV, kk > 0);
                            }
                            mma_commit(&o_full[cp & 1]);
                            mma_commit(&empty[st]);
                            ++np;
                            ++mma_issued;
                            progressed = true;
                        }
                    }
                    if (progressed) {
                        t_last = globaltimer_ns();
                    } else {
                        if (*abort_flag) {
                            ok = false;
                            break;
                        }
                        if (globaltimer_ns() - t_last > p.wait_ns) {
                            set_error(p.err, PKV_ERR_TIMEOUT);
                            *abort_flag = 1;
                            ok = false;
                            break;
                        }
                    }
                }
                if (!ok) break;
                mma_commit(&unit_free[rec]);  // the record's Q is free once these MMAs are done
                cbase += nchunks;
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const int st_tid = tid - 64;  // 0..127 among the softmax threads
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        long long cbase = 0;    // chunks of the units before this one
        unsigned red_use = 0;   // red_bar uses so far
        // The four softmax warps meet once per unit, after its last bounded
        // wait, and go on with the unit's output and merge only if all of
        // them got there without giving up: the merge (and its turn on the
        // counter) is then taken by all four or by none, with hardware
        // barriers that nothing outside these warps can hold up.
        auto agree = [&](bool mine) -> bool {
            __syncwarp();
            return soft_bar_and(mine);
        };
        auto merge_sync = [] {
            soft_bar_sync();
            return true;
        };
        for (int k = 0;; ++k) {
            const int rec = k & 1;
            const int* R = recs + rec * C::REC_INTS;
            bool ok = wait_all(&unit_full[rec], (k >> 1) & 1);
            if (ok && R[0]) {  // the queue is empty
                agree(false);
                break;
            }
            const int s = ok ? R[1] : 0, g = ok ? R[2] : 0, part = ok ? R[3] : 0, nparts = ok ? R[4] : 1;
            const int tok0 = ok ? R[5] : 0, tok1 = ok ? R[6] : 0;
            const int nchunks = ok ? R[7] : 0;
            const int* phys = reinterpret_cast<const int*>(smem + C::PHYS_OFF) + rec * C::MAX_PART_BLOCKS;
            const float* qsk = reinterpret_cast<const float*>(smem + C::KQ_OFF) + rec * 8;
            float m_run[G], l_run[G], acc[G], alpha_prev[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m_run[h] = -INFINITY;
                l_run[h] = 0.f;
                acc[h] = 0.f;
                alpha_prev[h] = 1.f;
            }
            auto fold = [&](long long cc, const float* alpha) -> bool {
                if (!wait_all(&o_full[cc & 1], (uint32_t)((cc >> 1) & 1))) return false;
                tc_fence_after();
                float ov[2 * G];
                tmem_ld_first<2 * G>(lane_addr + C::O_COL + (cc & 1) * 16, ov);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_free[cc & 1]);
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] = fmaf(acc[h], alpha[h], fmaf(ov[2 * h + 1], 0.0625f, ov[2 * h]));
                return true;
            };
            for (int c = 0; c < nchunks && ok; ++c) {
                const long long C_ = cbase + c;
                if (!wait_all(&s_full[C_ & 1], (uint32_t)((C_ >> 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float sv[2 * G];
                tmem_ld_first<2 * G>(lane_addr + C::S_COL + (C_ & 1) * 16, sv);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[C_ & 1]);
                const int rel = c * C::TILE + r;
                const bool valid = tok0 + rel < tok1 && phys[rel / BS] >= 0;
                float x[G];
#pragma unroll
                for (int h = 0; h < G; ++h)
                    x[h] = valid ? fmaf(sv[2 * h + 1], 0.0625f, sv[2 * h]) * qsk[h] : -INFINITY;
                float* rm = red_max + (red_use & 1) * 4 * C::RS;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float v = warp_max(x[h]);
                    if (lane == 0) rm[q4 * C::RS + h] = v;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&red_bar[red_use & 1]);
                if (!wait_all(&red_bar[red_use & 1], (red_use >> 1) & 1)) {
                    ok = false;
                    break;
                }
                ++red_use;
                constexpr int GP = G + (G & 1);
                float alpha[G], pr[GP];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float mc = fmaxf(fmaxf(rm[h], rm[C::RS + h]), fmaxf(rm[2 * C::RS + h], rm[3 * C::RS + h]));
                    const float m_new = fmaxf(m_run[h], mc);
                    alpha[h] = m_new == -INFINITY ? 1.f : exp2f(m_run[h] - m_new);
                    m_run[h] = m_new;
                    pr[h] = valid ? exp2f(x[h] - m_new) * 256.f : 0.f;
                }
                if constexpr (GP > G) pr[G] = 0.f;
                unsigned char* pbuf = smem + C::P_OFF + (C_ & 1) * C::PB;
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
                        const int rh = 2 * hh, rl = 2 * hh + 1;
                        pbuf[rh * C::ROW + (((r >> 4) ^ (rh & 7)) << 4) + (r & 15)] = (unsigned char)(hc >> (8 * u));
                        pbuf[rl * C::ROW + (((r >> 4) ^ (rl & 7)) << 4) + (r & 15)] = (unsigned char)(lc >> (8 * u));
                    }
                }
                {  // the V tile must have landed; rows that are not tokens get zero codes
                    const long long li = 2 * C_ + 1;
                    const int st = (int)(li % C::NSLOT);
                    if (!wait_all(&full[st], (uint32_t)((li / C::NSLOT) & 1))) {
                        ok = false;
                        break;
                    }
                    if (!valid) {
                        uint4* row = reinterpret_cast<uint4*>(smem + st * C::SLOT + r * C::ROW);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) row[kk] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[C_ & 1]);
                if (c >= 1 && !fold(C_ - 1, alpha_prev)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int h = 0; h < G; ++h) alpha_prev[h] = alpha[h];
            }
            if (ok && nchunks > 0) ok = fold(cbase + nchunks - 1, alpha_prev);
            if (ok) {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float v = l_run[h];
#pragma unroll
                    for (int msk = 16; msk; msk >>= 1) v += __shfl_xor_sync(0xffffffffu, v, msk);
                    if (lane == 0) red_sum[q4 * C::RS + h] = v;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&red_bar[red_use & 1]);
                ok = wait_all(&red_bar[red_use & 1], (red_use >> 1) & 1);
                ++red_use;
            }
            if (!agree(ok)) break;
            {
                const int H = p.num_heads;
                const long long sh0 = (long long)s * H + (long long)g * G;
                const float vsc = p.v_scales[g] * 0.00390625f;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    if (!PKV_DCHECK(p.err, sh0 + h < (long long)p.num_seqs * H && part < P)) continue;
                    const float L = (red_sum[h] + red_sum[C::RS + h]) +
                                    (red_sum[2 * C::RS + h] + red_sum[3 * C::RS + h]);
                    const float O = acc[h] * vsc;
                    if (nparts == 1) {
                        Elem<T>::store(static_cast<T*>(p.out) + (sh0 + h) * D + r, L > 0.f ? O / L : 0.f);
                    } else {
                        p.ws_o[((sh0 + h) * P + part) * D + r] = O;
                        if (r == 0) p.ws_ml[(sh0 + h) * P + part] = make_float2(m_run[h], L);
                    }
                }
                if (nparts > 1)
                    fused_merge_with<T, D, G, C::NSOFT>(p, s, g, nparts, sh0, merge_scratch, last_flag, st_tid,
                                                        merge_sync);
            }
            __syncwarp();
            if (lane == 0) {
                if (warp == 2) *units_done = k + 1;  // before the record can be reused
                mbar_arrive(&unit_free[rec]);
            }
            cbase += nchunks;
        }
    }

    tc_fence_before();
    __syncthreads();
    const bool aborted = *abort_flag != 0;
    // let this CTA's copies (after an abort) and MMAs land, then free TMEM
    if (aborted && warp == 0 && lane == 0) {
        for (long long li = loads_issued - C::NSLOT > 0 ? loads_issued - C::NSLOT : 0; li < loads_issued; ++li) {
            const int st = (int)(li % C::NSLOT);
            const unsigned long long t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[st], (uint32_t)((li / C::NSLOT) & 1)))
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
    if (aborted) {
        // every unit this CTA took and did not finish, then every unit left in
        // the queue, takes its turn on its merge counter with an empty partial
        if (p.order != nullptr) asm volatile("griddepcontrol.wait;" ::: "memory");
        const int first = *units_done, published = *units_published;
        const int orphan = *fetched_unit;  // index-order id, or -1
        __syncthreads();
        for (int k = first; k < published; ++k) {
            const int* R = recs + (k & 1) * C::REC_INTS;
            abort_merge_turn<T, D, G>(p, R[1], R[2], (long long)R[1] * p.num_heads + (long long)R[2] * G,
                                      R[3], R[4], last_flag);
        }
        // first the unit taken and not published, then the queue's entries
        // (whose first-wave units their own CTAs settle)
        for (int u = orphan, from_queue = 0;;) {
            int s = 0, g = 0, part = 0;
            bool take = false;
            if (from_queue) {
                take = u < num_units && queue_unit(p, u, s, g, part) &&
                       !(first_wave && unit_index(p, s, g, part) < (int)gridDim.x);
            } else if (u >= 0 && u < num_units) {
                index_unit(p, u, s, g, part);
                take = true;
            }
            if (take) {
                const int ctx = p.context_lens[s];
                const bool bad = ctx < 0 || ctx > max_ctx;
                const int nparts = bad ? 0 : (ctx + PTOK - 1) / PTOK;
                if (!bad && part < nparts)
                    abort_merge_turn<T, D, G>(p, s, g, (long long)s * p.num_heads + (long long)g * G, part,
                                              nparts, last_flag);
                else if (part == 0 && (bad || ctx == 0))
                    zero_rows<T, D, G>(p, (long long)s * p.num_heads + (long long)g * G);
            }
            __syncthreads();
            if (tid == 0) *queue_entry = atomicAdd(p.work, 1);
            __syncthreads();
            u = *queue_entry;
            from_queue = 1;
            if (u >= num_units) break;
        }
    }
    // the last CTA of the launch resets the queue for the next launch
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(p.work + 1, 1) == (int)gridDim.x - 1) {
            p.work[0] = 0;
            p.work[1] = 0;
            __threadfence();
        }
    }
}

}  // namespace tc
}  // namespace pkv
