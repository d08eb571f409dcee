// decode_attn.cuh -- block-aware paged decode attention for sm_100a.
//
// Implements the attention computation of "PagedAttention Explained: Virtual
// Memory for the KV Cache" (section "How PagedAttention works", item 5: the
// kernel follows the block table and gathers keys and values from
// non-contiguous blocks) for one decode query per sequence:
//     out[s][h] = softmax(scale * q[s][h] . K_s^T) V_s
// with K_s, V_s the first context_lens[s] tokens of sequence s, token t in
// physical block block_tables[s][t / bs] at slot t % bs (items 2-3).
//
// Design (B200):
//  * One CTA per (sequence, kv head, context partition).  A partition is a
//    fixed number of tokens (split-K); the CTA computes the partial softmax
//    state of every query head of the kv head's group, so each K/V byte is
//    read from HBM once per group (grouped-query attention).
//  * A producer warp walks the partition's block-table entries (loaded once
//    into shared memory and range-checked) and streams each physical block's
//    K slice and V slice -- contiguous bs*head_dim runs in the
//    [block][kv_head][slot][dim] pool -- into a ring of shared-memory stages
//    with bulk copies on the TMA engine, completing on mbarriers.  Enough
//    stages are kept in flight (~64 KB per CTA, 3 CTAs per SM) to cover HBM
//    latency; no multicast.
//  * Four "block lanes" of consumer warps take the staged blocks round-robin;
//    when the group has more than four heads, several warps share a block,
//    each with four heads.  Lane l owns one 16-byte chunk of the head
//    dimension and a subset of the rows, keeps q (pre-scaled by scale*log2 e)
//    for its chunk in registers, and accumulates partial dot products; a
//    transposing butterfly (each step halves the values a lane keeps) turns
//    them into full logits with few shuffles.  Online softmax in base 2 with
//    fp32 running max / sum, then PV into fp32 registers.
//  * Warps merge their (m, l, o) states through shared memory; a sequence
//    that fits one partition is normalised and written directly, otherwise
//    the partition's (m, l, o) go to the workspace and the last partition CTA
//    of the (sequence, kv head) to finish -- found with one atomicInc on a
//    per-group counter that wraps back to zero -- merges all of them in
//    partition order.  Which CTA merges never changes the arithmetic order,
//    which depends only on logical token positions, so outputs are
//    bit-identical under any physical placement of the blocks and across
//    runs.
//  * Faults never trap: a bad table entry or context length sets the device
//    error word and is skipped or zero-filled; every mbarrier wait is bounded.
#pragma once

#include <math.h>

#include "decode_common.cuh"

namespace pkv {

// T: type of q and out; TKV: type of the cached K and V (T, or fp8 e4m3).
template <typename T, typename TKV, int D, int BS, int G>
struct DecodeCfg {
    static constexpr int EPC = Elem<TKV>::kPer16B;
    static constexpr int GW = G < (EPC > 8 ? 2 : 4) ? G : (EPC > 8 ? 2 : 4);  // query heads per warp
    static constexpr int NHS = G / GW;        // warps sharing one staged block
    static constexpr int CPR = D / EPC;        // 16-byte chunks per row
    static constexpr int RPI = 32 / CPR;       // rows covered by one warp-wide load
    // tokens per stage: 16 (two bs-8 blocks, a bs-16 block or half of a bs-32
    // block), 32 for one-byte (fp8) caches so a stage still carries 4 KB of K
    static constexpr int ST = sizeof(TKV) == 1 ? 32 : 16;
    static constexpr uint32_t FULL_ROWS = ST == 32 ? 0xffffffffu : ((1u << ST) - 1u);
    static constexpr int TR = ST;              // rows per sub-tile (one stage)
    static constexpr int BPS = BS < ST ? ST / BS : 1;  // whole blocks per stage
    static constexpr int RPL = TR / RPI;       // rows per lane per sub-tile
    static constexpr int V = GW * RPL;         // partial logits per lane before the butterfly
    static constexpr int VPL = V >= CPR ? V / CPR : 1;  // logits per lane after it
    static constexpr int HLANES = CPR / GW;    // lanes of one head inside a row group
    static constexpr int NBL = 4;              // block lanes
    static constexpr int NCW = NBL * NHS;      // consumer warps
    static constexpr int THREADS = (NCW + 1) * 32;
    static constexpr int ROWB = D * (int)sizeof(TKV);     // bytes of one token row
    static constexpr int SLICE = BS * ROWB;               // bytes of one (block, kv head)
    static constexpr int STAGE_K = ST * ROWB;             // K rows of one stage
    static constexpr int STAGE = 2 * STAGE_K;             // K rows + V rows
    static constexpr int NST_RAW = (64 * 1024) / STAGE;
    static constexpr int NST = NST_RAW < NBL ? NBL : (NST_RAW > 16 ? 16 : NST_RAW);
    static constexpr int MAX_PART_TOKENS = 4096;
    static constexpr int MAX_PART_BLOCKS = MAX_PART_TOKENS / BS;
    static constexpr int STAGES_BYTES = NST * STAGE;
    static constexpr int MERGE_FLOATS = NBL * G * (D + 2);
    static constexpr int PSCR_FLOATS = NCW * RPI * RPL * GW;
    static constexpr int BAR_OFF = STAGES_BYTES;
    static constexpr int PHYS_OFF = BAR_OFF + 2 * NST * 8;
    static constexpr int PSCR_OFF = PHYS_OFF + MAX_PART_BLOCKS * 4;
    static constexpr int FLAG_OFF = PSCR_OFF + PSCR_FLOATS * 4;
    static constexpr int SMEM_BYTES = FLAG_OFF + 16;
    // fused merge scratch after the merge area
    static constexpr int MERGE_SCRATCH_BYTES =
        MERGE_FLOATS * 4 + ((2 * G + 3) / 4) * 16 + (THREADS > G * D / 4 ? THREADS : G * D / 4) * 16;

    static_assert(D % EPC == 0 && CPR <= 32 && 32 % CPR == 0, "head_dim chunking");
    static_assert(TR % RPI == 0 && RPL >= 1, "rows per lane");
    static_assert(NST % NBL == 0, "a stage always feeds the same block lane");
    static_assert(GW <= CPR, "a lane's logits after the butterfly belong to one head");
    static_assert(MERGE_FLOATS * 4 <= STAGES_BYTES, "merge area reuses the stages");
    static_assert(MERGE_SCRATCH_BYTES <= STAGES_BYTES, "fused merge scratch reuses the stages");
    static_assert(STAGE_K % 16 == 0 && SLICE % 16 == 0, "bulk copies move multiples of 16 bytes");
    static_assert(BS % ST == 0 || ST % BS == 0, "stages and blocks nest");
};

// Transposing butterfly over the CPR lanes of a row group: at each xor step a
// lane keeps half of its values (the upper half when its mask bit is set) and
// adds the partner's copy of that half.  After log2(V) halvings a lane holds
// V/CPR fully reduced values -- lane chunk c holds indices
// [c*V/CPR, (c+1)*V/CPR) -- or, when V < CPR, one value, index
// c / (CPR/V), replicated over CPR/V lanes by the remaining plain steps.
template <int N, int M>
struct TransposeReduce {
    static __device__ __forceinline__ void run(float* x, unsigned lane) {
        if constexpr (M == 0) {
            return;
        } else if constexpr (N > 1) {
            const bool upper = (lane & M) != 0;
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                const float send = upper ? x[i] : x[i + N / 2];
                const float keep = upper ? x[i + N / 2] : x[i];
                x[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
            }
            TransposeReduce<N / 2, M / 2>::run(x, lane);
        } else {
            x[0] += __shfl_xor_sync(0xffffffffu, x[0], M);
            TransposeReduce<1, M / 2>::run(x, lane);
        }
    }
};

template <typename T, typename TKV, int D, int BS, int G>
__global__ void __launch_bounds__(DecodeCfg<T, TKV, D, BS, G>::THREADS,
                                  DecodeCfg<T, TKV, D, BS, G>::THREADS > 320 ? 1 : 2)
    decode_partition_kernel(const DecodeParams p) {
    using C = DecodeCfg<T, TKV, D, BS, G>;
    constexpr bool kFp8 = sizeof(TKV) == 1;
    extern __shared__ __align__(128) unsigned char smem[];

    const int P = p.num_partitions;
    const int Hkv = p.num_kv_heads;
    const Unit unit = decode_unit(p, false);
    if (unit.s < 0) return;  // a schedule entry out of range (debug builds)
    const int part = unit.part, g = unit.g, s = unit.s;
    const int ctx = unit.ctx;
    const int max_ctx = p.max_blocks_per_seq * BS;

    if (ctx < 0 || ctx > max_ctx) {  // not a valid sequence: zero row, report once
        if (part == 0) {
            if (threadIdx.x == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            zero_rows<T, D, G>(p, (long long)s * p.num_heads + (long long)g * G);
        }
        return;
    }
    const int PT = p.partition_tokens;
    const int nparts = (ctx + PT - 1) / PT;
    if (part >= nparts) {
        if (ctx == 0 && part == 0) zero_rows<T, D, G>(p, (long long)s * p.num_heads + (long long)g * G);  // nothing attended
        return;
    }
    const int tok0 = part * PT;
    const int tok1 = min(ctx, tok0 + PT);
    const int nblk = (tok1 - tok0 + BS - 1) / BS;
    const int blk0 = tok0 / BS;
    const int nstg = (tok1 - tok0 + C::ST - 1) / C::ST;

    unsigned char* stages = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* empty = full + C::NST;
    int* phys = reinterpret_cast<int*>(smem + C::PHYS_OFF);
    float* pscr = reinterpret_cast<float*>(smem + C::PSCR_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::FLAG_OFF);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < C::NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], C::NHS);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    // The partition's table entries, read once, range-checked once.
    const int32_t* bt = p.block_tables + (long long)s * p.max_blocks_per_seq + blk0;
    for (int j = tid; j < nblk; j += blockDim.x) {
        int e = bt[j];
        if (e < 0 || e >= p.num_blocks) {
            set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            e = -1;
        }
        phys[j] = e;
    }
    __syncthreads();

    int issued = 0;  // stages issued (producer lane 0)
    // Per-warp softmax state (consumer warps).
    float m_run[C::GW];
    float o[C::GW][C::EPC];
    float l_run = 0.f;
#pragma unroll
    for (int gi = 0; gi < C::GW; ++gi) {
        m_run[gi] = -INFINITY;
#pragma unroll
        for (int e = 0; e < C::EPC; ++e) o[gi][e] = 0.f;
    }
    const int c = lane % C::CPR;
    const int r0 = lane / C::CPR;
    const int my_head = c / C::HLANES;  // head (within the warp's GW) of the logits this lane holds
    const int hs = warp / C::NBL;
    const int bl = warp % C::NBL;

    if (warp == C::NCW) {
        // ------------------------------------------------------ producer
        const char* kbase = static_cast<const char*>(p.k_cache);
        const char* vbase = static_cast<const char*>(p.v_cache);
        const long long pool_bytes = (long long)p.num_blocks * Hkv * C::SLICE;  // debug checks
        (void)pool_bytes;
        if constexpr (BS >= C::ST) {
            // One lane issues every copy (16 rows of one block, the whole
            // block when bs = 16): spreading two copies over the warp measured
            // slower here.
            if (lane == 0) {
                for (int j = 0; j < nstg; ++j) {
                    const int st = j % C::NST;
                    if (j >= C::NST) {
                        if (!mbar_wait_bounded(&empty[st], ((j / C::NST) - 1) & 1, abort_flag, p.wait_ns)) {
                            set_error(p.err, PKV_ERR_TIMEOUT);
                            *abort_flag = 1;
                            break;
                        }
                    }
                    unsigned char* dst = stages + st * C::STAGE;
                    const int e = phys[j * C::ST / BS];
                    const long long off =
                        (((long long)e * Hkv + g) * BS + (j * C::ST) % BS) * C::ROWB;
                    if (e >= 0 && PKV_DCHECK(p.err, off + C::STAGE_K <= pool_bytes && st < C::NST)) {
                        mbar_arrive_expect_tx(&full[st], 2 * C::STAGE_K);
                        bulk_g2s(dst, kbase + off, C::STAGE_K, &full[st]);
                        bulk_g2s(dst + C::STAGE_K, vbase + off, C::STAGE_K, &full[st]);
                    } else {
                        mbar_arrive(&full[st]);  // a skipped block still completes its phase
                    }
                    issued = j + 1;
                }
            }
        } else {
            // Whole blocks stacked row after row, several per stage: lane 0
            // waits for the slot and registers the byte count, then lane 2b
            // copies block b's K slice and lane 2b+1 its V slice, so the
            // stage's copies issue side by side.
            for (int j = 0; j < nstg; ++j) {
                const int st = j % C::NST;
                bool ready = true;
                if (lane == 0 && j >= C::NST)
                    ready = mbar_wait_bounded(&empty[st], ((j / C::NST) - 1) & 1, abort_flag, p.wait_ns);
                if (!__shfl_sync(0xffffffffu, ready, 0)) {
                    if (lane == 0) {
                        set_error(p.err, PKV_ERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    break;
                }
                const int b = lane >> 1;
                const int jb = j * C::BPS + b;
                const int e = (lane < 2 * C::BPS && jb < nblk) ? phys[jb] : -1;
                const long long off = ((long long)e * Hkv + g) * C::SLICE;
                const bool load = e >= 0 && PKV_DCHECK(p.err, off + C::SLICE <= pool_bytes && st < C::NST);
                const int nload = __popc(__ballot_sync(0xffffffffu, load));
                if (lane == 0) {
                    if (nload > 0)
                        mbar_arrive_expect_tx(&full[st], (uint32_t)(nload * C::SLICE));
                    else
                        mbar_arrive(&full[st]);
                }
                __syncwarp();  // the byte count is registered before any copy lands
                if (load) {
                    unsigned char* dst = stages + st * C::STAGE + (lane & 1) * C::STAGE_K + b * C::SLICE;
                    bulk_g2s(dst, ((lane & 1) ? vbase : kbase) + off, C::SLICE, &full[st]);
                }
                issued = j + 1;
            }
        }
    } else {
        // ------------------------------------------------------ consumers
        const int hbase = g * G + hs * C::GW;
        // fp8 caches: the kv head's K scale folds into the logit scale
        const float qs = kFp8 ? p.qscale * p.k_scales[g] : p.qscale;
        float qf[C::GW][C::EPC];
#pragma unroll
        for (int gi = 0; gi < C::GW; ++gi) {
            // this lane's EPC dims of q (one or more 16-byte loads of T)
            const uint4* qrow = reinterpret_cast<const uint4*>(
                static_cast<const T*>(p.q) + ((long long)s * p.num_heads + hbase + gi) * D + c * C::EPC);
            constexpr int QL = C::EPC / Elem<T>::kPer16B;
#pragma unroll
            for (int u = 0; u < QL; ++u) Elem<T>::unpack(qrow[u], qf[gi] + u * Elem<T>::kPer16B);
#pragma unroll
            for (int e = 0; e < C::EPC; ++e) qf[gi][e] *= qs;
        }
        float* my_pscr = pscr + (warp * C::RPI + r0) * (C::RPL * C::GW);
        const int vbase_idx = (C::V >= C::CPR) ? c * C::VPL : c / (C::CPR / C::V);
        const bool l_owner = (C::V >= C::CPR) || (c % (C::CPR / C::V) == 0);

        for (int j = bl; j < nstg; j += C::NBL) {
            const int st = j % C::NST;
            // every lane waits (bounded); the warp leaves together if any lane gave up
            const bool ready = mbar_wait_bounded(&full[st], (j / C::NST) & 1, abort_flag, p.wait_ns);
            if (!__all_sync(0xffffffffu, ready)) {
                if (lane == 0) {
                    set_error(p.err, PKV_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
                break;
            }
            // rows of this stage that hold tokens of the partition, from blocks
            // whose table entry was valid (warp-uniform)
            const int nvalid = min(C::ST, tok1 - (tok0 + j * C::ST));
            uint32_t rowmask = nvalid >= 32 ? 0xffffffffu : ((1u << nvalid) - 1u);
            if constexpr (BS >= C::ST) {
                if (phys[j * C::ST / BS] < 0) rowmask = 0;
            } else {
#pragma unroll
                for (int b = 0; b < C::BPS; ++b) {
                    const int jb = j * C::BPS + b;
                    if (jb >= nblk || phys[jb] < 0) rowmask &= ~(((1u << BS) - 1u) << (b * BS));
                }
            }
            if (rowmask != 0) {
                const uint4* Ks = reinterpret_cast<const uint4*>(stages + st * C::STAGE);
                const uint4* Vs = reinterpret_cast<const uint4*>(stages + st * C::STAGE + C::STAGE_K);
                const bool tail = rowmask != C::FULL_ROWS;
                {
                    constexpr int rbase = 0;
                    // ---- QK^T: partial dot products over this lane's chunk
                    float sc[C::V];
#pragma unroll
                    for (int k = 0; k < C::RPL; ++k) {
                        const int row = rbase + r0 + k * C::RPI;
                        float kf[C::EPC];
                        Elem<TKV>::unpack(Ks[row * C::CPR + c], kf);
#pragma unroll
                        for (int gi = 0; gi < C::GW; ++gi) {
                            float acc = 0.f;
#pragma unroll
                            for (int e = 0; e < C::EPC; ++e) acc = fmaf(qf[gi][e], kf[e], acc);
                            sc[gi * C::RPL + k] = acc;
                        }
                    }
                    TransposeReduce<C::V, C::CPR / 2>::run(sc, lane);
                    // ---- mask and sub-tile maximum per head
                    float mloc = -INFINITY;
#pragma unroll
                    for (int i = 0; i < C::VPL; ++i) {
                        const int k = (vbase_idx + i) % C::RPL;
                        const bool valid = (rowmask >> (rbase + r0 + k * C::RPI)) & 1u;
                        sc[i] = valid ? sc[i] : -INFINITY;
                        mloc = fmaxf(mloc, sc[i]);
                    }
#pragma unroll
                    for (int msk = 1; msk < C::HLANES; msk <<= 1)
                        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, msk));
#pragma unroll
                    for (int msk = C::CPR; msk < 32; msk <<= 1)
                        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, msk));
                    float m_mine = 0.f, a_mine = 0.f;
#pragma unroll
                    for (int gi = 0; gi < C::GW; ++gi) {
                        const float mt = __shfl_sync(0xffffffffu, mloc, gi * C::HLANES);
                        const float mnew = fmaxf(m_run[gi], mt);
                        const float alpha = exp2f(m_run[gi] - mnew);
                        m_run[gi] = mnew;
#pragma unroll
                        for (int e = 0; e < C::EPC; ++e) o[gi][e] *= alpha;
                        if (gi == my_head) {
                            m_mine = mnew;
                            a_mine = alpha;
                        }
                    }
                    // ---- probabilities of this lane's logits
                    float psum = 0.f;
#pragma unroll
                    for (int i = 0; i < C::VPL; ++i) {
                        sc[i] = exp2f(sc[i] - m_mine);
                        psum += sc[i];
                    }
                    l_run = l_run * a_mine + (l_owner ? psum : 0.f);
                    // publish to the warp's scratch as [row k][head]
#pragma unroll
                    for (int i = 0; i < C::VPL; ++i) {
                        const int idx = vbase_idx + i;
                        my_pscr[(idx % C::RPL) * C::GW + idx / C::RPL] = sc[i];
                    }
                    __syncwarp();
                    // ---- PV over this lane's rows and chunk
#pragma unroll
                    for (int k = 0; k < C::RPL; ++k) {
                        const int row = rbase + r0 + k * C::RPI;
                        float pk[C::GW];
                        if constexpr (C::GW == 4) {
                            const float4 t4 = *reinterpret_cast<const float4*>(my_pscr + k * 4);
                            pk[0] = t4.x;
                            pk[1] = t4.y;
                            pk[2] = t4.z;
                            pk[3] = t4.w;
                        } else if constexpr (C::GW == 2) {
                            const float2 t2 = *reinterpret_cast<const float2*>(my_pscr + k * 2);
                            pk[0] = t2.x;
                            pk[1] = t2.y;
                        } else {
                            pk[0] = my_pscr[k];
                        }
                        float vf[C::EPC];
                        Elem<TKV>::unpack(Vs[row * C::CPR + c], vf);
                        if (tail && !((rowmask >> row) & 1u)) continue;  // never read an unused slot into o
#pragma unroll
                        for (int gi = 0; gi < C::GW; ++gi)
#pragma unroll
                            for (int e = 0; e < C::EPC; ++e) o[gi][e] = fmaf(pk[gi], vf[e], o[gi][e]);
                    }
                    __syncwarp();
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        // warp-level totals: l over the lanes of a head, o over the row groups
#pragma unroll
        for (int msk = 1; msk < C::HLANES; msk <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, msk);
#pragma unroll
        for (int msk = C::CPR; msk < 32; msk <<= 1) {
            l_run += __shfl_xor_sync(0xffffffffu, l_run, msk);
#pragma unroll
            for (int gi = 0; gi < C::GW; ++gi)
#pragma unroll
                for (int e = 0; e < C::EPC; ++e) o[gi][e] += __shfl_xor_sync(0xffffffffu, o[gi][e], msk);
        }
    }

    __syncthreads();  // every block consumed: the stage memory is free for the merge
    if (*abort_flag) {
        if (warp == C::NCW && lane == 0) {
            // let this CTA's own bulk copies land before it exits
            for (int j = issued - C::NST > 0 ? issued - C::NST : 0; j < issued; ++j) {
                const int st = j % C::NST;
                const unsigned long long t0 = globaltimer_ns();
                while (!mbar_try_wait(&full[st], (j / C::NST) & 1)) {
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
                }
            }
        }
        __syncthreads();
        abort_merge_turn<T, D, G>(p, s, g, (long long)s * p.num_heads + (long long)g * G, part, nparts, reinterpret_cast<int*>(smem + C::FLAG_OFF) + 1);
        return;
    }

    float* mrg = reinterpret_cast<float*>(smem);  // [NBL][G][D + 2]
    if (warp < C::NCW) {
#pragma unroll
        for (int gi = 0; gi < C::GW; ++gi) {
            float* row = mrg + (bl * G + hs * C::GW + gi) * (D + 2);
            if (r0 == 0) {
#pragma unroll
                for (int e = 0; e < C::EPC; ++e) row[c * C::EPC + e] = o[gi][e];
            }
            if (lane == 0) row[D] = m_run[gi];
            if (lane == gi * C::HLANES) row[D + 1] = l_run;
        }
    }
    __syncthreads();

    const int H = p.num_heads;
    const long long sh0 = (long long)s * H + (long long)g * G;  // first query head of the group
    const float vsc = kFp8 ? p.v_scales[g] : 1.f;  // fp8: the kv head's V scale
    for (int t = tid; t < G * D; t += blockDim.x) {
        const int hg = t / D;
        const int d = t % D;
        float M = -INFINITY;
#pragma unroll
        for (int b = 0; b < C::NBL; ++b) M = fmaxf(M, mrg[(b * G + hg) * (D + 2) + D]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int b = 0; b < C::NBL; ++b) {
                const float* row = mrg + (b * G + hg) * (D + 2);
                const float w = exp2f(row[D] - M);
                L = fmaf(w, row[D + 1], L);
                O = fmaf(w, row[d], O);
            }
        }
        O *= vsc;
        const long long sh = sh0 + hg;
        if (!PKV_DCHECK(p.err, sh < (long long)p.num_seqs * H && part < P)) continue;
        if (nparts == 1) {
            Elem<T>::store(static_cast<T*>(p.out) + sh * D + d, L > 0.f ? O / L : 0.f);
        } else {
            p.ws_o[(sh * P + part) * D + d] = O;
            if (d == 0) p.ws_ml[sh * P + part] = make_float2(M, L);
        }
    }
    if (nparts == 1) return;
    fused_merge<T, D, G, C::THREADS>(p, s, g, nparts, sh0, reinterpret_cast<float*>(smem) + C::MERGE_FLOATS,
                                      reinterpret_cast<int*>(smem + C::FLAG_OFF) + 1);
}

}  // namespace pkv
