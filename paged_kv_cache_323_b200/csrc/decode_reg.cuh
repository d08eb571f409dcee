// decode_reg.cuh -- paged decode attention with one query head per kv head,
// the cache streamed through registers (sm_100a).
//
// Same computation as decode_attn.cuh ("PagedAttention Explained: Virtual
// Memory for the KV Cache", section "How PagedAttention works", item 5: the
// kernel follows the block table and gathers each block's keys and values),
// for one query head per kv head and bf16 caches:
//     out[s][h] = softmax(scale * q[s][h] . K_s^T) V_s
//
// Why a second form: at block size 8 a (block, kv head) slice of K is 2 KB.
// Staging such slices through shared memory costs one asynchronous copy each
// (bulk copy, or sixteen 16-byte cp.async per warp), and at that size the
// per-copy cost, not HBM, set the pace of the staged kernel.  Here each warp
// reads the cache with plain 16-byte loads straight into registers, which
// also beat the staged kernel at block sizes 16 and 32:
//  * One CTA per (sequence, kv head, partition), NW warps.  The partition's
//    table entries are read once into shared memory and range-checked.
//  * The partition is cut into chunks of 2 KB of K and 2 KB of V, each
//    contiguous in the [block][kv head][slot][dim] pool: 8 tokens at head_dim
//    128, 16 at head_dim 64 (8 when the block holds only 8), a whole block or
//    an aligned run of rows of a larger one.  Warp w takes chunks w, w + NW,
//    w + 2 NW, ...; lane l loads the 16-byte piece l % (D / 8) of rows
//    l / (D / 8), and every 32 / (D / 8) rows after it (one warp-wide load
//    covers 512 contiguous bytes).  The next chunk's K and V loads are
//    issued before the current chunk is computed (two register buffers), so
//    every warp keeps a whole chunk in flight while it works.
//  * Partial dot products over a lane's 8 dims are reduced by the transposing
//    butterfly of decode_attn.cuh; online softmax in base 2 with fp32 running
//    max and sum; PV into fp32 registers (8 dims per lane).  Unused slots of
//    the last block are never multiplied (they may hold NaN), and a block
//    whose table entry is out of range is skipped (error word set).
//  * Warps merge their (m, l, o) through shared memory in warp order; the
//    partition then ends like every other decode kernel, through the fused
//    split-K merge.  The arithmetic order depends only on logical token
//    positions, so outputs do not depend on where the blocks sit.
//  * There are no waits: nothing here can time out.
#pragma once

#include <math.h>

#include "decode_attn.cuh"

namespace pkv {

template <int D, int BS, int NW>
struct RegCfg {
    static constexpr int CPR = D / 8;        // 16-byte pieces (8 bf16) per row
    static constexpr int RPI = 32 / CPR;     // rows covered by one warp-wide load
    static constexpr int ROWB = D * 2;       // bytes of one token row
    // rows (tokens) per chunk: 2 KB of K (8 rows at head_dim 128, 16 at 64),
    // at most one block
    static constexpr int RW = BS < 2048 / ROWB ? BS : 2048 / ROWB;
    static constexpr int CPB = BS / RW;      // chunks per block
    static constexpr int RPL = RW / RPI;     // rows per lane per chunk
    static constexpr int THREADS = NW * 32;
    static constexpr int SLICE = BS * ROWB;  // bytes of one (block, kv head)
    static constexpr int MAX_PART_TOKENS = 4096;
    static constexpr int MAX_PART_BLOCKS = MAX_PART_TOKENS / BS;
    static constexpr int SCRATCH_FLOATS = merge_scratch_bytes<1, D, THREADS>() / 4;

    static_assert(D % 8 == 0 && CPR <= 32 && 32 % CPR == 0, "head_dim chunking");
    static_assert(BS % RW == 0 && RW % RPI == 0 && RPL >= 1 && RPL <= CPR, "rows per lane");
};

// 16 bytes of the cache, read once: no L1 allocation.
__device__ __forceinline__ uint4 ld_kv_stream(const void* ptr) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(ptr));
    return r;
}

template <int D, int BS, int NW, int MINB>
__global__ void __launch_bounds__(NW * 32, MINB) decode_reg_kernel(const DecodeParams p) {
    using C = RegCfg<D, BS, NW>;
    using T = __nv_bfloat16;
    __shared__ int phys[C::MAX_PART_BLOCKS];
    __shared__ float mrg[NW][D + 2];
    __shared__ __align__(16) float scratch[C::SCRATCH_FLOATS];
    __shared__ int last_flag;

    const Unit unit = decode_unit(p, false);
    if (unit.s < 0) return;  // a schedule entry out of range (debug builds)
    const int part = unit.part, g = unit.g, s = unit.s;
    const int ctx = unit.ctx;
    const int Hkv = p.num_kv_heads;
    const long long sh0 = (long long)s * p.num_heads + g;  // the kv head's one query head
    if (ctx < 0 || ctx > p.max_blocks_per_seq * BS) {  // not a valid sequence: zero row, report once
        if (part == 0) {
            if (threadIdx.x == 0) set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            zero_rows<T, D, 1>(p, sh0);
        }
        return;
    }
    const int PT = p.partition_tokens;
    const int nparts = (ctx + PT - 1) / PT;
    if (part >= nparts) {
        if (ctx == 0 && part == 0) zero_rows<T, D, 1>(p, sh0);  // nothing attended
        return;
    }
    const int tok0 = part * PT;
    const int tok1 = min(ctx, tok0 + PT);
    const int nblk = (tok1 - tok0 + BS - 1) / BS;
    const int nchk = (tok1 - tok0 + C::RW - 1) / C::RW;
    const int blk0 = tok0 / BS;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int32_t* bt = p.block_tables + (long long)s * p.max_blocks_per_seq + blk0;
    for (int j = tid; j < nblk; j += C::THREADS) {
        int e = bt[j];
        if (e < 0 || e >= p.num_blocks) {
            set_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            e = -1;
        }
        phys[j] = e;
    }

    const int c = lane % C::CPR;  // this lane's 16-byte piece of a row
    const int r0 = lane / C::CPR;  // its first row of a chunk
    float qf[8];
    {
        const uint4 qr = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) + sh0 * D + c * 8);
        Elem<T>::unpack(qr, qf);
#pragma unroll
        for (int e = 0; e < 8; ++e) qf[e] *= p.qscale;
    }
    __syncthreads();

    const long long lane_off = ((long long)g * BS + r0) * C::ROWB + c * 16;
    const char* kbase = static_cast<const char*>(p.k_cache) + lane_off;
    const char* vbase = static_cast<const char*>(p.v_cache) + lane_off;
    const long long slice_stride = (long long)Hkv * C::SLICE;  // one physical block
    const long long pool_bytes = (long long)p.num_blocks * slice_stride;  // debug checks
    (void)pool_bytes;

    // chunk q of the partition into registers (zeros for a skipped block)
    auto load = [&](int q, uint4 (&kr)[C::RPL], uint4 (&vr)[C::RPL]) {
        const int e = q < nchk ? phys[q / C::CPB] : -1;
        const long long off = (long long)e * slice_stride + (q % C::CPB) * (C::RW * C::ROWB);
        if (e >= 0 && PKV_DCHECK(p.err, off + (long long)g * C::SLICE + C::RW * C::ROWB <= pool_bytes)) {
#pragma unroll
            for (int k = 0; k < C::RPL; ++k) {
                kr[k] = ld_kv_stream(kbase + off + k * C::RPI * C::ROWB);
                vr[k] = ld_kv_stream(vbase + off + k * C::RPI * C::ROWB);
            }
        } else {
#pragma unroll
            for (int k = 0; k < C::RPL; ++k) kr[k] = vr[k] = make_uint4(0u, 0u, 0u, 0u);
        }
    };

    float m_run = -INFINITY, l_run = 0.f;
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = 0.f;
    // after the butterfly a lane holds the logit of row r0 + RPI * vi
    constexpr int SPREAD = C::CPR / C::RPL;  // lanes holding one logit
    const int vi = c / SPREAD;
    const bool l_owner = c % SPREAD == 0;

    auto compute = [&](int q, const uint4 (&kr)[C::RPL], const uint4 (&vr)[C::RPL]) {
        if (phys[q / C::CPB] < 0) return;  // out-of-range entry: skipped, error already set
        const int nvalid = min(C::RW, tok1 - (tok0 + q * C::RW));
        float sc[C::RPL];
#pragma unroll
        for (int k = 0; k < C::RPL; ++k) {
            float kf[8];
            Elem<T>::unpack(kr[k], kf);
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(qf[e], kf[e], acc);
            sc[k] = acc;
        }
        TransposeReduce<C::RPL, C::CPR / 2>::run(sc, lane);
        const float x = (r0 + C::RPI * vi) < nvalid ? sc[0] : -INFINITY;
        float mloc = x;
#pragma unroll
        for (int msk = SPREAD; msk < 32; msk <<= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, msk));
        const float mnew = fmaxf(m_run, mloc);
        const float alpha = exp2f(m_run - mnew);
        m_run = mnew;
        const float pr = exp2f(x - mnew);
        l_run = fmaf(l_run, alpha, l_owner ? pr : 0.f);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] *= alpha;
#pragma unroll
        for (int k = 0; k < C::RPL; ++k) {
            const float pk = __shfl_sync(0xffffffffu, pr, (lane & ~(C::CPR - 1)) | (k * SPREAD));
            if (r0 + C::RPI * k < nvalid) {  // never read an unused slot into o
                float vf[8];
                Elem<T>::unpack(vr[k], vf);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = fmaf(pk, vf[e], o[e]);
            }
        }
    };

    {
        uint4 ka[C::RPL], va[C::RPL], kb[C::RPL], vb[C::RPL];
        int q = warp;
        load(q, ka, va);
        while (q < nchk) {
            load(q + NW, kb, vb);
            compute(q, ka, va);
            q += NW;
            if (q >= nchk) break;
            load(q + NW, ka, va);
            compute(q, kb, vb);
            q += NW;
        }
    }

    // warp totals: l over all lanes (one owner per logit), o over the row groups
#pragma unroll
    for (int msk = 1; msk < 32; msk <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, msk);
#pragma unroll
    for (int msk = C::CPR; msk < 32; msk <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] += __shfl_xor_sync(0xffffffffu, o[e], msk);
    if (r0 == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) mrg[warp][c * 8 + e] = o[e];
    }
    if (lane == 0) {
        mrg[warp][D] = m_run;
        mrg[warp][D + 1] = l_run;
    }
    __syncthreads();

    const int P = p.num_partitions;
    for (int d = tid; d < D; d += C::THREADS) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, mrg[w][D]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float wt = exp2f(mrg[w][D] - M);
                L = fmaf(wt, mrg[w][D + 1], L);
                O = fmaf(wt, mrg[w][d], O);
            }
        }
        if (!PKV_DCHECK(p.err, sh0 < (long long)p.num_seqs * p.num_heads && part < P)) continue;
        if (nparts == 1) {
            Elem<T>::store(static_cast<T*>(p.out) + sh0 * D + d, L > 0.f ? O / L : 0.f);
        } else {
            p.ws_o[(sh0 * P + part) * D + d] = O;
            if (d == 0) p.ws_ml[sh0 * P + part] = make_float2(M, L);
        }
    }
    if (nparts == 1) return;
    fused_merge<T, D, 1, C::THREADS>(p, s, g, nparts, sh0, scratch, &last_flag);
}

}  // namespace pkv
