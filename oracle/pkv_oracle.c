/*
 * pkv_oracle.c -- plain, slow, obviously correct CPU reference for the paged
 * KV-cache decode path.  TEST INFRASTRUCTURE ONLY: it is called by the tests,
 * by the smoke check and by the CPU-baseline leg of the benchmark, never by the
 * product path.  It shares no code, header or constant with the CUDA library.
 *
 * What it follows (page titles and sections of the source pages):
 *  - "PagedAttention Explained: Virtual Memory for the KV Cache",
 *    section "How PagedAttention works", items 1-5: fixed-size blocks, a
 *    logical view per sequence (tokens 0..bs-1 in logical block 0, ...), a
 *    block table mapping logical to physical blocks placed anywhere, allocation
 *    on demand, and an attention computation that gathers keys and values
 *    through the table.
 *  - same page, section "Sharing blocks between sequences": shared blocks and
 *    copy-on-write ("copies that block first and updates the writer's table").
 *  - same page, section "The problem: the KV cache is big and unpredictable":
 *    the cache grows by one entry for every new token (the append step).
 *  - "What does PagedAttention change in LLM KV allocation?", section
 *    "Calculate unused block space": block count and unused slots.
 *
 * Attention itself is not written out on the pages; the reading used here is
 * the standard definition for one decode query:
 *     x_t = scale * sum_d q[d] * K[t][d]          t < L
 *     out = sum_t exp(x_t - max_t x) * V[t] / sum_t exp(x_t - max_t x)
 * computed in fp64 after an exact conversion of the fp32 / bf16 inputs.  Every
 * step is the definition itself: the contiguous K and V of a sequence are
 * assembled first by walking the block table, then the logits, the maximum,
 * the exponentials, the normaliser and the weighted sum are formed in that
 * order.  No online softmax, no partitions, no blocking.
 *
 * Pool layout read here: k_cache and v_cache are each
 *     [num_blocks][num_kv_heads][block_size][head_dim]
 * and token t of sequence s lives in physical block block_tables[s][t / bs],
 * slot t % bs.  Query head h reads kv head h / (num_heads / num_kv_heads).
 *
 * Pins: every function here is checked by the CPU tests against the worked
 * example of the pages, closed forms, invariants and a numpy brute force over
 * contiguous arrays; none is "parity unpinned".
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1
#define ORACLE_FP8 2 /* e4m3 codes: moved as bytes by append / copy / swap */

/* ---------------------------------------------------------------- values */

/* Exact widening of one stored element to double.  A bf16 value is the upper
 * half of an IEEE binary32, so shifting its 16 bits up gives the float it
 * stands for exactly; a float widens to double exactly. */
static double load_elem(const void* base, int64_t index, int dtype) {
    if (dtype == ORACLE_F32) {
        return (double)((const float*)base)[index];
    }
    uint16_t bits16 = ((const uint16_t*)base)[index];
    uint32_t bits32 = ((uint32_t)bits16) << 16;
    float f;
    memcpy(&f, &bits32, sizeof f);
    return (double)f;
}

static int elem_bytes(int dtype) { return dtype == ORACLE_F32 ? 4 : (dtype == ORACLE_FP8 ? 1 : 2); }

/* ------------------------------------------------- block-count accounting */

/* "Calculate unused block space": a sequence of L tokens in blocks of bs
 * tokens needs ceil(L / bs) blocks; the allocation holds that many times bs
 * slots; the slots not holding a token are unused. */
int64_t oracle_blocks_needed(int64_t L, int64_t bs) {
    if (L <= 0) return 0;
    return (L + bs - 1) / bs;
}

/* Per-sequence accounting summed over a batch: allocated slots and unused
 * slots, counting every sequence's blocks as its own. */
void oracle_waste_per_sequence(const int32_t* lens, int n, int bs,
                               int64_t* allocated_slots, int64_t* unused_slots) {
    int64_t alloc = 0, used = 0;
    for (int i = 0; i < n; ++i) {
        alloc += oracle_blocks_needed(lens[i], bs) * bs;
        used += lens[i] > 0 ? lens[i] : 0;
    }
    *allocated_slots = alloc;
    *unused_slots = alloc - used;
}

/* Physical accounting with sharing ("Sharing blocks between sequences"): each
 * physical block referenced by any table counts once; a slot counts as used
 * when at least one sequence has a token in it.  Slots of block p that hold
 * tokens for sequence s at logical block j are the first
 * min(bs, L_s - j*bs) slots. */
void oracle_waste_physical(const int32_t* block_tables, const int32_t* lens,
                           int n, int max_blocks_per_seq, int bs,
                           int num_blocks, int64_t* allocated_slots,
                           int64_t* unused_slots) {
    int32_t* filled = (int32_t*)calloc((size_t)num_blocks, sizeof(int32_t));
    uint8_t* seen = (uint8_t*)calloc((size_t)num_blocks, 1);
    for (int s = 0; s < n; ++s) {
        int64_t nb = oracle_blocks_needed(lens[s], bs);
        for (int64_t j = 0; j < nb; ++j) {
            int32_t p = block_tables[(int64_t)s * max_blocks_per_seq + j];
            int64_t here = lens[s] - j * bs;
            if (here > bs) here = bs;
            seen[p] = 1;
            if (here > filled[p]) filled[p] = (int32_t)here;
        }
    }
    int64_t alloc = 0, used = 0;
    for (int p = 0; p < num_blocks; ++p) {
        if (seen[p]) {
            alloc += bs;
            used += filled[p];
        }
    }
    free(filled);
    free(seen);
    *allocated_slots = alloc;
    *unused_slots = alloc - used;
}

/* ------------------------------------------------------------- the gather */

/* Assemble the contiguous keys (or values) of sequence s for kv head g:
 * out[t][d] = cache[block_tables[s][t / bs]][g][t % bs][d] for t < L, in
 * fp64.  This is the "logical view" of the sequence rebuilt from the table. */
void oracle_gather(double* out, const void* cache, int dtype,
                   const int32_t* block_tables, int s, int L, int g,
                   int num_kv_heads, int head_dim, int block_size,
                   int max_blocks_per_seq) {
    for (int t = 0; t < L; ++t) {
        int32_t p = block_tables[(int64_t)s * max_blocks_per_seq + t / block_size];
        int slot = t % block_size;
        int64_t row = (((int64_t)p * num_kv_heads + g) * block_size + slot) * head_dim;
        for (int d = 0; d < head_dim; ++d) {
            out[(int64_t)t * head_dim + d] = load_elem(cache, row + d, dtype);
        }
    }
}

/* ----------------------------------------------------- decode attention */

typedef struct {
    double* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    int dtype;
    const int32_t* block_tables;
    const int32_t* context_lens;
    int num_seqs, num_heads, num_kv_heads, head_dim, block_size;
    int max_blocks_per_seq;
    double scale;
    const int32_t* rows; /* (s, h) pairs, or NULL for every pair */
    int n_units;
    int next; /* shared work counter */
    pthread_mutex_t lock;
} attn_job;

/* Steps 2-4 of the definition for one query row over contiguous K and V
 * (L rows of D values, fp64): logits, softmax weights, weighted sum of V. */
static void attend_rows(double* o, const double* qd, const double* Kc, const double* Vc, int L,
                        int D, double scale) {
    double* x = (double*)malloc(sizeof(double) * (size_t)L);
    /* step 2: logits */
    for (int t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qd[d] * Kc[(int64_t)t * D + d];
        x[t] = scale * acc;
    }
    /* step 3: softmax weights */
    double m = x[0];
    for (int t = 1; t < L; ++t)
        if (x[t] > m) m = x[t];
    double Z = 0.0;
    for (int t = 0; t < L; ++t) {
        x[t] = exp(x[t] - m);
        Z += x[t];
    }
    /* step 4: weighted sum of values */
    for (int t = 0; t < L; ++t) {
        double w = x[t] / Z;
        for (int d = 0; d < D; ++d) o[d] += w * Vc[(int64_t)t * D + d];
    }
    free(x);
}

/* One (s, h) unit, written as the definition. */
static void attend_one(attn_job* job, int unit) {
    int s, h;
    if (job->rows) {
        s = job->rows[2 * unit];
        h = job->rows[2 * unit + 1];
    } else {
        s = unit / job->num_heads;
        h = unit % job->num_heads;
    }
    const int D = job->head_dim;
    const int group = job->num_heads / job->num_kv_heads;
    const int g = h / group;
    const int L = job->context_lens[s];
    double* o = job->out + (int64_t)unit * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (L <= 0) return; /* nothing attended: the output row is zero */

    double* Kc = (double*)malloc(sizeof(double) * (size_t)L * D);
    double* Vc = (double*)malloc(sizeof(double) * (size_t)L * D);
    double* qd = (double*)malloc(sizeof(double) * (size_t)D);

    /* step 1: the logical (contiguous) view of this sequence's cache */
    oracle_gather(Kc, job->k_cache, job->dtype, job->block_tables, s, L, g,
                  job->num_kv_heads, D, job->block_size, job->max_blocks_per_seq);
    oracle_gather(Vc, job->v_cache, job->dtype, job->block_tables, s, L, g,
                  job->num_kv_heads, D, job->block_size, job->max_blocks_per_seq);
    for (int d = 0; d < D; ++d)
        qd[d] = load_elem(job->q, ((int64_t)s * job->num_heads + h) * D + d, job->dtype);

    attend_rows(o, qd, Kc, Vc, L, D, job->scale);
    free(Kc);
    free(Vc);
    free(qd);
}

static void* attn_worker(void* arg) {
    attn_job* job = (attn_job*)arg;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        int unit = job->next++;
        pthread_mutex_unlock(&job->lock);
        if (unit >= job->n_units) break;
        attend_one(job, unit);
    }
    return NULL;
}

/* Decode attention for every (s, h) (rows == NULL, out is
 * [num_seqs][num_heads][head_dim]) or for the n_rows listed (s, h) pairs (out
 * is [n_rows][head_dim]).  Returns 0, or -1 on an argument the definition
 * does not cover. */
int oracle_paged_attention(double* out, const void* q, const void* k_cache,
                           const void* v_cache, int dtype,
                           const int32_t* block_tables,
                           const int32_t* context_lens, int num_seqs,
                           int num_heads, int num_kv_heads, int head_dim,
                           int block_size, int max_blocks_per_seq, double scale,
                           const int32_t* rows, int n_rows, int nthreads) {
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0) return -1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return -1;
    for (int s = 0; s < num_seqs; ++s)
        if (context_lens[s] > (int64_t)max_blocks_per_seq * block_size) return -1;
    attn_job job;
    job.out = out;
    job.q = q;
    job.k_cache = k_cache;
    job.v_cache = v_cache;
    job.dtype = dtype;
    job.block_tables = block_tables;
    job.context_lens = context_lens;
    job.num_seqs = num_seqs;
    job.num_heads = num_heads;
    job.num_kv_heads = num_kv_heads;
    job.head_dim = head_dim;
    job.block_size = block_size;
    job.max_blocks_per_seq = max_blocks_per_seq;
    job.scale = scale;
    job.rows = rows;
    job.n_units = rows ? n_rows : num_seqs * num_heads;
    job.next = 0;
    pthread_mutex_init(&job.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads == 1) {
        attn_worker(&job);
    } else {
        pthread_t* tid = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
        for (int i = 0; i < nthreads; ++i) pthread_create(&tid[i], NULL, attn_worker, &job);
        for (int i = 0; i < nthreads; ++i) pthread_join(tid[i], NULL);
        free(tid);
    }
    pthread_mutex_destroy(&job.lock);
    return 0;
}

/* ------------------------------------------------------ append and copy */

/* The cache grows by one entry per new token: token i's key and value rows
 * (all kv heads) go to the slot slot_mapping[i]; that slot lives in block
 * slot / bs at offset slot % bs.  A slot of -1 means "no write".  Byte copy,
 * so the stored bits are exactly the given bits. */
void oracle_kv_append(void* k_cache, void* v_cache, const void* k, const void* v,
                      const int64_t* slot_mapping, int num_tokens,
                      int num_kv_heads, int head_dim, int block_size, int dtype) {
    const int64_t row_bytes = (int64_t)head_dim * elem_bytes(dtype);
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0) continue;
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int g = 0; g < num_kv_heads; ++g) {
            int64_t dst = ((blk * num_kv_heads + g) * block_size + off) * row_bytes;
            int64_t src = ((int64_t)i * num_kv_heads + g) * row_bytes;
            memcpy((char*)k_cache + dst, (const char*)k + src, (size_t)row_bytes);
            memcpy((char*)v_cache + dst, (const char*)v + src, (size_t)row_bytes);
        }
    }
}

/* Copy-on-write: for each (src, dst) pair the whole physical block -- keys
 * and values of every kv head and slot -- is copied from src to dst, in pair
 * order.  The caller updates the writer's block table afterwards. */
void oracle_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs,
                        int num_pairs, int num_kv_heads, int head_dim,
                        int block_size, int dtype) {
    const int64_t block_bytes =
        (int64_t)num_kv_heads * block_size * head_dim * elem_bytes(dtype);
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        memmove((char*)k_cache + dst * block_bytes, (const char*)k_cache + src * block_bytes,
                (size_t)block_bytes);
        memmove((char*)v_cache + dst * block_bytes, (const char*)v_cache + src * block_bytes,
                (size_t)block_bytes);
    }
}

/* Preemption by swapping ("PagedAttention Explained: Virtual Memory for the
 * KV Cache", section "Preemption and scheduling": a sequence's blocks move to
 * CPU memory and come back later): for each (src, dst) pair, the whole block
 * src of the source pools is copied to block dst of the destination pools. */
void oracle_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                        const int64_t* pairs, int num_pairs, int num_kv_heads, int head_dim,
                        int block_size, int dtype) {
    /* one block: every kv head, every slot, every dimension */
    const int64_t block_bytes = (int64_t)elem_bytes(dtype) * head_dim * block_size * num_kv_heads;
    for (int i = 0; i < num_pairs; ++i) {
        const int64_t src = pairs[2 * i];     /* block in the source pools */
        const int64_t dst = pairs[2 * i + 1]; /* block in the destination pools */
        memcpy((char*)dst_k + dst * block_bytes, (const char*)src_k + src * block_bytes,
               (size_t)block_bytes);
        memcpy((char*)dst_v + dst * block_bytes, (const char*)src_v + src * block_bytes,
               (size_t)block_bytes);
    }
}

/* ------------------------------------------------ fp8 (e4m3) KV cache */
/* "What does PagedAttention change in LLM KV allocation?", section "Sharing
 * requires more than allocation": where the raw KV data does not fit, cache
 * quantization is one of the remedies.  Reading used here: K and V stored as
 * OCP FP8 E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; largest finite 448), one float scale per kv
 * head: stored value = code * scale. */

/* Exact value of an e4m3 code. */
double oracle_e4m3_value(uint8_t code) {
    const int sign = code >> 7;
    const int e = (code >> 3) & 15;
    const int m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9); /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp(8.0 + m, e - 10); /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Nearest e4m3 code to y, ties to the even code, magnitudes of 448 and more
 * clamped to 448 (saturating); NaN stays NaN.  Written as a search over the
 * 127 non-negative finite codes, which is the definition of rounding. */
uint8_t oracle_e4m3_encode(float y) {
    if (isnan(y)) return 0x7F;
    const uint8_t sign = signbit(y) ? 0x80 : 0x00;
    const double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7E;
    int best = 0;
    double best_err = a;
    for (int c = 1; c <= 0x7E; ++c) {
        const double err = fabs(oracle_e4m3_value((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return sign | (uint8_t)best;
}

/* Append with quantization: token i's bf16 rows (raw bits) become codes of
 * (float)x / scale[g] (one correctly rounded fp32 division) at slot
 * slot_mapping[i]; -1 skips. */
void oracle_kv_append_fp8(uint8_t* k_cache, uint8_t* v_cache, const float* k_scales,
                          const float* v_scales, const uint16_t* k, const uint16_t* v,
                          const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                          int head_dim, int block_size) {
    for (int i = 0; i < num_tokens; ++i) {
        const int64_t slot = slot_mapping[i];
        if (slot < 0) { /* no write for this token */
            continue;
        }
        const int64_t blk = slot / block_size;
        const int64_t off = slot - blk * block_size;
        for (int g = 0; g < num_kv_heads; ++g) {
            const int64_t dst = ((blk * num_kv_heads + g) * block_size + off) * head_dim;
            const int64_t src = ((int64_t)i * num_kv_heads + g) * head_dim;
            for (int d = 0; d < head_dim; ++d) {
                const float kx = (float)load_elem(k, src + d, ORACLE_BF16);
                const float vx = (float)load_elem(v, src + d, ORACLE_BF16);
                k_cache[dst + d] = oracle_e4m3_encode(kx / k_scales[g]);
                v_cache[dst + d] = oracle_e4m3_encode(vx / v_scales[g]);
            }
        }
    }
}

/* Offset of token t (kv head g) in a [block][kv head][slot][dim] pool, the
 * token's block taken from this sequence's table row. */
static int64_t fp8_token_row(const int32_t* table_row, int t, int block_size, int num_kv_heads,
                             int g, int head_dim) {
    const int32_t blk = table_row[t / block_size];
    return (((int64_t)blk * num_kv_heads + g) * block_size + t % block_size) * head_dim;
}

/* Decode attention over an e4m3 cache: the same definition as
 * oracle_paged_attention with K[t][d] = code * k_scale[g] and V likewise
 * (each product exact in fp64); q (bf16 bits) and out as there. */
int oracle_paged_attention_fp8(double* out, const uint16_t* q, const uint8_t* k_cache,
                               const uint8_t* v_cache, const float* k_scales,
                               const float* v_scales, const int32_t* block_tables,
                               const int32_t* context_lens, int num_seqs, int num_heads,
                               int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, double scale) {
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim > 1024) return -1;
    const int D = head_dim, group = num_heads / num_kv_heads;
    for (int s = 0; s < num_seqs; ++s) {
        const int L = context_lens[s];
        if (L > (int64_t)max_blocks_per_seq * block_size) return -1;
        const int32_t* table_row = block_tables + (int64_t)s * max_blocks_per_seq;
        for (int h = 0; h < num_heads; ++h) {
            const int g = h / group; /* contiguous query-head groups */
            double* o = out + ((int64_t)s * num_heads + h) * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (L <= 0) continue;
            /* the logical view, dequantised: code * scale of the kv head */
            double* Kc = (double*)malloc(sizeof(double) * (size_t)L * D);
            double* Vc = (double*)malloc(sizeof(double) * (size_t)L * D);
            double qd[1024];
            for (int t = 0; t < L; ++t) {
                const int64_t row = fp8_token_row(table_row, t, block_size, num_kv_heads, g, D);
                for (int d = 0; d < D; ++d) {
                    Kc[(int64_t)t * D + d] = oracle_e4m3_value(k_cache[row + d]) * (double)k_scales[g];
                    Vc[(int64_t)t * D + d] = oracle_e4m3_value(v_cache[row + d]) * (double)v_scales[g];
                }
            }
            for (int d = 0; d < D; ++d)
                qd[d] = load_elem(q, ((int64_t)s * num_heads + h) * D + d, ORACLE_BF16);
            attend_rows(o, qd, Kc, Vc, L, D, scale);
            free(Kc);
            free(Vc);
        }
    }
    return 0;
}
