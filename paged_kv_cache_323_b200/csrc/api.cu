// api.cu -- the C ABI of libpagedkv.so (declared in include/pagedkv.h):
// argument validation, status codes, launch selection, the library-owned
// split-K workspace, the per-device error word and the launch profiler.
// Every compute step runs in the kernels of decode_attn.cuh, decode_tc.cuh,
// decode_tc_fp8.cuh and kv_ops.cuh.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <climits>
#include <mutex>
#include <vector>

#include "../../include/pagedkv.h"
#include "kv_ops.cuh"
#include "launch.h"
#include "plan.cuh"

// One error record per device (a __device__ variable exists once per device
// context): [0] the first device fault's status, [1] the source line of the
// first failed index check (debug builds only).  Kernels receive its device
// address; pkv_get_device_error reads and clears [0], pkv_debug_failed_line [1].
__device__ int g_pkv_device_error[2];

namespace {

constexpr int kMaxDevices = 64;
constexpr int kAutoPartitionTokens = 1024;
constexpr int kMinPartitionTokens = 512;  // bounds the automatic choice from below
constexpr int kMaxPartitionTokens = 4096;

// Library-owned split-K workspace of paged_attention_decode: one buffer per
// (device, stream), grown stream-ordered on that stream.
struct StreamWorkspace {
    int dev;
    cudaStream_t stream;
    void* ptr;
    size_t bytes;
};

std::mutex g_mu;
std::vector<StreamWorkspace> g_stream_ws;
std::atomic<int> g_tc_gqa{1};  // tensor-core kernel for grouped-query heads where it applies
// Longest-first schedule of the decode grid: 0 never, 1 where it pays (the
// tensor-core kernels with 2 to 4 partitions per sequence), 2 always.
std::atomic<int> g_longest_first{1};
// fp8 tensor-core decode in persistent form where a workspace holds its queue
std::atomic<int> g_fp8_persistent{1};
// register-streamed kernel for bf16 MHA over 8-token blocks (else the staged one)
std::atomic<int> g_reg_stream{1};
std::atomic<unsigned long long> g_launches{0};
std::atomic<unsigned long long> g_wait_ns{pkv::kWaitTimeoutNs};  // decode pipeline wait limit

// ---------------------------------------------------------- profiler
struct ProfRecord {
    int kind;
    int device;
    cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof;
std::vector<std::pair<int, cudaEvent_t>> g_free_events;  // (device, event)

cudaEvent_t take_event(int dev) {
    for (size_t i = 0; i < g_free_events.size(); ++i) {
        if (g_free_events[i].first == dev) {
            cudaEvent_t e = g_free_events[i].second;
            g_free_events[i] = g_free_events.back();
            g_free_events.pop_back();
            return e;
        }
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

int current_device(int* dev) {
    if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return PKV_ERR_CUDA;
    return PKV_OK;
}

// Device address of the current device's error word.  Looked up on every
// call (a symbol lookup, no allocation), so it stays right if the caller
// resets the device and a new context takes the old one's place.
int error_word(int dev, int** out) {
    (void)dev;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pkv_device_error) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return PKV_ERR_CUDA;
    }
    *out = static_cast<int*>(p);
    return PKV_OK;
}

// Launch `kernels` kernels through `fn`, counting them and (when profiling)
// bracketing them with one pair of events on their stream.
template <class Fn>
int launch(int kind, cudaStream_t st, Fn&& fn, int kernels = 1) {
    cudaEvent_t a = nullptr, b = nullptr;
    int dev = 0;
    bool prof = false;
    {
        std::lock_guard<std::mutex> lk(g_prof_mu);
        prof = g_prof_on;
        if (prof) {
            cudaGetDevice(&dev);
            a = take_event(dev);
            b = take_event(dev);
            prof = a && b;
        }
    }
    if (prof) cudaEventRecord(a, st);
    cudaError_t e = fn();
    if (e == cudaSuccess) e = cudaGetLastError();
    g_launches.fetch_add((unsigned long long)kernels);
    if (prof) {
        cudaEventRecord(b, st);
        std::lock_guard<std::mutex> lk(g_prof_mu);
        g_prof.push_back(ProfRecord{kind, dev, a, b});
    }
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elt_bytes(int dtype) { return dtype == PKV_F32 ? 4 : dtype == PKV_FP8_E4M3 ? 1 : 2; }

bool known_dtype(int dtype) { return dtype == PKV_F32 || dtype == PKV_BF16 || dtype == PKV_FP8_E4M3; }

bool decode_shape_supported(int head_dim, int block_size, int group) {
    const bool d_ok = head_dim == 64 || head_dim == 128;
    const bool bs_ok = block_size == 8 || block_size == 16 || block_size == 32;
    const bool g_ok = group == 1 || group == 2 || group == 4 || group == 8;
    return d_ok && bs_ok && g_ok;
}


size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Decode workspace.  First the counters, in a region that nothing else is
// ever written to: the persistent kernels' work queue (16 ints at offset 0)
// and the split-K merge counters, one int per (sequence, kv head), in at
// least kFixedCounterSlots slots; then the longest-first schedule of the
// launch ([B * P] int2); then, when sequences are split, the fp32 partial
// outputs [B][H][P][D] and the (m, l) pairs [B][H][P]; each region 256-byte
// aligned.  Every launch, complete or stopped by a timeout, leaves the
// counters it used at zero, so the fixed region is zero between calls
// whatever shape each call has.  A batch with more (sequence, kv head)
// units than kFixedCounterSlots also uses counters past the fixed region,
// where an earlier call may have left other data: decode_impl clears that
// part on every such call.
constexpr long long kFixedCounterSlots = 65536;
constexpr size_t kWorkBytes = 64;  // the work queue's counters

struct WorkspaceLayout {
    size_t work_off, cnt_off, plan_off, o_off, ml_off, total;
};

WorkspaceLayout workspace_layout(long long num_seqs, long long num_heads, long long parts, long long D) {
    WorkspaceLayout w{0, 0, 0, 0, 0, 0};
    if (num_seqs <= 0 || parts <= 0) return w;
    const long long slots = num_seqs * num_heads > kFixedCounterSlots ? num_seqs * num_heads
                                                                      : kFixedCounterSlots;
    w.work_off = 0;
    w.cnt_off = kWorkBytes;
    w.plan_off = align256(kWorkBytes + size_t(slots) * sizeof(int));
    w.o_off = w.plan_off + align256(size_t(num_seqs) * parts * sizeof(int2));
    w.ml_off = w.o_off;
    w.total = w.o_off;
    if (parts > 1) {
        w.ml_off = w.o_off + align256(size_t(num_seqs) * num_heads * parts * D * sizeof(float));
        w.total = w.ml_off + align256(size_t(num_seqs) * num_heads * parts * sizeof(float2));
    }
    return w;
}

size_t workspace_bytes_for(long long num_seqs, long long num_heads, long long parts, long long D) {
    return workspace_layout(num_seqs, num_heads, parts, D).total;
}

// Partition size when the caller passes 0.
//  * CUDA-core kernels: 1024 tokens (fewer split-K merges than 512 at no loss
//    of parallelism on batch-64 MHA; 2048 for tokens of at most 256 bytes
//    per kv head), doubled (up to 4096) while a sequence
//    of the maximum length would still be split into more than 64 partitions
//    and the grid keeps at least four waves of 3 CTAs per SM.
//  * Tensor-core kernels: 4096 tokens, halved (down to 512) while the grid
//    would have fewer than min_ctas CTAs (4 × 148 × 2 unless given).  Their CTAs carry a
//    fixed set-up and drain cost, so long partitions pay: on B200 the
//    parallel-sampling GQA batch ran at 0.75 / 0.88 / 0.97 of peak with
//    1024 / 2048 / 4096-token partitions.
int auto_partition_tokens(long long num_seqs, long long num_kv_heads, long long max_ctx, bool tc,
                          bool short_tokens = false, long long min_ctas = 4LL * 148 * 2) {
    if (tc) {
        // The tensor-core kernels run 2 to 4 CTAs per SM, and a CTA's start
        // (table and q fetch, first TMA round trip) and merge are a fixed
        // cost: keep partitions as long as the grid still gives 4 waves of 2
        // CTAs per SM (batch-8 128K-token GQA: 543 us at 4096 tokens, 565 us
        // at 2048; the fp8 parallel-sampling batch at 4 CTAs per SM: 153 /
        // 171 / 209 us at 4096 / 2048 / 1024).
        long long pt = kMaxPartitionTokens;
        while (pt > kMinPartitionTokens && num_seqs * num_kv_heads * ((max_ctx + pt - 1) / pt) < min_ctas)
            pt /= 2;
        return (int)pt;
    }
    // Where a token of one kv head carries at most 256 bytes of K and V (fp8
    // caches, bf16 at head_dim 64) a CTA's fixed cost weighs twice as much
    // per token: 2048 tokens (batch-64 MHA over fp8 on the staged kernel:
    // 154 us at 1024, 139 us at 2048; bf16 at head_dim 64 on the
    // register-streamed kernel: 104.7 / 102.4 us), against 1024 for 512-byte
    // tokens (bf16 at head_dim 128: 194.3 us at 1024, 200.9 at 2048)
    long long pt = short_tokens ? 2 * kAutoPartitionTokens : kAutoPartitionTokens;
    const long long min_cc_ctas = 4LL * 148 * 3;
    while (pt < kMaxPartitionTokens && (max_ctx + pt - 1) / pt > 64 &&
           num_seqs * num_kv_heads * ((max_ctx + 2 * pt - 1) / (2 * pt)) >= min_cc_ctas)
        pt *= 2;
    return (int)pt;
}

// Whether the tensor-core kernel serves this shape (any partition size that
// is a multiple of 128 tokens).
bool tc_shape(int dtype, int head_dim, int block_size, int group, int num_kv_heads) {
    return g_tc_gqa.load() != 0 &&
           pkv::decode_tc_supported(dtype, head_dim, block_size, group, num_kv_heads, 128);
}

int resolve_partition_tokens(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                             int block_size, long long max_ctx, int dtype, int partition_tokens) {
    if (partition_tokens != 0) return partition_tokens;
    const int group = num_kv_heads > 0 ? num_heads / num_kv_heads : 1;
    const bool tc = tc_shape(dtype, head_dim, block_size, group, num_kv_heads);
    const bool fp8 = dtype == PKV_FP8_E4M3;
    const int elt = dtype == PKV_F32 ? 4 : (dtype == PKV_BF16 ? 2 : 1);
    const bool short_tokens = 2LL * head_dim * elt <= 256;  // K and V bytes of one token, one kv head
    // The head_dim-64 tensor-core kernel runs one CTA per pair of kv heads,
    // always in longest-first order, where the last CTAs to start are the
    // shortest: its partitions stay long while the grid fills one wave of 5
    // CTAs per SM (batch-64 MHA: 59.3 us at 2048 tokens, 68.4 at 1024, 76.1
    // at 512).
    const bool pairs = tc && head_dim == 64;
    int pt = pairs ? auto_partition_tokens(num_seqs, num_kv_heads / 2, max_ctx, tc, short_tokens, 148LL * 5)
                   : auto_partition_tokens(num_seqs, num_kv_heads, max_ctx, tc, short_tokens);
    // the persistent fp8 tensor-core kernel holds two tables of at most 128
    // blocks per CTA: 2048 tokens at block size 16 (batch-64 MHA 106.5 us at
    // 2048 against 112.1 us at 1024; the parallel-sampling batch 125.3 / 144.1)
    if (tc && fp8 && head_dim == 128 && g_fp8_persistent.load() != 0 &&
        pkv::decode_tc_fp8_persistent_supported(block_size, group, 128)) {
        const int cap = pkv::decode_tc_fp8_persistent_max_tokens(block_size);
        if (pt > cap) pt = cap;
    }
    return pt;
}

}  // namespace

// Not exported: the workspace paged_attention_decode_ex needs for the
// partition size it would pick, and where the merge counters sit in it.
extern "C" void pkv_internal_decode_scratch(int num_seqs, int num_heads, int num_kv_heads,
                                            int head_dim, int block_size, int max_blocks_per_seq,
                                            int dtype, int partition_tokens, size_t* total,
                                            size_t* cnt_off, size_t* cnt_bytes) {
    *total = *cnt_off = *cnt_bytes = 0;
    if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        max_blocks_per_seq <= 0 || partition_tokens < 0)
        return;
    const long long max_ctx = (long long)max_blocks_per_seq * block_size;
    const long long pt = resolve_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim,
                                                  block_size, max_ctx, dtype, partition_tokens);
    const long long parts = (max_ctx + pt - 1) / pt;
    const WorkspaceLayout w = workspace_layout(num_seqs, num_heads, parts, head_dim);
    *total = w.total;
    if (w.total > 0) {  // the work queue and the merge counters this batch uses
        *cnt_off = w.work_off;
        *cnt_bytes = w.cnt_off + size_t(num_seqs) * num_kv_heads * sizeof(int);
    }
}

extern "C" {

size_t paged_attention_workspace_size(int num_seqs, int num_heads, int max_context, int head_dim,
                                      int partition_tokens) {
    if (num_seqs <= 0 || num_heads <= 0 || max_context <= 0 || head_dim <= 0 ||
        partition_tokens < 0)
        return 0;
    // the automatic size is never below kMinPartitionTokens, which bounds its workspace
    const long long pt = partition_tokens == 0 ? kMinPartitionTokens : partition_tokens;
    const long long parts = (max_context + pt - 1) / pt;
    return workspace_bytes_for(num_seqs, num_heads, parts, head_dim);
}

int paged_attention_partition_tokens(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                     int block_size, int max_context, int dtype,
                                     int partition_tokens) {
    if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || max_context <= 0 ||
        partition_tokens < 0)
        return 0;
    return resolve_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                    max_context, dtype, partition_tokens);
}

}  // extern "C"

namespace {

// Shared body of the decode entry points.  dtype: q and out; kv_dtype: the
// caches (dtype itself, or PKV_FP8_E4M3 with bf16 q / out and per-kv-head
// scales k_scales / v_scales in device memory).
int decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                const float* k_scales, const float* v_scales, const int32_t* block_tables,
                const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                int head_dim, int block_size, int max_blocks_per_seq, float scale, int num_blocks,
                int dtype, int kv_dtype, int partition_tokens, void* workspace,
                size_t workspace_bytes, void* stream) {
    if (num_seqs < 0) return PKV_ERR_INVALID;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_ERR_NULL;
    if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0) return PKV_ERR_INVALID;
    if (head_dim <= 0 || block_size <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0)
        return PKV_ERR_INVALID;
    if (dtype != PKV_F32 && dtype != PKV_BF16) return PKV_ERR_INVALID;
    const bool fp8 = kv_dtype == PKV_FP8_E4M3;
    if (kv_dtype != dtype && !(fp8 && dtype == PKV_BF16)) return PKV_ERR_INVALID;
    if (fp8 && (!k_scales || !v_scales)) return PKV_ERR_NULL;
    if (!isfinite(scale)) return PKV_ERR_INVALID;
    const int group = num_heads / num_kv_heads;
    if (!decode_shape_supported(head_dim, block_size, group)) return PKV_ERR_UNSUPPORTED;
    if (partition_tokens < 0 || partition_tokens > kMaxPartitionTokens ||
        partition_tokens % block_size != 0)
        return PKV_ERR_INVALID;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_ERR_INVALID;
    const long long max_ctx = (long long)max_blocks_per_seq * block_size;
    if (max_ctx > INT_MAX) return PKV_ERR_INVALID;
    const int pt = resolve_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim,
                                            block_size, max_ctx, kv_dtype, partition_tokens);
    const long long parts = (max_ctx + pt - 1) / pt;
    const bool use_tc = g_tc_gqa.load() != 0 &&
                        pkv::decode_tc_supported(kv_dtype, head_dim, block_size, group, num_kv_heads, pt);
    const bool use_reg = !use_tc && g_reg_stream.load() != 0 &&
                         pkv::decode_reg_supported(kv_dtype, head_dim, block_size, group);
    const long long grid = parts * num_kv_heads * (long long)num_seqs;
    if (grid > INT_MAX || (long long)num_seqs * num_heads > INT_MAX) return PKV_ERR_INVALID;
    const size_t need = workspace_bytes_for(num_seqs, num_heads, parts, head_dim);
    // Split-K needs the workspace.  Without a split it only holds the
    // longest-first schedule: a NULL workspace then runs in index order.
    if (parts > 1 || workspace != nullptr) {
        if (workspace == nullptr || workspace_bytes < need ||
            (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
            return PKV_ERR_WORKSPACE;
    }
    int dev = 0;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    int* err = nullptr;
    if (error_word(dev, &err) != PKV_OK) return PKV_ERR_CUDA;

    pkv::DecodeParams p;
    p.out = out;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    const WorkspaceLayout wl = workspace_layout(num_seqs, num_heads, parts, head_dim);
    char* wsb = static_cast<char*>(workspace);
    const bool split = parts > 1;
    p.ws_o = split ? reinterpret_cast<float*>(wsb + wl.o_off) : nullptr;
    p.ws_ml = split ? reinterpret_cast<float2*>(wsb + wl.ml_off) : nullptr;
    p.counters = split ? reinterpret_cast<int*>(wsb + wl.cnt_off) : nullptr;
    p.work = workspace != nullptr ? reinterpret_cast<int*>(wsb + wl.work_off) : nullptr;
    // The schedule pays where index order leaves the longest work for last:
    // the tensor-core kernels run 2 to 4 partitions per sequence
    // partition-major, so the later partitions, which only the longest
    // sequences have, come at the end of the launch (parallel-sampling batch:
    // 257 -> 250 us bf16), and the persistent fp8 kernel takes its units in
    // queue order, so a long unit taken last runs alone (parallel-sampling
    // batch 136.2 -> 125.3 us, batch-64 MHA 109.6 -> 106.5 us).  Elsewhere it
    // does not: with one partition per sequence and nearly equal lengths (a
    // shared-prefix batch) longest first starts the CTAs in synchronised
    // waves that read the shared blocks in step (+4 %), and the planning
    // kernel itself costs about 4 us per launch.
    const bool persistent = use_tc && fp8 && head_dim == 128 && workspace != nullptr &&
                            g_fp8_persistent.load() != 0 &&
                            pkv::decode_tc_fp8_persistent_supported(block_size, group, pt);
    const int sched = g_longest_first.load();
    const bool pairs = use_tc && head_dim == 64;  // head_dim-64 kernel (batch-64 MHA 67.2 -> 59.3 us)
    const bool plan = workspace != nullptr &&
                      (sched == 2 ||
                       (sched == 1 && (persistent || pairs || (use_tc && parts >= 2 && parts <= 4))));
    int2* order = plan ? reinterpret_cast<int2*>(wsb + wl.plan_off) : nullptr;
    p.order = order;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long units = (long long)num_seqs * num_kv_heads;
    if (split && units > kFixedCounterSlots) {
        // counters past the fixed region may hold an earlier call's partials
        if (cudaMemsetAsync(wsb + wl.cnt_off + kFixedCounterSlots * sizeof(int), 0,
                            size_t(units - kFixedCounterSlots) * sizeof(int), st) != cudaSuccess)
            return PKV_ERR_CUDA;
    }
    p.k_scales = fp8 ? k_scales : nullptr;
    p.v_scales = fp8 ? v_scales : nullptr;
    p.err = err;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.partition_tokens = pt;
    p.num_partitions = (int)parts;
    p.qscale = scale * 1.4426950408889634f;  // log2(e): softmax runs in base 2
    p.wait_ns = g_wait_ns.load();

    // the schedule first (one CTA), then the decode grid as its programmatic
    // dependent: counted and profiled together as the decode
    return launch(PKV_KERNEL_DECODE, st, [&] {
        if (order != nullptr) {
            pkv::plan_kernel<<<1, pkv::kPlanThreads, 0, st>>>(context_lens, num_seqs, (int)parts, pt,
                                                            (int)max_ctx, order, err);
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        if (use_tc)
            return pkv::launch_decode_tc(p, kv_dtype, head_dim, block_size, group, grid, persistent, st);
        if (use_reg) return pkv::launch_decode_reg(p, head_dim, block_size, group, grid, st);
        if (fp8) return pkv::launch_decode_partition_fp8(p, head_dim, block_size, group, grid, st);
        return dtype == PKV_F32 ? pkv::launch_decode_partition_f32(p, head_dim, block_size, group, grid, st)
                                : pkv::launch_decode_partition_bf16(p, head_dim, block_size, group, grid, st);
    }, order != nullptr ? 2 : 1);
}

}  // namespace

extern "C" {

int paged_attention_decode_ex(void* out, const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, const int32_t* context_lens,
                              int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int max_blocks_per_seq, float scale, int num_blocks,
                              int dtype, int partition_tokens, void* workspace,
                              size_t workspace_bytes, void* stream) {
    return decode_impl(out, q, k_cache, v_cache, nullptr, nullptr, block_tables, context_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                       max_blocks_per_seq, scale, num_blocks, dtype, dtype, partition_tokens,
                       workspace, workspace_bytes, stream);
}

int paged_attention_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const float* k_scales, const float* v_scales,
                               const int32_t* block_tables, const int32_t* context_lens,
                               int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                               int block_size, int max_blocks_per_seq, float scale,
                               int num_blocks, int partition_tokens, void* workspace,
                               size_t workspace_bytes, void* stream) {
    return decode_impl(out, q, k_cache, v_cache, k_scales, v_scales, block_tables, context_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                       max_blocks_per_seq, scale, num_blocks, PKV_BF16, PKV_FP8_E4M3,
                       partition_tokens, workspace, workspace_bytes, stream);
}

int paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                           int num_heads, int num_kv_heads, int head_dim, int block_size,
                           int max_blocks_per_seq, float scale, void* stream) {
    if (num_seqs < 0) return PKV_ERR_INVALID;
    if (num_seqs == 0) return PKV_OK;
    if (num_heads <= 0 || head_dim <= 0 || block_size <= 0 || max_blocks_per_seq <= 0)
        return PKV_ERR_INVALID;
    const long long max_ctx = (long long)max_blocks_per_seq * block_size;
    if (max_ctx > INT_MAX) return PKV_ERR_INVALID;
    const size_t need = paged_attention_workspace_size(num_seqs, num_heads, (int)max_ctx, head_dim, 0);
    void* ws = nullptr;
    if (need > 0) {  // always: the workspace holds the schedule
        int dev = 0;
        if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        std::lock_guard<std::mutex> lk(g_mu);
        StreamWorkspace* d = nullptr;
        for (StreamWorkspace& e : g_stream_ws)
            if (e.dev == dev && e.stream == st) d = &e;
        if (d == nullptr) {
            g_stream_ws.push_back(StreamWorkspace{dev, st, nullptr, 0});
            d = &g_stream_ws.back();
        }
        if (d->bytes < need) {
            // grow on the call's stream: calls on it are ordered, so the old
            // buffer is released only after the launches that read it
            cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
            if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return PKV_ERR_CUDA;
            if (cap != cudaStreamCaptureStatusNone) return PKV_ERR_WORKSPACE;
            size_t grow = need + need / 4;
            void* fresh = nullptr;
            if (cudaMallocAsync(&fresh, grow, st) != cudaSuccess) return PKV_ERR_CUDA;
            if (cudaMemsetAsync(fresh, 0, grow, st) != cudaSuccess) return PKV_ERR_CUDA;  // counters start at 0
            if (d->ptr != nullptr && cudaFreeAsync(d->ptr, st) != cudaSuccess) return PKV_ERR_CUDA;
            d->ptr = fresh;
            d->bytes = grow;
        }
        ws = d->ptr;
    }
    return paged_attention_decode_ex(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                                     num_heads, num_kv_heads, head_dim, block_size,
                                     max_blocks_per_seq, scale, INT_MAX, PKV_BF16, 0, ws, need,
                                     stream);
}

int kv_cache_append(void* k_cache, void* v_cache, const void* k, const void* v,
                    const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int dtype, void* stream) {
    if (num_tokens < 0) return PKV_ERR_INVALID;
    if (num_tokens == 0) return PKV_OK;
    if (!k_cache || !v_cache || !k || !v || !slot_mapping) return PKV_ERR_NULL;
    if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PKV_ERR_INVALID;
    if (dtype != PKV_F32 && dtype != PKV_BF16) return PKV_ERR_INVALID;
    const int row_bytes = head_dim * elt_bytes(dtype);
    if (row_bytes % 16 != 0 || row_bytes > 256 * 16) return PKV_ERR_UNSUPPORTED;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v))
        return PKV_ERR_INVALID;
    int dev = 0;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    int* err = nullptr;
    if (error_word(dev, &err) != PKV_OK) return PKV_ERR_CUDA;
    pkv::AppendParams p;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.k = k;
    p.v = v;
    p.slot_mapping = slot_mapping;
    p.err = err;
    p.num_slots = (long long)num_blocks * block_size;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.chunks_per_row = row_bytes / 16;
    const long long rows = (long long)num_tokens * num_kv_heads;
    const long long rows_per_cta = 256 / p.chunks_per_row;
    long long blocks = (rows + rows_per_cta - 1) / rows_per_cta;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launch(PKV_KERNEL_APPEND, st, [&] {
        pkv::kv_append_kernel<<<(unsigned)blocks, 256, 0, st>>>(p);
        return cudaGetLastError();
    });
}

int kv_cache_append_fp8(void* k_cache, void* v_cache, const float* k_scales,
                        const float* v_scales, const void* k, const void* v,
                        const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, void* stream) {
    if (num_tokens < 0) return PKV_ERR_INVALID;
    if (num_tokens == 0) return PKV_OK;
    if (!k_cache || !v_cache || !k_scales || !v_scales || !k || !v || !slot_mapping)
        return PKV_ERR_NULL;
    if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PKV_ERR_INVALID;
    if (head_dim % 16 != 0 || head_dim > 256 * 16) return PKV_ERR_UNSUPPORTED;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v))
        return PKV_ERR_INVALID;
    int dev = 0;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    int* err = nullptr;
    if (error_word(dev, &err) != PKV_OK) return PKV_ERR_CUDA;
    pkv::AppendFp8Params p;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.k_scales = k_scales;
    p.v_scales = v_scales;
    p.k = k;
    p.v = v;
    p.slot_mapping = slot_mapping;
    p.err = err;
    p.num_slots = (long long)num_blocks * block_size;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.chunks_per_row = head_dim / 16;
    const long long rows = (long long)num_tokens * num_kv_heads;
    const long long rows_per_cta = 256 / p.chunks_per_row;
    long long blocks = (rows + rows_per_cta - 1) / rows_per_cta;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launch(PKV_KERNEL_APPEND, st, [&] {
        pkv::kv_append_fp8_kernel<<<(unsigned)blocks, 256, 0, st>>>(p);
        return cudaGetLastError();
    });
}

int copy_blocks(void* k_cache, void* v_cache, const int64_t* src_dst_pairs, int num_pairs,
                int num_kv_heads, int head_dim, int block_size, int num_blocks, int dtype,
                void* stream) {
    if (num_pairs < 0) return PKV_ERR_INVALID;
    if (num_pairs == 0) return PKV_OK;
    if (!k_cache || !v_cache || !src_dst_pairs) return PKV_ERR_NULL;
    if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PKV_ERR_INVALID;
    if (!known_dtype(dtype)) return PKV_ERR_INVALID;
    const long long block_bytes = (long long)num_kv_heads * block_size * head_dim * elt_bytes(dtype);
    if (block_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return PKV_ERR_INVALID;
    int dev = 0;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    int* err = nullptr;
    if (error_word(dev, &err) != PKV_OK) return PKV_ERR_CUDA;
    pkv::CopyParams p;
    p.dst_k = k_cache;
    p.dst_v = v_cache;
    p.src_k = k_cache;
    p.src_v = v_cache;
    p.pairs = src_dst_pairs;
    p.err = err;
    p.chunks_per_block = block_bytes / 16;
    p.num_pairs = num_pairs;
    p.num_src_blocks = num_blocks;
    p.num_dst_blocks = num_blocks;
    long long per_pair = (p.chunks_per_block + 1023) / 1024;  // 256 threads x 4 chunks
    if (per_pair > 64) per_pair = 64;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launch(PKV_KERNEL_COPY_BLOCKS, st, [&] {
        pkv::copy_blocks_kernel<<<dim3((unsigned)num_pairs, (unsigned)per_pair), 256, 0, st>>>(p);
        return cudaGetLastError();
    });
}

int swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                const int64_t* src_dst_pairs, int num_pairs, int num_kv_heads, int head_dim,
                int block_size, int num_src_blocks, int num_dst_blocks, int dtype, void* stream) {
    if (num_pairs < 0) return PKV_ERR_INVALID;
    if (num_pairs == 0) return PKV_OK;
    if (!dst_k || !dst_v || !src_k || !src_v || !src_dst_pairs) return PKV_ERR_NULL;
    if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_src_blocks <= 0 ||
        num_dst_blocks <= 0)
        return PKV_ERR_INVALID;
    if (!known_dtype(dtype)) return PKV_ERR_INVALID;
    const long long block_bytes = (long long)num_kv_heads * block_size * head_dim * elt_bytes(dtype);
    if (block_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
    // every pointer must be device memory or page-locked host memory the
    // device can reach; host pointers are replaced by their device mapping
    const void* ptrs[5] = {dst_k, dst_v, src_k, src_v, src_dst_pairs};
    void* mapped[5];
    for (int i = 0; i < 5; ++i) {
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, ptrs[i]) != cudaSuccess) {
            cudaGetLastError();
            return PKV_ERR_INVALID;
        }
        if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
            mapped[i] = const_cast<void*>(ptrs[i]);
        } else if (a.type == cudaMemoryTypeHost && a.devicePointer != nullptr) {
            mapped[i] = static_cast<char*>(a.devicePointer) +
                        (static_cast<const char*>(ptrs[i]) - static_cast<const char*>(a.hostPointer));
        } else {
            return PKV_ERR_INVALID;  // pageable host memory: pin it first
        }
        if (i < 4 && (reinterpret_cast<uintptr_t>(mapped[i]) & 15u) != 0) return PKV_ERR_INVALID;
    }
    int dev = 0;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    int* err = nullptr;
    if (error_word(dev, &err) != PKV_OK) return PKV_ERR_CUDA;
    pkv::CopyParams p;
    p.dst_k = mapped[0];
    p.dst_v = mapped[1];
    p.src_k = mapped[2];
    p.src_v = mapped[3];
    p.pairs = static_cast<const int64_t*>(mapped[4]);
    p.err = err;
    p.chunks_per_block = block_bytes / 16;
    p.num_pairs = num_pairs;
    p.num_src_blocks = num_src_blocks;
    p.num_dst_blocks = num_dst_blocks;
    long long per_pair = (p.chunks_per_block + 1023) / 1024;
    if (per_pair > 64) per_pair = 64;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launch(PKV_KERNEL_SWAP_BLOCKS, st, [&] {
        pkv::copy_blocks_kernel<<<dim3((unsigned)num_pairs, (unsigned)per_pair), 256, 0, st>>>(p);
        return cudaGetLastError();
    });
}

int pkv_selftest_bounded_wait(int timeout_us, void* stream) {
    if (timeout_us <= 0 || timeout_us > 1000000) return PKV_ERR_INVALID;
    int dev = 0;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    int* err = nullptr;
    if (error_word(dev, &err) != PKV_OK) return PKV_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    pkv::bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(err, 1000ull * (unsigned long long)timeout_us);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_debug_build(void) {
#ifdef PKV_DEBUG
    return 1;
#else
    return 0;
#endif
}

int pkv_debug_failed_line(void* stream, int* line) {
    if (!line) return PKV_ERR_NULL;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PKV_ERR_CUDA;
    int dev = 0;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    int* err = nullptr;
    if (error_word(dev, &err) != PKV_OK) return PKV_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, err + 1, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return PKV_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(err + 1, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return PKV_ERR_CUDA;
    *line = v;
    return PKV_OK;
}

int pkv_get_device_error(void* stream, int* code) {
    if (!code) return PKV_ERR_NULL;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PKV_ERR_CUDA;
    int dev = 0;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    int* err = nullptr;
    if (error_word(dev, &err) != PKV_OK) return PKV_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, err, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return PKV_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(err, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return PKV_ERR_CUDA;
    *code = v;
    return PKV_OK;
}

const char* pkv_status_string(int status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_ERR_NULL: return "a required pointer is NULL";
        case PKV_ERR_INVALID: return "an argument is out of range";
        case PKV_ERR_UNSUPPORTED: return "no kernel for this shape or type";
        case PKV_ERR_CUDA: return "CUDA runtime error";
        case PKV_ERR_WORKSPACE: return "split-K workspace missing or too small";
        case PKV_ERR_DEVICE_BOUNDS: return "device: table entry, slot or context length out of range";
        case PKV_ERR_TIMEOUT: return "device: a bounded wait ran out of time";
        case PKV_ERR_OUT_OF_BLOCKS: return "no free block left in the pool (preempt and retry)";
        default: return "unknown status";
    }
}

int pkv_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = on != 0;
    return PKV_OK;
}

int pkv_profile_read(int kind, long long* launches, double* total_ms) {
    if (!launches || !total_ms) return PKV_ERR_NULL;
    if (kind < 0 || kind >= PKV_KERNEL_KINDS) return PKV_ERR_INVALID;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    long long n = 0;
    double ms = 0.0;
    for (const ProfRecord& r : g_prof) {
        if (r.kind != kind) continue;
        if (cudaEventSynchronize(r.stop) != cudaSuccess) return PKV_ERR_CUDA;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) return PKV_ERR_CUDA;
        ms += t;
        ++n;
    }
    *launches = n;
    *total_ms = ms;
    return PKV_OK;
}

int pkv_profile_reset(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (const ProfRecord& r : g_prof) {
        cudaEventSynchronize(r.stop);
        g_free_events.emplace_back(r.device, r.start);
        g_free_events.emplace_back(r.device, r.stop);
    }
    g_prof.clear();
    return PKV_OK;
}

unsigned long long pkv_launch_count(void) { return g_launches.load(); }

int pkv_set_wait_limit_us(int microseconds) {
    if (microseconds < 0 || microseconds > 1000000) return PKV_ERR_INVALID;
    const unsigned long long ns =
        microseconds == 0 ? pkv::kWaitTimeoutNs : 1000ull * (unsigned long long)microseconds;
    return (int)(g_wait_ns.exchange(ns) / 1000ull);
}

int pkv_set_longest_first(int mode) {
    if (mode < 0 || mode > 2) return PKV_ERR_INVALID;
    return g_longest_first.exchange(mode);
}

PKV_API int pkv_internal_set_fp8_persistent(int enable) {
    return g_fp8_persistent.exchange(enable != 0 ? 1 : 0);
}

PKV_API int pkv_internal_set_reg_stream(int enable) {
    return g_reg_stream.exchange(enable != 0 ? 1 : 0);
}

int pkv_set_tensor_core_gqa(int enable) {
    return g_tc_gqa.exchange(enable != 0 ? 1 : 0);
}

int pkv_version(void) { return 100; }

}  // extern "C"
