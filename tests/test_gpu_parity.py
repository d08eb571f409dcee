"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Bars: append / copy / pool state bit-exact; attention max abs error <= 1e-5
for fp32 caches, |gpu - ref| <= 2e-2 + 1e-2 |ref| for bf16 caches.  Reduced
versions of every workload and the full-size workloads are all compared
element by element (the full sizes through a compact host copy of the
blocks they reference).
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_323_b200 import workload as wl
from steps import assert_close, assert_pool_equal, full_size_check, gpu_step, oracle_step, to_device

pytestmark = pytest.mark.gpu


def _full_check(w, partition_tokens=0):
    ref, kref, vref = oracle_step(w)
    out, kc, vc = gpu_step(w, partition_tokens=partition_tokens)
    assert_pool_equal(kc, kref, "k pool")
    assert_pool_equal(vc, vref, "v pool")
    return assert_close(out, ref, w.dtype)


# ------------------------------------------------------- reduced workloads
@pytest.mark.parametrize("pt", [0, 16, 32])
def test_tiny_fp32(pt):
    w = wl.tiny()
    _full_check(w, partition_tokens=pt)


@pytest.mark.parametrize("pt", [0, 64])
def test_mha_reduced(pt):
    w = wl.mha(num_seqs=8, num_blocks=2048)
    _full_check(w, partition_tokens=pt)


@pytest.mark.parametrize("bs", [8, 32])
def test_mha_contiguous_reduced(bs):
    """The contiguous-placement comparator computes the same attention."""
    w = wl.mha(num_seqs=6, num_blocks=2048 * 16 // bs, block_size=bs, contiguous=True)
    _full_check(w)


def test_gqa_sampling_reduced():
    w = wl.gqa_sampling(groups=6, prompt_median=300, prompt_max=2000)
    assert len(w.cow_pairs) > 0
    _full_check(w)


def test_long_context_reduced():
    w = wl.long_context(num_seqs=2, ctx_range=(3000, 9000))
    _full_check(w)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_prefix_sweep_reduced(bs):
    w = wl.prefix_sweep(bs, num_seqs=12, prefix=256, suffix_range=(16, 200))
    _full_check(w)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_shape_grid(dtype, D, bs, G):
    """Every supported (dtype, head_dim, block_size, group) on ragged lengths
    that span several partitions and end mid-block."""
    lens = [1, bs - 1, bs, 3 * bs + 5, 700, 1111]
    w = wl.custom(100 + G, lens, heads=2 * G, kv_heads=2, head_dim=D, block_size=bs, dtype=dtype,
                  maxb=-(-1111 // bs) + 2)
    _full_check(w, partition_tokens=256)


# ------------------------------------------------------------ full size
# Every row of every full-size workload (the bench configurations) against
# the oracle, and every pool block the step touches byte for byte.


def test_mha_full():
    """Batch-64 MHA: all 64 x 32 rows."""
    full_size_check(wl.mha(device="cuda"))


def test_gqa_sampling_full():
    """Parallel sampling with copy-on-write: all 256 x 32 rows."""
    full_size_check(wl.gqa_sampling(device="cuda"))


def test_long_context_full():
    """Batch-8 contexts of 32K-128K tokens: all 8 x 64 rows."""
    full_size_check(wl.long_context(device="cuda"))


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_prefix_sweep_full(bs):
    """1024 sequences on one shared prefix: all 1024 x 32 rows per block size."""
    full_size_check(wl.prefix_sweep(bs, device="cuda"))


# ----------------------------------------------------------- invariants
def test_permutation_bit_identical():
    """Blocks can sit anywhere: moving them (data and table together) leaves
    the GPU output bit-identical, since the reduction order is logical."""
    w = wl.mha(num_seqs=6, num_blocks=600, heads=8)
    out1, _, _ = gpu_step(w)
    perm = np.random.default_rng(5).permutation(w.num_blocks)
    w2 = wl.Workload(**{**w.__dict__})
    w2.k_cache = torch.empty_like(w.k_cache)
    w2.v_cache = torch.empty_like(w.v_cache)
    w2.k_cache[torch.from_numpy(perm)] = w.k_cache
    w2.v_cache[torch.from_numpy(perm)] = w.v_cache
    w2.block_tables = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    bs = w.block_size
    w2.slot_mapping = np.asarray([perm[s // bs] * bs + s % bs for s in w.slot_mapping], dtype=np.int64)
    out2, _, _ = gpu_step(w2)
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("make,pt", [
    (lambda: wl.mha(num_seqs=16, num_blocks=3000, heads=8), 0),
    (lambda: wl.mha(num_seqs=16, num_blocks=6000, heads=8, block_size=8), 256),
    (lambda: wl.gqa_sampling(groups=6, prompt_median=500, prompt_max=3000), 0),
    (lambda: wl.gqa_sampling(groups=6, prompt_median=500, prompt_max=3000, dtype="fp8"), 512),
], ids=["mha", "mha_bs8_split", "gqa_tensor_core", "gqa_fp8_split"])
def test_schedule_does_not_change_bits(make, pt):
    """The longest-first schedule only reorders the grid: outputs are
    bit-identical to index order, and both match the oracle."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = make()
    ref, _, _ = oracle_step(w)
    outs = []
    for mode in (2, 0):  # planned longest first, index order
        prev = pk.set_longest_first(mode)
        try:
            out, _, _ = gpu_step(w, partition_tokens=pt)  # the step is idempotent on fresh copies
        finally:
            pk.set_longest_first(prev)
        outs.append(out.clone())
    assert torch.equal(outs[0], outs[1])
    assert_close(outs[0], ref, "bf16" if w.dtype == "fp8" else w.dtype)


def test_shared_blocks_identical_rows():
    """Sequences pointing at the same physical blocks with the same query get
    bit-identical outputs."""
    w = wl.prefix_sweep(16, num_seqs=4, prefix=512, suffix_range=(16, 16))
    w.slot_mapping = np.full_like(w.slot_mapping, -1)  # nothing appended: every row reads the same bytes
    w.block_tables = np.repeat(w.block_tables[:1], 4, axis=0)
    w.context_lens = np.repeat(w.context_lens[:1], 4)
    w.q = w.q[:1].repeat(4, 1, 1).contiguous()
    out, _, _ = gpu_step(w)
    for s in range(1, 4):
        assert torch.equal(out[s], out[0])


def test_copy_on_write_leaves_siblings():
    """Copy-on-write: every block that is neither a copy destination nor an
    append target -- the shared full prompt blocks in particular -- is
    byte-identical before and after the step; the whole pool and every
    output match the oracle."""
    w = wl.gqa_sampling(groups=4, prompt_median=200, prompt_max=800)
    assert len(w.cow_pairs) > 0
    kpre, vpre = w.k_cache.clone(), w.v_cache.clone()
    ref, kref, vref = oracle_step(w)
    out, kc, vc = gpu_step(w)
    written = set(w.cow_pairs[:, 1].tolist()) | set((w.slot_mapping // w.block_size).tolist())
    keep = torch.tensor(sorted(set(range(w.num_blocks)) - written))
    assert torch.equal(kc.cpu()[keep], kpre[keep]) and torch.equal(vc.cpu()[keep], vpre[keep])
    assert_pool_equal(kc, kref, "k pool")
    assert_pool_equal(vc, vref, "v pool")
    assert_close(out, ref, w.dtype)


def test_nan_poisoned_unused_slots():
    """Unused slots, unallocated blocks and table entries past the context
    are poisoned; outputs stay finite and equal to the oracle's, which proves
    nothing outside the context is read."""
    w = wl.mha(num_seqs=6, num_blocks=900, heads=8)
    bs = w.block_size
    used = np.zeros((w.num_blocks, bs), dtype=bool)
    for s in range(w.num_seqs):
        L = int(w.context_lens[s])
        for t in range(L):
            used[w.block_tables[s][t // bs], t % bs] = True
    mask = torch.from_numpy(~used)[:, None, :, None].expand_as(w.k_cache)
    w.k_cache = w.k_cache.masked_fill(mask, float("nan"))
    w.v_cache = w.v_cache.masked_fill(mask, float("nan"))
    # entries past each context point at a poisoned, unused block
    poison_blk = int(np.argmax((~used).all(axis=1)))
    for s in range(w.num_seqs):
        nb = -(-int(w.context_lens[s]) // bs)
        w.block_tables[s, nb:] = poison_blk
    _full_check(w)


def test_single_vs_split_partitions():
    """One partition per sequence and many partitions both meet the bar."""
    w = wl.mha(num_seqs=4, num_blocks=600, heads=4, ctx_range=(1500, 2048))
    ref, _, _ = oracle_step(w)
    for pt in (2048, 512, 128, 16):
        out, _, _ = gpu_step(w, partition_tokens=pt)
        assert_close(out, ref, w.dtype, what=f"partition {pt}")


def test_plain_entry_point_matches_ex():
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.mha(num_seqs=6, num_blocks=900, heads=8)
    t = to_device(w)
    out_ex, _, _ = gpu_step(w, t)
    out2 = torch.empty_like(out_ex)
    pk.paged_attention_decode(out2, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                              t["context_lens"], w.scale)
    torch.cuda.synchronize()
    assert torch.equal(out_ex, out2)


# ------------------------------------------------------------ edge cases
@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("pt", [64, 128, 0])
def test_edge_lengths(dtype, pt):
    """Empty context (zero row), one token, exact block multiples, and the
    maximum context the table can describe; partitions of 64 tokens run the
    CUDA-core kernel, of 128 (and the automatic size) the tensor-core one."""
    bs = 16
    maxb = 12
    lens = [0, 1, bs, 2 * bs, maxb * bs, 5]
    w = wl.custom(7, lens, heads=8, kv_heads=2, head_dim=128, block_size=bs, dtype=dtype, maxb=maxb)
    ref, kref, vref = oracle_step(w)
    out, kc, vc = gpu_step(w, partition_tokens=pt)
    assert_pool_equal(kc, kref, "k pool")
    assert_close(out, ref, "bf16")
    assert torch.count_nonzero(out[0]) == 0


def test_empty_calls_are_noops():
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.tiny()
    t = to_device(w)
    before = t["k_cache"].clone()
    empty_i64 = torch.empty(0, dtype=torch.int64, device="cuda")
    pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"][:0], t["v_new"][:0], empty_i64)
    pk.copy_blocks(t["k_cache"], t["v_cache"], empty_i64.reshape(0, 2))
    q0 = t["q"][:0]
    pk.paged_attention_decode_ex(torch.empty_like(q0), q0, t["k_cache"], t["v_cache"],
                                 t["block_tables"][:0], t["context_lens"][:0], w.scale)
    torch.cuda.synchronize()
    assert torch.equal(before, t["k_cache"])
    assert pk.get_device_error() == 0


def test_skip_slots():
    """slot -1 writes nothing."""
    w = wl.tiny()
    w.slot_mapping[1] = -1
    _full_check(w)


# ------------------------------------------------------- device faults
def test_bad_table_entry_sets_error():
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.mha(num_seqs=3, num_blocks=400, heads=4)
    w.block_tables[1, 2] = w.num_blocks + 7
    t = to_device(w)
    out, _, _ = gpu_step(w, t, check_error=False)
    assert pk.get_device_error() == pk.PKV_ERR_DEVICE_BOUNDS
    assert torch.isfinite(out.float()).all()
    assert pk.get_device_error() == 0  # read-and-clear


def test_bad_context_zero_row_and_error():
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.tiny()
    t = to_device(w)
    t["context_lens"][2] = w.max_blocks_per_seq * w.block_size + 1
    out, _, _ = gpu_step(w, t, check_error=False)
    assert pk.get_device_error() == pk.PKV_ERR_DEVICE_BOUNDS
    assert torch.count_nonzero(out[2]) == 0


def test_bad_slot_and_pair_set_error():
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.tiny()
    t = to_device(w)
    before = t["k_cache"].clone()
    bad = torch.tensor([w.num_blocks * w.block_size + 3], dtype=torch.int64, device="cuda")
    pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"][:1], t["v_new"][:1], bad)
    assert pk.get_device_error() == pk.PKV_ERR_DEVICE_BOUNDS
    pk.copy_blocks(t["k_cache"], t["v_cache"],
                   torch.tensor([[0, w.num_blocks]], dtype=torch.int64, device="cuda"))
    assert pk.get_device_error() == pk.PKV_ERR_DEVICE_BOUNDS
    assert torch.equal(before, t["k_cache"])


def test_launch_count_and_profiler():
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.mha(num_seqs=4, num_blocks=600, heads=4, ctx_range=(600, 2048))
    # the default schedule leaves this CUDA-core launch unplanned: append,
    # decode (split-K merge fused); planned, the schedule kernel comes first
    # and the profiler counts it with the decode as one decode launch
    for mode, kernels in ((1, 2), (2, 3)):
        prev = pk.set_longest_first(mode)
        t = to_device(w)
        pk.profile_reset()
        pk.profile_enable(True)
        n0 = pk.launch_count()
        gpu_step(w, t)
        pk.profile_enable(False)
        pk.set_longest_first(prev)
        assert pk.launch_count() - n0 == kernels, mode
        n, ms = pk.profile_read(pk.KERNEL_DECODE)
        assert n == 1 and ms > 0
        n, _ = pk.profile_read(pk.KERNEL_APPEND)
        assert n == 1
        pk.profile_reset()


def test_bounded_wait_runs_out_without_fault():
    """A device wait that nothing satisfies gives up after its limit and
    reports PKV_ERR_TIMEOUT; the context then keeps working."""
    import time

    from paged_kv_cache_323_b200 import pagedkv as pk

    assert pk.get_device_error() == 0
    t0 = time.perf_counter()
    pk.selftest_bounded_wait(20000)  # 20 ms
    code = pk.get_device_error()
    elapsed = time.perf_counter() - t0
    assert code == pk.PKV_ERR_TIMEOUT
    assert 0.015 <= elapsed < 5.0
    _full_check(wl.tiny())  # the context is still usable


@pytest.mark.parametrize("kind", ["mha", "gqa"])
def test_cuda_graph_capture_and_replay(kind):
    """A whole step (copy-on-write copies, append, decode with a caller
    workspace) captured into a CUDA graph and replayed matches the eager
    step bit for bit: the calls neither synchronise nor allocate."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    if kind == "mha":
        w = wl.mha(num_seqs=8, num_blocks=2048)
    else:
        w = wl.gqa_sampling(groups=4, prompt_median=400, prompt_max=3000)
    t = to_device(w)
    ws = torch.zeros(pk.paged_attention_workspace_size(
        w.num_seqs, w.num_heads, w.max_blocks_per_seq * w.block_size, w.head_dim), dtype=torch.uint8,
        device="cuda")
    k0, v0 = t["k_cache"].clone(), t["v_cache"].clone()

    def step():
        if len(w.cow_pairs):
            pk.copy_blocks(t["k_cache"], t["v_cache"], t["cow_pairs"])
        pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"], t["v_new"], t["slot_mapping"])
        pk.paged_attention_decode_ex(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                     t["context_lens"], w.scale, num_blocks=w.num_blocks,
                                     workspace=ws)

    step()  # eager, also sets kernel attributes outside capture
    torch.cuda.synchronize()
    eager = t["out"].clone()
    t["k_cache"].copy_(k0)
    t["v_cache"].copy_(v0)
    t["out"].zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.synchronize()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert pk.get_device_error() == 0
    assert torch.equal(t["out"], eager)


def test_copy_blocks_more_pairs_than_a_grid_row():
    """70,000 copy-on-write pairs in one call (beyond 65,535, the largest
    grid y extent), bit-exact against the oracle."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    n, nb = 70000, 140010
    g = torch.Generator().manual_seed(17)
    kc = torch.randn(nb, 1, 8, 64, generator=g)
    vc = torch.randn(nb, 1, 8, 64, generator=g)
    perm = np.random.default_rng(17).permutation(nb)
    pairs = np.stack([perm[:n], perm[n:2 * n]], 1).astype(np.int64)
    k_ref, v_ref = kc.numpy().copy(), vc.numpy().copy()
    oracle.copy_blocks(k_ref, v_ref, pairs)
    kd, vd = kc.cuda(), vc.cuda()
    pk.copy_blocks(kd, vd, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    assert pk.get_device_error() == 0
    assert np.array_equal(kd.cpu().numpy(), k_ref) and np.array_equal(vd.cpu().numpy(), v_ref)
