"""The tensor-core decode kernel over fp8 (e4m3) caches against the oracle, and
against the CUDA-core fp8 kernel on the same inputs.

It serves head_dim 128, groups of 1/2/4/8 query heads and partitions that
are multiples of 128 tokens: both products on e4m3 tensor cores over the
codes as they land, q and the probabilities each split into two e4m3 terms.
The cases span partial 128-token chunks, partial blocks, several partitions
(fused split-K merge), long partitions that wrap the ring of slots, NaN codes
in unused slots, bad table entries, and block permutations.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_323_b200 import workload as wl
from steps import assert_close, assert_pool_equal, full_size_check, gpu_step, oracle_step, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[False, True], ids=["per_unit", "persistent"])
def tc_mode(request):
    """The tensor-core fp8 kernel in both forms: one CTA per unit, and the
    persistent one (used wherever a workspace is given and partitions are at
    most 2048 tokens)."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    prev = pk.set_tensor_core_gqa(True)
    prev_p = pk._set_fp8_persistent(request.param)
    yield pk
    pk._set_fp8_persistent(prev_p)
    pk.set_tensor_core_gqa(prev)


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_tc_fp8_small(tc_mode, bs, G):
    lens = [1, 5, 127, 128, 129, 300, 640]
    w = wl.custom(400 + G + bs, lens, heads=2 * G, kv_heads=2, head_dim=128, block_size=bs,
                  dtype="fp8", maxb=-(-640 // bs) + 1)
    ref, kref, vref = oracle_step(w)
    out, kc, vc = gpu_step(w, partition_tokens=256)
    assert_pool_equal(kc, kref, "k pool (codes)")
    assert_pool_equal(vc, vref, "v pool (codes)")
    assert_close(out, ref, "bf16")


@pytest.mark.parametrize("pt", [128, 512, 2048, 0])
def test_tc_fp8_partitions(tc_mode, pt):
    w = wl.gqa_sampling(groups=4, prompt_median=600, prompt_max=3000, dtype="fp8")
    ref, _, _ = oracle_step(w)
    out, _, _ = gpu_step(w, partition_tokens=pt)
    assert_close(out, ref, "bf16")


@pytest.mark.parametrize("G", [1, 4])
def test_tc_fp8_matches_cuda_core(tc_mode, G):
    pk = tc_mode
    w = wl.custom(33 + G, [900, 77, 1500, 256], heads=8 * G, kv_heads=8, head_dim=128,
                  block_size=16, dtype="fp8")
    ref, _, _ = oracle_step(w)
    out_tc, _, _ = gpu_step(w)
    pk.set_tensor_core_gqa(False)
    out_cc, _, _ = gpu_step(w)
    pk.set_tensor_core_gqa(True)
    assert_close(out_tc, ref, "bf16", "tensor-core kernel")
    assert_close(out_cc, ref, "bf16", "CUDA-core kernel")
    d = (out_tc.float() - out_cc.float()).abs().max().item()
    assert d <= 2e-2, d


def test_tc_fp8_nan_codes_and_bad_entry(tc_mode):
    pk = tc_mode
    w = wl.custom(78, [200, 333, 50], heads=16, kv_heads=2, head_dim=128, block_size=16,
                  dtype="fp8", num_blocks=60, maxb=24)
    bs = w.block_size
    used = np.zeros((w.num_blocks, bs), dtype=bool)
    for s in range(w.num_seqs):
        for t in range(int(w.context_lens[s])):
            used[w.block_tables[s][t // bs], t % bs] = True
    mask = torch.from_numpy(~used)[:, None, :, None].expand(w.k_cache.shape)
    w.k_cache = w.k_cache.view(torch.uint8).masked_fill(mask, 0x7F).view(torch.float8_e4m3fn)
    w.v_cache = w.v_cache.view(torch.uint8).masked_fill(mask, 0xFF).view(torch.float8_e4m3fn)
    ref, _, _ = oracle_step(w)
    out, _, _ = gpu_step(w, partition_tokens=128)
    assert_close(out, ref, "bf16")
    # a table entry outside the pool: error word set, output finite
    w.block_tables[1, 3] = w.num_blocks + 5
    t = to_device(w)
    out, _, _ = gpu_step(w, t, partition_tokens=128, check_error=False)
    assert pk.get_device_error() == pk.PKV_ERR_DEVICE_BOUNDS
    assert torch.isfinite(out.float()).all()


def test_tc_fp8_permutation_bit_identical(tc_mode):
    w = wl.custom(92, [700, 1000, 257], heads=32, kv_heads=8, head_dim=128, block_size=16,
                  dtype="fp8")
    out1, _, _ = gpu_step(w)
    perm = np.random.default_rng(4).permutation(w.num_blocks)
    w2 = wl.Workload(**{**w.__dict__})
    p = torch.from_numpy(perm)
    w2.k_cache = torch.empty_like(w.k_cache.view(torch.uint8))
    w2.v_cache = torch.empty_like(w.v_cache.view(torch.uint8))
    w2.k_cache[p] = w.k_cache.view(torch.uint8)
    w2.v_cache[p] = w.v_cache.view(torch.uint8)
    w2.k_cache = w2.k_cache.view(torch.float8_e4m3fn)
    w2.v_cache = w2.v_cache.view(torch.float8_e4m3fn)
    w2.block_tables = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    bs = w.block_size
    w2.slot_mapping = np.asarray([perm[s // bs] * bs + s % bs for s in w.slot_mapping], dtype=np.int64)
    out2, _, _ = gpu_step(w2)
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("make", [
    lambda: wl.gqa_sampling(device="cuda", dtype="fp8"),
    lambda: wl.long_context(device="cuda", dtype="fp8"),
], ids=["gqa_sampling", "long_context"])
def test_tc_fp8_full_size(tc_mode, make):
    """Every row of the full-size fp8 workloads (256 x 32, 8 x 64)."""
    full_size_check(make())


@pytest.mark.parametrize("pt", [0, 1024])
def test_tc_fp8_group8_bs32_long_partitions(tc_mode, pt):
    """Eight query heads per kv head, 32-token blocks, partitions of many
    128-token chunks (the ring of slots wraps several times) and several
    partitions per sequence, at a size the oracle checks in full."""
    w = wl.custom(57, [9000, 4097, 300, 12345], heads=64, kv_heads=8, head_dim=128,
                  block_size=32, dtype="fp8")
    ref, kref, vref = oracle_step(w)
    out, kc, vc = gpu_step(w, partition_tokens=pt)
    assert_pool_equal(kc, kref, "k pool (codes)")
    assert_close(out, ref, "bf16")



@pytest.mark.parametrize("G,bs,pt,lens", [
    (4, 16, 128, None), (4, 16, 1024, None), (4, 16, 2048, None), (4, 8, 1024, None), (4, 32, 4096, None),
    (1, 16, 256, None), (2, 16, 512, None),
    # every sequence in one partition: the first wave takes units in index order, the queue the rest
    (1, 16, 2048, [1, 130, 700, 2048, 1500, 0, 2000, 129] * 40),
    (4, 16, 2048, [1, 130, 700, 2048, 1500, 0, 2000, 129] * 3),
])
def test_tc_fp8_persistent_same_bits(G, bs, pt, lens):
    """The persistent form computes every unit with the same arithmetic in
    the same order as the one-CTA-per-unit kernel -- the split-K merge's
    partition order included, which does not depend on how many threads run
    it -- so the outputs are identical bit for bit under every schedule,
    launch after launch on one workspace (the queue is back at zero after
    each launch)."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    if lens is None:
        w = wl.custom(71, [1, 130, 700, 2049, 4500, 0, 3000, 129], heads=4 * G, kv_heads=4, head_dim=128,
                      block_size=bs, dtype="fp8")
    else:
        w = wl.custom(71, lens, heads=4 * G, kv_heads=4, head_dim=128, block_size=bs, dtype="fp8",
                      maxb=pt // bs)
    ref, _, _ = oracle_step(w)
    t = to_device(w)
    ks = torch.from_numpy(w.k_scales).cuda()
    vs = torch.from_numpy(w.v_scales).cuda()
    pk.kv_cache_append_fp8(t["k_cache"], t["v_cache"], ks, vs, t["k_new"], t["v_new"], t["slot_mapping"])
    need = pk.paged_attention_workspace_size(w.num_seqs, w.num_heads,
                                             w.max_blocks_per_seq * w.block_size, w.head_dim, pt)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = []
    prev = pk._set_fp8_persistent(False)
    prev_sched = pk.set_longest_first(1)
    try:
        for persistent, sched in ((False, 1), (True, 0), (True, 1), (True, 2), (True, 1), (False, 2),
                                  (False, 0), (True, 0)):
            pk._set_fp8_persistent(persistent)
            pk.set_longest_first(sched)
            t["out"].fill_(float("nan"))
            pk.paged_attention_decode_fp8(t["out"], t["q"], t["k_cache"], t["v_cache"], ks, vs,
                                          t["block_tables"], t["context_lens"], w.scale,
                                          num_blocks=w.num_blocks, partition_tokens=pt, workspace=ws)
            torch.cuda.synchronize()
            assert pk.get_device_error() == 0
            outs.append(t["out"].clone())
    finally:
        pk._set_fp8_persistent(prev)
        pk.set_longest_first(prev_sched)
    assert_close(outs[0], ref, "bf16")
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    assert int(ws[:8].view(torch.int32).abs().sum()) == 0  # queue counters back at zero


def test_tc_fp8_bad_context_zero_rows(tc_mode):
    """A context length past the table: that sequence's rows are zero and
    the error word says so; every other row still matches the oracle (in
    the persistent form the producer settles such units from the queue)."""
    pk = tc_mode
    w = wl.custom(91, [300, 700, 129, 1000, 64], heads=8, kv_heads=4, head_dim=128, block_size=16,
                  dtype="fp8")
    ref, _, _ = oracle_step(w)
    t = to_device(w)
    t["context_lens"][2] = w.max_blocks_per_seq * w.block_size + 1
    out, _, _ = gpu_step(w, t, partition_tokens=256, check_error=False)
    assert pk.get_device_error() == pk.PKV_ERR_DEVICE_BOUNDS
    assert torch.count_nonzero(out[2]) == 0
    keep = [0, 1, 3, 4]
    assert_close(out[keep], ref[keep], "bf16")


def test_tc_fp8_many_units_twice(tc_mode):
    """More (sequence, kv head) units than the workspace's fixed counter
    region holds (65536), split into partitions, twice on one workspace:
    the counters past the region are cleared per call and both calls match
    the oracle."""
    pk = tc_mode
    rng = np.random.default_rng(5)
    # mostly short sequences (the pool stays near 1 GB), a fifth long enough to split
    lens = np.where(rng.random(2100) < 0.8, rng.integers(1, 65, size=2100),
                    rng.integers(129, 300, size=2100)).tolist()
    w = wl.custom(93, lens, heads=32, kv_heads=32, head_dim=128, block_size=16, dtype="fp8")
    assert w.num_seqs * w.num_kv_heads > 65536
    ref, _, _ = oracle_step(w)
    t = to_device(w)
    ks = torch.from_numpy(w.k_scales).cuda()
    vs = torch.from_numpy(w.v_scales).cuda()
    pk.kv_cache_append_fp8(t["k_cache"], t["v_cache"], ks, vs, t["k_new"], t["v_new"], t["slot_mapping"])
    pt = 128
    need = pk.paged_attention_workspace_size(w.num_seqs, w.num_heads, w.max_blocks_per_seq * w.block_size,
                                             w.head_dim, pt)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        t["out"].fill_(float("nan"))
        pk.paged_attention_decode_fp8(t["out"], t["q"], t["k_cache"], t["v_cache"], ks, vs,
                                      t["block_tables"], t["context_lens"], w.scale,
                                      num_blocks=w.num_blocks, partition_tokens=pt, workspace=ws)
        torch.cuda.synchronize()
        assert pk.get_device_error() == 0
        assert_close(t["out"], ref, "bf16")
