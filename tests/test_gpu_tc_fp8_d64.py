"""The head_dim-64 tensor-core decode kernel over fp8 (e4m3) caches against the
oracle, and against the CUDA-core fp8 kernel on the same inputs.

One CTA serves a pair of kv heads of a sequence ("PagedAttention Explained",
section "How PagedAttention works", item 5: both heads follow the same block
table): 64-byte swizzled tiles of the two heads' rows, one QK^T over both heads
with a block-structured Q, one PV whose 128 rows are the two heads' dims.  The
cases span partial chunks and blocks, several partitions (fused split-K merge),
1, 2 and 4 query heads per kv head, more than one pair per sequence, NaN codes
in unused slots, bad table entries, and an odd kv-head count (which stays on
the CUDA-core kernel).
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_323_b200 import workload as wl
from steps import assert_close, assert_pool_equal, gpu_step, oracle_step, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture
def tc_on():
    from paged_kv_cache_323_b200 import pagedkv as pk

    prev = pk.set_tensor_core_gqa(True)
    yield pk
    pk.set_tensor_core_gqa(prev)


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("kv_heads", [2, 4])
def test_d64_pairs_small(tc_on, bs, G, kv_heads):
    lens = [1, 5, 127, 128, 129, 300, 640]
    w = wl.custom(500 + 10 * G + bs + kv_heads, lens, heads=kv_heads * G, kv_heads=kv_heads, head_dim=64,
                  block_size=bs, dtype="fp8", maxb=-(-640 // bs) + 1)
    ref, kref, vref = oracle_step(w)
    out, kc, vc = gpu_step(w, partition_tokens=256)
    assert_pool_equal(kc, kref, "k pool (codes)")
    assert_pool_equal(vc, vref, "v pool (codes)")
    assert_close(out, ref, "bf16")


@pytest.mark.parametrize("pt", [128, 512, 2048, 0])
def test_d64_partitions(tc_on, pt):
    w = wl.custom(61, [3000, 1, 777, 2048, 4100], heads=16, kv_heads=8, head_dim=64, block_size=16,
                  dtype="fp8")
    ref, _, _ = oracle_step(w)
    out, _, _ = gpu_step(w, partition_tokens=pt)
    assert_close(out, ref, "bf16")


@pytest.mark.parametrize("G", [1, 2])
def test_d64_matches_cuda_core(tc_on, G):
    pk = tc_on
    w = wl.custom(83 + G, [900, 77, 1500, 256], heads=8 * G, kv_heads=8, head_dim=64, block_size=16,
                  dtype="fp8")
    ref, _, _ = oracle_step(w)
    out_tc, _, _ = gpu_step(w)
    pk.set_tensor_core_gqa(False)
    out_cc, _, _ = gpu_step(w)
    pk.set_tensor_core_gqa(True)
    assert_close(out_tc, ref, "bf16", "tensor-core kernel")
    assert_close(out_cc, ref, "bf16", "CUDA-core kernel")
    d = (out_tc.float() - out_cc.float()).abs().max().item()
    assert d <= 2e-2, d


def test_d64_odd_kv_heads_stay_on_cuda_cores(tc_on):
    w = wl.custom(97, [400, 33, 1000], heads=6, kv_heads=3, head_dim=64, block_size=16, dtype="fp8")
    ref, _, _ = oracle_step(w)
    out, _, _ = gpu_step(w, partition_tokens=256)
    assert_close(out, ref, "bf16")


def test_d64_nan_codes_and_bad_entry(tc_on):
    pk = tc_on
    w = wl.custom(79, [200, 333, 50], heads=8, kv_heads=4, head_dim=64, block_size=16, dtype="fp8",
                  num_blocks=60, maxb=24)
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
    w.block_tables[1, 3] = w.num_blocks + 5
    t = to_device(w)
    out, _, _ = gpu_step(w, t, partition_tokens=128, check_error=False)
    assert pk.get_device_error() == pk.PKV_ERR_DEVICE_BOUNDS
    assert torch.isfinite(out.float()).all()


def test_d64_schedule_does_not_change_bits(tc_on):
    pk = tc_on
    w = wl.custom(88, [1, 4000, 700, 129, 2500, 0], heads=8, kv_heads=8, head_dim=64, block_size=16,
                  dtype="fp8")
    outs = []
    prev = pk.set_longest_first(0)
    try:
        for mode in (0, 2, 1):
            pk.set_longest_first(mode)
            out, _, _ = gpu_step(w, partition_tokens=512)
            outs.append(out)
    finally:
        pk.set_longest_first(prev)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
