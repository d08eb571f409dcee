"""The register-streamed decode kernel (bf16 MHA over 8-token blocks, head_dim
128) against the oracle, and the staged kernel it replaces on the same
inputs ("How PagedAttention works", items 2-5: the kernel walks the block
table and gathers each block's keys and values wherever they sit).

Both forms meet the bf16 bar on every case; the register form is the
default for this shape and is selected explicitly here so each case runs
both ways.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_323_b200 import workload as wl
from steps import assert_close, assert_pool_equal, full_size_check, gpu_step, oracle_step

pytestmark = pytest.mark.gpu

FORMS = {"register": True, "staged": False}


@pytest.fixture(params=sorted(FORMS))
def form(request):
    from paged_kv_cache_323_b200 import pagedkv as pk

    prev = pk._set_reg_stream(FORMS[request.param])
    assert prev is True  # the register form is the default
    yield request.param
    pk._set_reg_stream(prev)


@pytest.mark.parametrize("pt", [0, 8, 24, 64, 256, 4096])
def test_edge_lengths(form, pt):
    """Empty (zero row), one token, one short of / exactly / one past a
    block, ragged tails, the table's maximum context; partitions from one
    block (8 tokens) to the 4096-token maximum."""
    maxb = 160
    lens = [0, 1, 7, 8, 9, 15, 16, 17, 100, 1000, maxb * 8, 5, 1279, 63]
    w = wl.custom(21, lens, heads=4, kv_heads=4, head_dim=128, block_size=8, dtype="bf16", maxb=maxb)
    ref, kref, vref = oracle_step(w)
    out, kc, vc = gpu_step(w, partition_tokens=pt)
    assert_pool_equal(kc, kref, "k pool")
    assert_pool_equal(vc, vref, "v pool")
    assert_close(out, ref, "bf16")
    assert torch.count_nonzero(out[0]) == 0


def test_reduced_batch(form):
    """A batch-64-like MHA batch cut to 8 sequences, several partitions."""
    w = wl.mha(num_seqs=8, num_blocks=4096, heads=8, block_size=8)
    ref, _, _ = oracle_step(w)
    for pt in (0, 128, 512):
        out, _, _ = gpu_step(w, partition_tokens=pt)
        assert_close(out, ref, "bf16", what=f"partition {pt}")


def test_nan_poisoned_unused_slots(form):
    """Unused slots and blocks past each context hold NaN: outputs stay
    finite and match the oracle, so nothing outside the context is read
    into the result."""
    w = wl.mha(num_seqs=6, num_blocks=1800, heads=4, block_size=8, ctx_range=(1, 700))
    bs = w.block_size
    used = np.zeros((w.num_blocks, bs), dtype=bool)
    for s in range(w.num_seqs):
        for t in range(int(w.context_lens[s])):
            used[w.block_tables[s][t // bs], t % bs] = True
    mask = torch.from_numpy(~used)[:, None, :, None].expand_as(w.k_cache)
    w.k_cache = w.k_cache.masked_fill(mask, float("nan"))
    w.v_cache = w.v_cache.masked_fill(mask, float("nan"))
    poison_blk = int(np.argmax((~used).all(axis=1)))
    for s in range(w.num_seqs):
        nb = -(-int(w.context_lens[s]) // bs)
        w.block_tables[s, nb:] = poison_blk
    ref, _, _ = oracle_step(w)
    for pt in (0, 64):
        out, _, _ = gpu_step(w, partition_tokens=pt)
        assert_close(out, ref, "bf16", what=f"partition {pt}")


def test_permutation_bit_identical(form):
    """Moving blocks (data and table together) leaves the output
    bit-identical: the reduction order is logical."""
    w = wl.mha(num_seqs=6, num_blocks=1200, heads=8, block_size=8)
    out1, _, _ = gpu_step(w, partition_tokens=256)
    perm = np.random.default_rng(9).permutation(w.num_blocks)
    w2 = wl.Workload(**{**w.__dict__})
    w2.k_cache = torch.empty_like(w.k_cache)
    w2.v_cache = torch.empty_like(w.v_cache)
    w2.k_cache[torch.from_numpy(perm)] = w.k_cache
    w2.v_cache[torch.from_numpy(perm)] = w.v_cache
    w2.block_tables = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    bs = w.block_size
    w2.slot_mapping = np.asarray([perm[s // bs] * bs + s % bs for s in w.slot_mapping], dtype=np.int64)
    out2, _, _ = gpu_step(w2, partition_tokens=256)
    assert torch.equal(out1, out2)


def test_schedule_does_not_change_bits(form):
    """Longest-first and index order give the same bits."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.mha(num_seqs=16, num_blocks=6000, heads=8, block_size=8)
    outs = []
    for mode in (2, 0):
        prev = pk.set_longest_first(mode)
        try:
            out, _, _ = gpu_step(w, partition_tokens=256)
        finally:
            pk.set_longest_first(prev)
        outs.append(out.clone())
    assert torch.equal(outs[0], outs[1])


def test_bad_table_entry_sets_error(form):
    """An entry past the pool sets the error word; its block is skipped and
    the outputs stay finite."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.mha(num_seqs=3, num_blocks=800, heads=4, block_size=8)
    w.block_tables[1, 2] = w.num_blocks + 7
    out, _, _ = gpu_step(w, check_error=False)
    assert pk.get_device_error() == pk.PKV_ERR_DEVICE_BOUNDS
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("contiguous", [False, True], ids=["paged", "contiguous"])
def test_full_size(form, contiguous):
    """Batch-64 MHA at block size 8 (32 = 32 heads, contexts U[128, 2048],
    pool of 32768 blocks): all 64 x 32 rows, paged and contiguous
    placement."""
    full_size_check(wl.mha(block_size=8, contiguous=contiguous, device="cuda"))
