"""Host-side checks of the seeded workload generators (no GPU)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_323_b200 import workload as wl


def _check_tables(w: wl.Workload, shared_ok=frozenset()):
    bs = w.block_size
    owners = {}
    for s in range(w.num_seqs):
        L = int(w.context_lens[s])
        nb = oracle.blocks_needed(L, bs)
        row = w.block_tables[s]
        assert np.all(row[:nb] >= 0) and np.all(row[:nb] < w.num_blocks)
        assert np.all(row[nb:] == -1)
        for p in row[:nb]:
            owners.setdefault(int(p), set()).add(s)
    for p, who in owners.items():
        if len(who) > 1:
            assert p in shared_ok, f"block {p} shared by {sorted(who)} unexpectedly"
    return owners


def _check_slots(w: wl.Workload, positions):
    """slot_mapping[i] lands in the block the table names for that position."""
    bs = w.block_size
    i = 0
    for s, pos in enumerate(positions):
        for t in pos:
            slot = int(w.slot_mapping[i])
            assert slot // bs == w.block_tables[s][t // bs]
            assert slot % bs == t % bs
            i += 1
    assert i == len(w.slot_mapping)


def test_tiny_matches_spec():
    w = wl.tiny()
    assert w.context_lens.tolist() == [35, 16, 1, 50]
    assert (w.num_heads, w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks) == (4, 4, 64, 16, 32)
    assert w.q.dtype == torch.float32 and w.scale == 0.125
    _check_tables(w)
    _check_slots(w, [[L - 1] for L in w.context_lens.tolist()])
    # seeded: the same seed gives the same draw
    w2 = wl.tiny()
    assert torch.equal(w.k_cache, w2.k_cache) and np.array_equal(w.block_tables, w2.block_tables)


def test_mha_small_variant():
    w = wl.mha(num_seqs=6, num_blocks=1024)
    assert np.all((w.context_lens >= 128) & (w.context_lens <= 2048))
    assert w.max_blocks_per_seq == 128
    assert w.k_cache.dtype == torch.bfloat16
    _check_tables(w)
    _check_slots(w, [[L - 1] for L in w.context_lens.tolist()])


def test_gqa_sampling_cow_structure():
    w = wl.gqa_sampling(groups=6, prompt_median=60, prompt_max=200)
    samples = w.meta["samples"]
    prompts = w.meta["prompts"]
    bs = w.block_size
    shared = set()
    for gi, P in enumerate(prompts):
        nb = -(-P // bs)
        first = w.block_tables[gi * samples][:nb]
        for i in range(samples):
            row = w.block_tables[gi * samples + i]
            full = P // bs
            assert np.array_equal(row[:full], first[:full])  # full prompt blocks shared
            shared.update(int(x) for x in row[:full])
        if P % bs:
            partial = [int(w.block_tables[gi * samples + i][nb - 1]) for i in range(samples)]
            assert len(set(partial)) == samples  # every writer ends with its own copy of the partial block
            shared.update(partial)
    _check_tables(w, shared_ok=frozenset(shared))
    pairs = w.cow_pairs
    n_partial = sum(1 for P in prompts if P % bs)
    assert pairs.shape == (n_partial * (samples - 1), 2)
    assert len(set(pairs[:, 1].tolist())) == len(pairs)  # distinct destinations
    assert not set(pairs[:, 1].tolist()) & set(pairs[:, 0].tolist())
    gens = w.meta["gens"]
    positions = []
    for gi, P in enumerate(prompts):
        for i in range(samples):
            positions.append(list(range(P, P + gens[gi][i])))
    _check_slots(w, positions)


def test_prefix_sweep_shares_prefix():
    for bs in (8, 16, 32):
        w = wl.prefix_sweep(bs, num_seqs=5)
        pref = w.meta["prefix_blocks"]
        for s in range(5):
            assert w.block_tables[s][: len(pref)].tolist() == pref
        _check_tables(w, shared_ok=frozenset(pref))
        # padded-slot waste: at most bs-1 per sequence, the prefix counted once
        alloc, unused = oracle.waste_physical(w.block_tables, w.context_lens, bs, w.num_blocks)
        assert 0 <= unused <= 5 * (bs - 1)


def test_long_context_small_variant():
    w = wl.long_context(num_seqs=2, ctx_range=(600, 1500))
    assert w.group == 8 and w.block_size == 32
    # q is scaled by 0.5 before rounding to bf16
    assert float(w.q.float().abs().max()) < 0.5 * 6
    _check_tables(w)


def test_custom_edge_lengths():
    w = wl.custom(9, [0, 1, 16, 17], heads=4, kv_heads=2, head_dim=64, block_size=16, dtype="bf16")
    assert w.block_tables.shape == (4, 2)
    assert len(w.slot_mapping) == 3  # nothing is appended for the empty sequence
    _check_tables(w)


def test_bits_roundtrip():
    t = torch.randn(3, 5).to(torch.bfloat16)
    assert torch.equal(wl.from_numpy_bits(wl.to_numpy_bits(t), "bf16"), t)


def test_contiguous_placement():
    """The contiguous comparator lays each sequence's blocks out consecutively."""
    w = wl.mha(num_seqs=5, num_blocks=700, contiguous=True)
    nxt = 0
    for s in range(5):
        nb = oracle.blocks_needed(int(w.context_lens[s]), w.block_size)
        assert w.block_tables[s][:nb].tolist() == list(range(nxt, nxt + nb))
        nxt += nb
    _check_tables(w)


def test_kv_bytes_unique_counts_shared_blocks_once():
    from paged_kv_cache_323_b200 import workload as wl

    w = wl.tiny()
    assert w.kv_bytes_unique() == w.kv_bytes_logical()  # no sharing
    # two sequences over one shared full block (16 slots) plus private tails of
    # 5 and 9 slots; the shared block counts 16 slots once
    w.block_tables = np.array([[3, 7, -1, -1], [3, 9, -1, -1], [0, -1, -1, -1], [1, 2, 4, 5]],
                              dtype=np.int32)
    w.context_lens = np.array([21, 25, 0, 50], dtype=np.int32)
    per_slot = w.num_kv_heads * w.head_dim * 2 * w.elt
    assert w.kv_bytes_unique() == (16 + 5 + 9 + 50) * per_slot
    assert w.kv_bytes_logical() == (21 + 25 + 50) * per_slot


@pytest.mark.parametrize("make", [lambda: wl.tiny(), lambda: wl.gqa_sampling(groups=8, prompt_max=3000),
                                  lambda: wl.prefix_sweep(8, num_seqs=32, prefix=512)],
                         ids=["tiny", "gqa_sampling", "prefix_bs8"])
def test_padded_slot_waste_matches_oracle(make):
    """The bench's waste figures equal the oracle's waste accounting."""
    w = make()
    got = w.padded_slot_waste()
    alloc, unused = oracle.waste_per_sequence(w.context_lens, w.block_size)
    assert (got["per_sequence_allocated"], got["per_sequence_unused"]) == (alloc, unused)
    palloc, punused = oracle.waste_physical(w.block_tables, w.context_lens, w.block_size, w.num_blocks)
    assert (got["physical_allocated"], got["physical_unused"]) == (palloc, punused)
