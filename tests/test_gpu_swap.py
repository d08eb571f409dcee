"""Preemption by swapping on the GPU: swap_blocks between the device pool and
a pinned host pool (bit-exact against the oracle), and a whole preempt /
resume cycle driven by the native block manager, after which the resumed
sequence's attention output is bit-identical to its output before
preemption (its blocks come back to other physical places; the kernels'
arithmetic order depends only on logical positions)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_323_b200 import workload as wl
from steps import assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_swap_out_and_in_bit_exact(dtype):
    from paged_kv_cache_323_b200 import pagedkv as pk

    rng = np.random.default_rng(4)
    tdt = wl.DTYPES[dtype]
    dk = torch.randn(40, 8, 16, 128).to(tdt).cuda()
    dv = torch.randn(40, 8, 16, 128).to(tdt).cuda()
    hk = torch.zeros(12, 8, 16, 128, dtype=tdt).pin_memory()
    hv = torch.zeros(12, 8, 16, 128, dtype=tdt).pin_memory()
    out_pairs = np.stack([rng.choice(40, 9, replace=False), rng.choice(12, 9, replace=False)], 1)
    ref_hk, ref_hv = wl.to_numpy_bits(hk).copy(), wl.to_numpy_bits(hv).copy()
    oracle.swap_blocks(ref_hk, ref_hv, wl.to_numpy_bits(dk), wl.to_numpy_bits(dv), out_pairs)
    pk.swap_blocks(hk, hv, dk, dv, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    assert pk.get_device_error() == 0
    assert np.array_equal(wl.to_numpy_bits(hk).view(np.uint8), ref_hk.view(np.uint8))
    assert np.array_equal(wl.to_numpy_bits(hv).view(np.uint8), ref_hv.view(np.uint8))
    # back in, to other device blocks, with the pairs themselves in pinned host memory
    in_pairs = np.stack([out_pairs[:, 1], rng.choice(40, 9, replace=False)], 1)
    ref_dk, ref_dv = wl.to_numpy_bits(dk).copy(), wl.to_numpy_bits(dv).copy()
    oracle.swap_blocks(ref_dk, ref_dv, ref_hk, ref_hv, in_pairs)
    pk.swap_blocks(dk, dv, hk, hv, torch.from_numpy(in_pairs).pin_memory())
    torch.cuda.synchronize()
    assert np.array_equal(wl.to_numpy_bits(dk).view(np.uint8), ref_dk.view(np.uint8))
    assert np.array_equal(wl.to_numpy_bits(dv).view(np.uint8), ref_dv.view(np.uint8))


def test_swap_rejects_pageable_and_bad_pairs():
    from paged_kv_cache_323_b200 import pagedkv as pk

    dk = torch.zeros(4, 2, 8, 64, dtype=torch.bfloat16, device="cuda")
    pageable = torch.zeros(4, 2, 8, 64, dtype=torch.bfloat16)
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    rc = pk.lib.swap_blocks(pageable.data_ptr(), pageable.data_ptr(), dk.data_ptr(), dk.data_ptr(),
                            pairs.data_ptr(), 1, 2, 64, 8, 4, 4, pk.PKV_BF16, None)
    assert rc == pk.PKV_ERR_INVALID
    bad = torch.tensor([[0, 9]], dtype=torch.int64, device="cuda")
    pk.swap_blocks(dk, dk, dk.clone(), dk.clone(), bad)
    assert pk.get_device_error() == pk.PKV_ERR_DEVICE_BOUNDS


def test_preempt_and_resume_with_block_manager():
    from paged_kv_cache_323_b200 import pagedkv as pk

    H, Hkv, D, bs, nblk = 16, 4, 128, 16, 64
    bm = pk.BlockManager(nblk, bs, num_host_blocks=32,
                         free_order=np.random.default_rng(8).permutation(nblk))
    kc = torch.zeros(nblk, Hkv, bs, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    hk = torch.zeros(32, Hkv, bs, D, dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    g = torch.Generator(device="cuda").manual_seed(11)

    def write(seq, n):
        slots, pairs = bm.append(seq, n)
        if len(pairs):
            pk.copy_blocks(kc, vc, torch.from_numpy(pairs).cuda())
        k = torch.randn(n, Hkv, D, generator=g, device="cuda").to(torch.bfloat16)
        v = torch.randn(n, Hkv, D, generator=g, device="cuda").to(torch.bfloat16)
        pk.kv_cache_append(kc, vc, k, v, torch.from_numpy(slots).cuda())

    def decode(seqs, q):
        bt, lens = bm.tables(seqs, 32)
        out = torch.empty_like(q)
        pk.paged_attention_decode_ex(out, q, kc, vc, torch.from_numpy(bt).cuda(),
                                     torch.from_numpy(lens).cuda(), D ** -0.5, num_blocks=nblk)
        return out

    a, b, c = bm.add_sequence(), bm.add_sequence(), bm.add_sequence()
    write(a, 300)
    write(b, 150)
    write(c, 200)
    q = torch.randn(1, H, D, generator=g, device="cuda").to(torch.bfloat16)
    before = decode([c], q)
    # the pool runs short: swap out the most recently arrived sequence
    victim = bm.pick_victim()
    assert victim == c
    pk.swap_blocks(hk, hv, kc, vc, torch.from_numpy(bm.swap_out(victim)).cuda())
    write(a, 250)  # reuses the freed device blocks
    write(b, 100)
    assert bm.stats()["swapped_sequences"] == 1
    # a finishes; c comes back into whatever blocks are free now
    bm.free(a)
    pk.swap_blocks(kc, vc, hk, hv, torch.from_numpy(bm.swap_in(victim)).cuda())
    after = decode([c], q)
    torch.cuda.synchronize()
    assert pk.get_device_error() == 0
    assert torch.equal(before, after)
    st = bm.stats()
    assert st["preemptions"] == 1 and st["live_sequences"] == 2


def test_block_manager_step_matches_oracle():
    """A decode step assembled by the block manager (forked samples, copy on
    write, multi-token append) against the oracle on the same pool."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    H, Hkv, D, bs, nblk = 16, 2, 128, 16, 96
    bm = pk.BlockManager(nblk, bs, free_order=np.random.default_rng(2).permutation(nblk))
    gen = torch.Generator().manual_seed(5)
    kc = torch.randn(nblk, Hkv, bs, D, generator=gen).to(torch.bfloat16)
    vc = torch.randn(nblk, Hkv, bs, D, generator=gen).to(torch.bfloat16)
    p = bm.add_sequence()
    slots0, _ = bm.append(p, 203)
    samples = [p] + [bm.fork(p) for _ in range(3)]
    all_pairs, all_slots, counts = [], [], []
    for s in samples:
        n = 1 + 7 * s % 20
        slots, pairs = bm.append(s, n)
        all_pairs += [list(x) for x in pairs]
        all_slots += slots.tolist()
        counts.append(n)
    T = len(all_slots)
    k_new = torch.randn(T, Hkv, D, generator=gen).to(torch.bfloat16)
    v_new = torch.randn(T, Hkv, D, generator=gen).to(torch.bfloat16)
    bt, lens = bm.tables(samples, 16)
    q = torch.randn(len(samples), H, D, generator=gen).to(torch.bfloat16)
    pairs = np.asarray(all_pairs, dtype=np.int64).reshape(-1, 2)
    slots = np.asarray(all_slots, dtype=np.int64)
    # oracle
    k_ref, v_ref = wl.to_numpy_bits(kc).copy(), wl.to_numpy_bits(vc).copy()
    oracle.copy_blocks(k_ref, v_ref, pairs)
    oracle.kv_append(k_ref, v_ref, wl.to_numpy_bits(k_new), wl.to_numpy_bits(v_new), slots)
    ref = oracle.paged_attention(wl.to_numpy_bits(q), k_ref, v_ref, bt, lens, D ** -0.5)
    # device
    kd, vd = kc.cuda(), vc.cuda()
    pk.copy_blocks(kd, vd, torch.from_numpy(pairs).cuda())
    pk.kv_cache_append(kd, vd, k_new.cuda(), v_new.cuda(), torch.from_numpy(slots).cuda())
    out = torch.empty_like(q).cuda()
    pk.paged_attention_decode_ex(out, q.cuda(), kd, vd, torch.from_numpy(bt).cuda(),
                                 torch.from_numpy(lens).cuda(), D ** -0.5, num_blocks=nblk)
    torch.cuda.synchronize()
    assert np.array_equal(wl.to_numpy_bits(kd).view(np.uint8), k_ref.view(np.uint8))
    assert_close(out, ref, "bf16")
