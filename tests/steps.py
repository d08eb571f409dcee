"""One decode step on a workload, through the CUDA library and through the
oracle, plus the comparison rules of the parity tests.

A step is: copy-on-write block copies, then the append of the step's new
tokens, then one decode query per sequence.  The GPU side calls only the
C-ABI binding; the oracle side calls only ``oracle/``.  They share the
workload's inputs and nothing else.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_323_b200 import workload as wl

# Tolerances: fp32 caches, max abs error 1e-5; bf16 caches with fp32
# accumulation, |gpu - ref| <= 2e-2 + 1e-2 |ref| elementwise (allclose form).
F32_ATOL = 1e-5
BF16_ATOL = 2e-2
BF16_RTOL = 1e-2


def to_device(w: wl.Workload, device="cuda") -> dict:
    t = {
        "q": w.q.to(device),
        "k_cache": w.k_cache.to(device),
        "v_cache": w.v_cache.to(device),
        "k_new": w.k_new.to(device),
        "v_new": w.v_new.to(device),
        "block_tables": torch.from_numpy(w.block_tables).to(device),
        "context_lens": torch.from_numpy(w.context_lens).to(device),
        "slot_mapping": torch.from_numpy(w.slot_mapping).to(device),
        "cow_pairs": torch.from_numpy(w.cow_pairs).to(device),
    }
    t["out"] = torch.empty_like(t["q"])
    return t


def gpu_step(w: wl.Workload, t: dict | None = None, partition_tokens: int = 0,
             check_error: bool = True):
    """Run the step in place on device tensors ``t``; returns (out, k_cache, v_cache)."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    if t is None:
        t = to_device(w)
    if len(w.cow_pairs):
        pk.copy_blocks(t["k_cache"], t["v_cache"], t["cow_pairs"])
    if w.dtype == "fp8":
        ks = torch.from_numpy(w.k_scales).to(t["q"].device)
        vs = torch.from_numpy(w.v_scales).to(t["q"].device)
        pk.kv_cache_append_fp8(t["k_cache"], t["v_cache"], ks, vs, t["k_new"], t["v_new"],
                               t["slot_mapping"])
        pk.paged_attention_decode_fp8(t["out"], t["q"], t["k_cache"], t["v_cache"], ks, vs,
                                      t["block_tables"], t["context_lens"], w.scale,
                                      num_blocks=w.num_blocks, partition_tokens=partition_tokens)
    else:
        pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"], t["v_new"], t["slot_mapping"])
        pk.paged_attention_decode_ex(t["out"], t["q"], t["k_cache"], t["v_cache"],
                                     t["block_tables"], t["context_lens"], w.scale,
                                     num_blocks=w.num_blocks, partition_tokens=partition_tokens)
    torch.cuda.synchronize()
    if check_error:
        code = pk.get_device_error()
        assert code == 0, f"device error word {code}"
    return t["out"], t["k_cache"], t["v_cache"]


def _fp8_attention(q, kc, vc, w: wl.Workload) -> np.ndarray:
    """The oracle's fp8 attention over the batch, run as one call per slice of
    sequences on a pool of host threads (each call is independent and the
    ctypes call releases the GIL; the arithmetic is the oracle's own)."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    B = q.shape[0]
    nthreads = max(1, min(B, os.cpu_count() or 1))
    bounds = np.linspace(0, B, nthreads + 1).astype(int)

    def part(i):
        a, b = bounds[i], bounds[i + 1]
        if a == b:
            return np.zeros((0,) + q.shape[1:], dtype=np.float64)
        return oracle.paged_attention_fp8(q[a:b], kc, vc, w.k_scales, w.v_scales,
                                          w.block_tables[a:b], w.context_lens[a:b], w.scale)

    with ThreadPoolExecutor(nthreads) as ex:
        return np.concatenate(list(ex.map(part, range(nthreads))), axis=0)


def oracle_step(w: wl.Workload):
    """The same step on host copies; returns (out fp64, k pool, v pool) as numpy."""
    kc = wl.to_numpy_bits(w.k_cache).copy()
    vc = wl.to_numpy_bits(w.v_cache).copy()
    if len(w.cow_pairs):
        oracle.copy_blocks(kc, vc, w.cow_pairs)
    if w.dtype == "fp8":
        oracle.kv_append_fp8(kc, vc, w.k_scales, w.v_scales, wl.to_numpy_bits(w.k_new),
                             wl.to_numpy_bits(w.v_new), w.slot_mapping)
        out = _fp8_attention(wl.to_numpy_bits(w.q), kc, vc, w)
        return out, kc, vc
    oracle.kv_append(kc, vc, wl.to_numpy_bits(w.k_new), wl.to_numpy_bits(w.v_new), w.slot_mapping)
    out = oracle.paged_attention(wl.to_numpy_bits(w.q), kc, vc, w.block_tables, w.context_lens,
                                 w.scale)
    return out, kc, vc


def assert_close(gpu: torch.Tensor, ref: np.ndarray, dtype: str, what: str = "out"):
    g = gpu.detach().float().cpu().double().numpy().reshape(ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err = np.abs(g - ref)
    if dtype == "f32":
        assert err.max() <= F32_ATOL, f"{what}: max abs err {err.max():.3e} > {F32_ATOL}"
    else:
        bound = BF16_ATOL + BF16_RTOL * np.abs(ref)
        bad = err > bound
        assert not bad.any(), (f"{what}: {int(bad.sum())} elements outside 2e-2 + 1e-2|ref|; "
                               f"max abs err {err.max():.3e}")
    return float(err.max())


def assert_pool_equal(gpu: torch.Tensor, ref: np.ndarray, what: str):
    g = wl.to_numpy_bits(gpu)
    assert g.shape == ref.shape
    same = g.view(np.uint8) == ref.view(np.uint8)
    assert same.all(), f"{what}: {int((~same).sum())} bytes differ"


def subset(w: wl.Workload, seqs, pool_device_k=None, pool_device_v=None) -> wl.Workload:
    """The step restricted to the sequences ``seqs``, on a compact pool that
    holds only the blocks they reference (and copy-on-write sources), taken
    from the workload's pre-step pool (``meta["blocks"]`` lists them in pool
    order).  Used to check full-size workloads against the oracle."""
    seqs = [int(s) for s in seqs]
    pos = {s: i for i, s in enumerate(seqs)}
    kpool = w.k_cache if pool_device_k is None else pool_device_k
    vpool = w.v_cache if pool_device_v is None else pool_device_v
    bs = w.block_size
    sel_pairs = [i for i, s in enumerate(w.pair_seq.tolist()) if s in pos]
    blocks = set()
    for s in seqs:
        nb = -(-int(w.context_lens[s]) // bs)
        blocks.update(int(x) for x in w.block_tables[s][:nb])
    for i in sel_pairs:
        blocks.update(int(x) for x in w.cow_pairs[i])
    order = sorted(blocks)
    remap = {b: i for i, b in enumerate(order)}
    idx = torch.tensor(order, dtype=torch.long, device=kpool.device)
    if kpool.dtype == torch.float8_e4m3fn:  # gather the codes as bytes
        k_sub = kpool.view(torch.uint8).index_select(0, idx).cpu().view(torch.float8_e4m3fn)
        v_sub = vpool.view(torch.uint8).index_select(0, idx).cpu().view(torch.float8_e4m3fn)
    else:
        k_sub = kpool.index_select(0, idx).cpu()
        v_sub = vpool.index_select(0, idx).cpu()
    bt = np.full((len(seqs), w.max_blocks_per_seq), -1, dtype=np.int32)
    for i, s in enumerate(seqs):
        nb = -(-int(w.context_lens[s]) // bs)
        bt[i, :nb] = [remap[int(x)] for x in w.block_tables[s][:nb]]
    toks = [i for i, s in enumerate(w.token_seq.tolist()) if s in pos]
    slots = np.asarray([remap[int(w.slot_mapping[i]) // bs] * bs + int(w.slot_mapping[i]) % bs
                        for i in toks], dtype=np.int64)
    tok_idx = torch.tensor(toks, dtype=torch.long)
    pairs = np.asarray([[remap[int(w.cow_pairs[i][0])], remap[int(w.cow_pairs[i][1])]]
                        for i in sel_pairs], dtype=np.int64).reshape(-1, 2)
    seq_idx = torch.tensor(seqs, dtype=torch.long)
    return wl.Workload(
        name=w.name + "_subset", dtype=w.dtype, num_seqs=len(seqs), num_heads=w.num_heads,
        num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, block_size=bs, num_blocks=len(order),
        max_blocks_per_seq=w.max_blocks_per_seq, scale=w.scale,
        context_lens=w.context_lens[seqs].copy(), block_tables=bt, cow_pairs=pairs,
        slot_mapping=slots, token_seq=np.asarray([pos[int(w.token_seq[i])] for i in toks],
                                                 dtype=np.int32),
        pair_seq=np.asarray([pos[int(w.pair_seq[i])] for i in sel_pairs], dtype=np.int32),
        q=w.q.index_select(0, seq_idx.to(w.q.device)).cpu(), k_cache=k_sub, v_cache=v_sub,
        k_new=w.k_new.index_select(0, tok_idx.to(w.k_new.device)).cpu(),
        v_new=w.v_new.index_select(0, tok_idx.to(w.v_new.device)).cpu(),
        meta={"blocks": order}, k_scales=w.k_scales, v_scales=w.v_scales)


def full_size_check(w: wl.Workload, partition_tokens: int = 0) -> float:
    """Every output row of a full-size step, element by element, and every
    pool block the step reads or writes, byte for byte.  The oracle runs on
    a compact host copy of the blocks the batch references (all sequences);
    the GPU runs the whole workload in place."""
    sub = subset(w, range(w.num_seqs))  # taken before the GPU step changes the pools
    ref, kref, vref = oracle_step(sub)
    out, kc, vc = gpu_step(w, partition_tokens=partition_tokens)
    idx = torch.tensor(sub.meta["blocks"], dtype=torch.long, device=kc.device)
    if kc.dtype == torch.float8_e4m3fn:
        k_used = kc.view(torch.uint8).index_select(0, idx).view(torch.float8_e4m3fn)
        v_used = vc.view(torch.uint8).index_select(0, idx).view(torch.float8_e4m3fn)
    else:
        k_used, v_used = kc.index_select(0, idx), vc.index_select(0, idx)
    assert_pool_equal(k_used, kref, "k pool (referenced blocks)")
    assert_pool_equal(v_used, vref, "v pool (referenced blocks)")
    return assert_close(out, ref, "bf16" if w.dtype == "fp8" else w.dtype)
