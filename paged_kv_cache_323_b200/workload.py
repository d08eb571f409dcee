"""Seeded synthetic workloads for the paged decode step.

This module only DRAWS inputs: sequence lengths, the sharing structure, the
physical placement of blocks, and the tensors.  It holds none of the
attention arithmetic, and both the CUDA path and the CPU oracle consume what it
produces.  It is the only module the two sides share.

The workloads mirror the serving scenarios the pages describe: many concurrent
sequences of varied length ("PagedAttention Explained: Virtual Memory for the
KV Cache", section "The problem: the KV cache is big and unpredictable"),
parallel sampling and shared prefixes with copy-on-write (section "Sharing
blocks between sequences"), and block-size tuning (section "Trade-offs and
related techniques").

Draw order, fixed per workload: lengths -> sharing structure -> physical
placement (a seeded permutation of the pool's blocks, consumed as a free list)
-> q -> the whole K/V pool (unused slots included) -> the new tokens' K/V.
Structure comes from ``numpy.random.Generator(PCG64(seed))``.  Tensors come
from the same numpy generator on the CPU, or from a ``torch.Generator`` seeded
with ``seed`` on the GPU for pools too large to draw on the host; fp32 N(0, 1)
draws are rounded to bf16 by round-to-nearest-even (``Tensor.to``).

A decode step on a workload is: copy-on-write block copies (``cow_pairs``,
possibly none), then the append of the step's new tokens (``slot_mapping``),
then one decode query per sequence over ``context_lens`` tokens, which count
the tokens appended in this step.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.float8_e4m3fn}


@dataclass
class Workload:
    name: str
    dtype: str  # "f32" or "bf16"
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    max_blocks_per_seq: int
    scale: float
    context_lens: np.ndarray  # int32 [B]
    block_tables: np.ndarray  # int32 [B][max_blocks_per_seq], -1 where unallocated
    cow_pairs: np.ndarray  # int64 [n][2] (src, dst)
    slot_mapping: np.ndarray  # int64 [T]
    token_seq: np.ndarray  # int32 [T]: the sequence each new token belongs to
    pair_seq: np.ndarray  # int32 [n]: the writer each copy-on-write pair serves
    q: torch.Tensor  # [B][H][D]
    k_cache: torch.Tensor  # [N][Hkv][bs][D], state BEFORE the step
    v_cache: torch.Tensor
    k_new: torch.Tensor  # [T][Hkv][D]
    v_new: torch.Tensor
    meta: dict = field(default_factory=dict)
    k_scales: np.ndarray | None = None  # fp8 caches: float32 [Hkv], stored value = code * scale
    v_scales: np.ndarray | None = None

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads

    @property
    def elt(self) -> int:
        return {"f32": 4, "bf16": 2, "fp8": 1}[self.dtype]

    def kv_bytes_logical(self) -> int:
        """K and V bytes one decode step reads, counting every sequence."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * self.head_dim * 2 * self.elt

    def padded_slot_waste(self) -> dict:
        """Slots allocated but holding no token: per sequence (every table
        counted on its own) and physical (each distinct block once, with the
        longest prefix any sequence uses)."""
        bs = self.block_size
        lens = self.context_lens.astype(np.int64)
        alloc = int(((lens + bs - 1) // bs * bs).sum())
        used_slots = {}
        for s in range(self.num_seqs):
            L = int(lens[s])
            for j in range(-(-L // bs)):
                b = int(self.block_tables[s][j])
                used_slots[b] = max(used_slots.get(b, 0), min(bs, L - j * bs))
        phys_alloc = len(used_slots) * bs
        phys_used = sum(used_slots.values())
        return {"per_sequence_allocated": alloc, "per_sequence_unused": alloc - int(lens.sum()),
                "physical_allocated": phys_alloc, "physical_unused": phys_alloc - phys_used}

    def kv_bytes_unique(self) -> int:
        """The same over distinct physical blocks: a block shared by several
        sequences counts once, with the longest prefix any of them uses."""
        bs = self.block_size
        used = {}
        for s in range(self.num_seqs):
            L = int(self.context_lens[s])
            for j in range(-(-L // bs)):
                b = int(self.block_tables[s][j])
                used[b] = max(used.get(b, 0), min(bs, L - j * bs))
        return sum(used.values()) * self.num_kv_heads * self.head_dim * 2 * self.elt


class _Pool:
    """Free list of physical blocks in a seeded random order, with refcounts."""

    def __init__(self, rng: np.random.Generator, num_blocks: int):
        self.order = list(rng.permutation(num_blocks).astype(np.int64))
        self.pos = 0
        self.ref = np.zeros(num_blocks, dtype=np.int64)

    def take(self) -> int:
        if self.pos >= len(self.order):
            raise RuntimeError("out of free KV blocks")
        b = int(self.order[self.pos])
        self.pos += 1
        self.ref[b] = 1
        return b


def _normal(shape, rng: np.random.Generator, tgen, device, dtype: str, mult=1.0):
    """N(0, 1) fp32 draws times `mult` (a number, or per-kv-head values
    broadcast over dim 1), rounded to `dtype` (nearest even, by torch)."""
    if device == "cpu" or device is None:
        x = torch.from_numpy(rng.standard_normal(size=shape, dtype=np.float32))
    else:
        x = torch.randn(*shape, generator=tgen, device=device, dtype=torch.float32)
    if isinstance(mult, np.ndarray):
        x = x * torch.from_numpy(mult.astype(np.float32)).to(x.device).view(1, -1, *([1] * (len(shape) - 2)))
    elif mult != 1.0:
        x = x * mult
    return x.to(DTYPES[dtype]).contiguous()


def fp8_scales(num_kv_heads: int):
    """Per-kv-head scales of the fp8 workloads (stored value = code * scale):
    codes of N(0, 1) / scale stay well inside e4m3's +-448."""
    g = np.arange(num_kv_heads, dtype=np.float32)
    return ((1.0 + 0.37 * g) / 32.0).astype(np.float32), ((1.0 + 0.21 * g) / 24.0).astype(np.float32)


def _finish(name, dtype, rng, seed, device, *, lens, tables, cow_pairs, new_pos, num_blocks,
            H, Hkv, D, bs, maxb, q_mult=1.0, meta=None, pair_seq=()) -> Workload:
    """Shared tail of every generator: slots of the new tokens, then tensors."""
    B = len(lens)
    slots, owners = [], []
    for s, positions in enumerate(new_pos):
        for t in positions:
            slots.append(int(tables[s][t // bs]) * bs + t % bs)
            owners.append(s)
    slot_mapping = np.asarray(slots, dtype=np.int64)
    tgen = None
    if device not in (None, "cpu"):
        tgen = torch.Generator(device=device)
        tgen.manual_seed(seed)
    act = "bf16" if dtype == "fp8" else dtype  # q and new tokens of an fp8 cache are bf16
    ks = vs = None
    kmul = vmul = 1.0
    if dtype == "fp8":
        ks, vs = fp8_scales(Hkv)
        kmul, vmul = 1.0 / ks, 1.0 / vs
    q = _normal((B, H, D), rng, tgen, device, act, q_mult)
    k_cache = _normal((num_blocks, Hkv, bs, D), rng, tgen, device, dtype, kmul)
    v_cache = _normal((num_blocks, Hkv, bs, D), rng, tgen, device, dtype, vmul)
    T = len(slot_mapping)
    k_new = _normal((T, Hkv, D), rng, tgen, device, act)
    v_new = _normal((T, Hkv, D), rng, tgen, device, act)
    bt = np.full((B, maxb), -1, dtype=np.int32)
    for s, row in enumerate(tables):
        bt[s, : len(row)] = row
    return Workload(
        name=name, dtype=dtype, num_seqs=B, num_heads=H, num_kv_heads=Hkv, head_dim=D,
        block_size=bs, num_blocks=num_blocks, max_blocks_per_seq=maxb,
        scale=float(np.float32(1.0 / math.sqrt(D))), context_lens=np.asarray(lens, dtype=np.int32),
        block_tables=bt, cow_pairs=np.asarray(cow_pairs, dtype=np.int64).reshape(-1, 2),
        slot_mapping=slot_mapping, token_seq=np.asarray(owners, dtype=np.int32),
        pair_seq=np.asarray(pair_seq, dtype=np.int32), q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new,
        v_new=v_new, meta=meta or {}, k_scales=ks, v_scales=vs)


class _InOrderPool(_Pool):
    """Free list in ascending block order: each sequence's blocks come out
    consecutive, as with one contiguous reservation per request."""

    def __init__(self, num_blocks: int):
        self.order = list(range(num_blocks))
        self.pos = 0
        self.ref = np.zeros(num_blocks, dtype=np.int64)


def _private(lens, rng, num_blocks, bs, new_per_seq=1, contiguous=False):
    """Every sequence owns its blocks; the last ``new_per_seq`` positions are new."""
    pool = _InOrderPool(num_blocks) if contiguous else _Pool(rng, num_blocks)
    tables, new_pos = [], []
    for L in lens:
        nb = -(-int(L) // bs)
        tables.append([pool.take() for _ in range(nb)])
        n_new = min(new_per_seq, int(L))
        new_pos.append(list(range(int(L) - n_new, int(L))))
    return tables, new_pos


def tiny(seed: int = 1, device="cpu") -> Workload:
    """4 sequences, lengths {35, 16, 1, 50}, bs 16, 4 = 4 heads, d 64, fp32, pool 32."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = [35, 16, 1, 50]
    tables, new_pos = _private(lens, rng, 32, 16)
    return _finish("tiny", "f32", rng, seed, device, lens=lens, tables=tables, cow_pairs=[],
                   new_pos=new_pos, num_blocks=32, H=4, Hkv=4, D=64, bs=16, maxb=4)


def mha(seed: int = 2, device="cpu", num_seqs: int = 64, ctx_range=(128, 2048),
        num_blocks: int | None = None, heads: int = 32, head_dim: int = 128, block_size: int = 16,
        dtype: str = "bf16", contiguous: bool = False) -> Workload:
    """Batch 64, 32 = 32 heads, d 128, bf16, bs 16, ctx U[128, 2048], pool of
    16384 blocks (the same 256 Ki tokens at other block sizes).  With
    ``contiguous`` every sequence's blocks are consecutive in the pool (the
    layout of a contiguous per-request cache, still read through the table)
    instead of a seeded random placement."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = rng.integers(ctx_range[0], ctx_range[1], size=num_seqs, endpoint=True).tolist()
    if num_blocks is None:
        num_blocks = 16384 * 16 // block_size
    tables, new_pos = _private(lens, rng, num_blocks, block_size, contiguous=contiguous)
    maxb = -(-ctx_range[1] // block_size)
    return _finish("mha", dtype, rng, seed, device, lens=lens, tables=tables, cow_pairs=[],
                   new_pos=new_pos, num_blocks=num_blocks, H=heads, Hkv=heads, D=head_dim,
                   bs=block_size, maxb=maxb)


def gqa_sampling(seed: int = 3, device="cpu", groups: int = 64, samples: int = 4,
                 prompt_median: int = 1024, prompt_sigma: float = 1.0, prompt_max: int = 8192,
                 gen_range=(1, 64), heads: int = 32, kv_heads: int = 8, head_dim: int = 128,
                 block_size: int = 16, dtype: str = "bf16", slack: float = 0.10) -> Workload:
    """Parallel sampling: groups of samples share their prompt's blocks by refcount.

    Each sample then writes its own 1..64 generated tokens in this step.  A
    writer whose first target block is shared (refcount > 1) gets a private
    copy first (copy-on-write, table updated, refcount decremented); the last
    holder writes in place.  Prompt lengths are round(exp(N(ln median, sigma)))
    clipped to [1, max]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    prompts = np.clip(np.rint(np.exp(rng.normal(math.log(prompt_median), prompt_sigma, size=groups))),
                      1, prompt_max).astype(np.int64)
    gens = rng.integers(gen_range[0], gen_range[1], size=(groups, samples), endpoint=True)
    bs = block_size
    need = 0
    for P, gs in zip(prompts, gens):
        need += -(-int(P) // bs) + samples
        need += sum(-(-int(P + g) // bs) - -(-int(P) // bs) for g in gs)
    num_blocks = int(math.ceil(need * (1.0 + slack)))
    pool = _Pool(rng, num_blocks)
    tables, new_pos, lens, cow, cow_seq = [], [], [], [], []
    for P, gs in zip(prompts, gens):
        P = int(P)
        shared = [pool.take() for _ in range(-(-P // bs))]
        for b in shared:
            pool.ref[b] = samples
        for i in range(samples):
            table = list(shared)
            L = P + int(gs[i])
            first = P // bs  # logical block of the first new token
            if first < len(table) and pool.ref[table[first]] > 1:
                src = table[first]
                dst = pool.take()
                pool.ref[src] -= 1
                cow.append((src, dst))
                cow_seq.append(len(tables))
                table[first] = dst
            while len(table) < -(-L // bs):
                table.append(pool.take())
            tables.append(table)
            lens.append(L)
            new_pos.append(list(range(P, L)))
    maxb = max(len(t) for t in tables)
    return _finish("gqa_sampling", dtype, rng, seed, device, lens=lens, tables=tables,
                   cow_pairs=cow, new_pos=new_pos, num_blocks=num_blocks, H=heads, Hkv=kv_heads,
                   D=head_dim, bs=bs, maxb=maxb, pair_seq=cow_seq,
                   meta={"prompts": prompts.tolist(), "gens": gens.tolist(), "samples": samples})


def long_context(seed: int = 4, device="cpu", num_seqs: int = 8, ctx_range=(32768, 131072),
                 heads: int = 64, kv_heads: int = 8, head_dim: int = 128, block_size: int = 32,
                 dtype: str = "bf16", q_mult: float = 0.5) -> Workload:
    """Batch 8, ctx U[32768, 131072], 64 / 8 heads, d 128, bs 32, q scaled by 0.5."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = rng.integers(ctx_range[0], ctx_range[1], size=num_seqs, endpoint=True).tolist()
    num_blocks = sum(-(-int(L) // block_size) for L in lens)
    tables, new_pos = _private(lens, rng, num_blocks, block_size)
    maxb = -(-ctx_range[1] // block_size)
    return _finish("long_context", dtype, rng, seed, device, lens=lens, tables=tables,
                   cow_pairs=[], new_pos=new_pos, num_blocks=num_blocks, H=heads, Hkv=kv_heads,
                   D=head_dim, bs=block_size, maxb=maxb, q_mult=q_mult)


def prefix_sweep(block_size: int, seed: int = 5, device="cpu", num_seqs: int = 1024,
                 prefix: int = 2048, suffix_range=(16, 512), heads: int = 32, kv_heads: int = 8,
                 head_dim: int = 128, dtype: str = "bf16") -> Workload:
    """1024 sequences share one 2048-token prefix (same physical blocks), then
    own a suffix of U[16, 512] tokens whose last token is appended this step."""
    rng = np.random.Generator(np.random.PCG64(seed))
    suffixes = rng.integers(suffix_range[0], suffix_range[1], size=num_seqs, endpoint=True)
    bs = block_size
    if prefix % bs:
        raise ValueError("the prefix must fill whole blocks (no shared partial block)")
    n_prefix = -(-prefix // bs)
    need = n_prefix + sum(-(-(prefix + int(x)) // bs) - prefix // bs for x in suffixes)
    num_blocks = int(need)
    pool = _Pool(rng, num_blocks)
    shared = [pool.take() for _ in range(n_prefix)]
    for b in shared:
        pool.ref[b] = num_seqs
    tables, new_pos, lens = [], [], []
    for x in suffixes:
        L = prefix + int(x)
        table = list(shared)
        while len(table) < -(-L // bs):
            table.append(pool.take())
        tables.append(table)
        lens.append(L)
        new_pos.append([L - 1])
    maxb = -(-(prefix + suffix_range[1]) // bs)
    return _finish(f"prefix_sweep_bs{bs}", dtype, rng, seed, device, lens=lens, tables=tables,
                   cow_pairs=[], new_pos=new_pos, num_blocks=num_blocks, H=heads, Hkv=kv_heads,
                   D=head_dim, bs=bs, maxb=maxb, meta={"prefix_blocks": shared})


def custom(seed: int, lens, *, heads: int, kv_heads: int, head_dim: int, block_size: int,
           dtype: str, num_blocks: int | None = None, new_per_seq: int = 1, device="cpu",
           maxb: int | None = None) -> Workload:
    """Private blocks for the given lengths (edge cases: empty, ragged, extremes)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = [int(x) for x in lens]
    need = sum(-(-L // block_size) for L in lens)
    if num_blocks is None:
        num_blocks = max(1, need + 3)
    tables, new_pos = _private(lens, rng, num_blocks, block_size, new_per_seq)
    if maxb is None:
        maxb = max([1] + [len(t) for t in tables])
    return _finish("custom", dtype, rng, seed, device, lens=lens, tables=tables, cow_pairs=[],
                   new_pos=new_pos, num_blocks=num_blocks, H=heads, Hkv=kv_heads, D=head_dim,
                   bs=block_size, maxb=maxb)


def to_numpy_bits(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a tensor for the oracle: float32 as is, bf16 as raw bits."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    raise TypeError(t.dtype)


def from_numpy_bits(a: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
    return torch.from_numpy(a.copy())
