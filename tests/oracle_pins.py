"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
an independent fact: the worked example and block ranges printed on the pages
(``tests/golden/``), bounds the pages state, closed forms of attention,
invariances the paged layout implies, and a numpy brute force over contiguous
arrays that never sees a block table.  ``test_oracle_pins.py`` runs them;
``test_oracle_mutants.py`` plants mistakes in copies of the oracle and checks
that every planted mistake fails at least one pin.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import oracle
from oracle.brute import attention_contiguous

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- helpers
def read_golden_kv(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = (x.strip() for x in line.split("="))
            out[k] = int(v)
    return out


def read_golden_rows(name: str) -> list[list[int]]:
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(x) for x in line.split()])
    return rows


def to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """float array -> the oracle's input form: float32, or bf16 bits (RNE via torch)."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32))
    if dtype == "f32":
        return t.numpy().copy()
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def values(x: np.ndarray) -> np.ndarray:
    """The exact values an oracle input stands for, via torch's own conversion."""
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    return x.astype(np.float64)


def scatter(logical: list[np.ndarray], bs: int, num_blocks: int, rng, dtype: str,
            perm=None, fill=None):
    """Place per-sequence contiguous arrays [L][Hkv][D] into a pool of blocks.

    Written from the layout, not from the oracle: sequence s takes the next
    ceil(L/bs) blocks of a permutation, and block j receives rows j*bs .. of the
    sequence, transposed to [Hkv][rows][D].  Unused slots hold noise."""
    hkv, d = logical[0].shape[1], logical[0].shape[2]
    pool = rng.standard_normal((num_blocks, hkv, bs, d)).astype(np.float32) if fill is None else \
        np.full((num_blocks, hkv, bs, d), fill, dtype=np.float32)
    pool = to_dtype(pool, dtype)
    if perm is None:
        perm = rng.permutation(num_blocks)
    maxb = max(1, max(-(-x.shape[0] // bs) for x in logical))
    tables = np.full((len(logical), maxb), -1, dtype=np.int32)
    nxt = 0
    for s, arr in enumerate(logical):
        arr = to_dtype(arr, dtype) if arr.dtype != pool.dtype else arr
        for j in range(-(-arr.shape[0] // bs)):
            p = int(perm[nxt])
            nxt += 1
            tables[s, j] = p
            chunk = arr[j * bs:(j + 1) * bs]
            pool[p, :, : chunk.shape[0], :] = np.transpose(chunk, (1, 0, 2))
    return pool, tables


def random_case(seed: int, lens, H: int, Hkv: int, D: int, bs: int, dtype: str, spare: int = 5):
    rng = np.random.default_rng(seed)
    lk = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lens]
    lv = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lens]
    nblk = sum(-(-L // bs) for L in lens) + spare
    perm = rng.permutation(nblk)
    kp, tables = scatter(lk, bs, nblk, rng, dtype, perm=perm)
    vp, _ = scatter(lv, bs, nblk, rng, dtype, perm=perm)
    q = to_dtype(rng.standard_normal((len(lens), H, D)).astype(np.float32), dtype)
    lk = [to_dtype(x, dtype) for x in lk]
    lv = [to_dtype(x, dtype) for x in lv]
    return q, kp, vp, tables, np.asarray(lens, dtype=np.int32), lk, lv


def brute_all(q, lk, lv, scale, H, Hkv):
    G = H // Hkv
    out = np.zeros((q.shape[0], H, q.shape[2]))
    for s in range(q.shape[0]):
        for h in range(H):
            g = h // G
            out[s, h] = attention_contiguous(values(q)[s, h], values(lk[s])[:, g, :],
                                             values(lv[s])[:, g, :], scale)
    return out


# -------------------------------------------------------------------- pins
def pin_worked_example():
    gold = read_golden_kv("worked_example_unused_block_space.txt")
    bs, L = gold["block_size"], gold["sequence_length"]
    assert oracle.blocks_needed(L, bs) == gold["blocks"]
    alloc, unused = oracle.waste_per_sequence([L], bs)
    assert alloc == gold["allocated_slots"]
    assert unused == gold["unused_slots"]
    assert round(100.0 * unused / alloc) == gold["unused_percent_rounded"]


def pin_logical_block_ranges():
    """Token t of a sequence must come from the block at logical index t // bs."""
    for bs, first, last, j in read_golden_rows("logical_block_ranges.txt"):
        nblk = j + 2
        # each block's rows hold the block's own id, so the gathered value names the block
        pool = np.zeros((nblk, 1, bs, 1), dtype=np.float32)
        for p in range(nblk):
            pool[p] = p
        table = np.asarray([list(reversed(range(nblk)))], dtype=np.int32)  # logical j -> nblk-1-j
        got = oracle.gather(pool, table, 0, last + 1, 0)[:, 0]
        for t in (first, last):
            assert got[t] == nblk - 1 - j, (bs, t, got[t])


def pin_slot_within_block():
    """Slot t % bs of the block holds token t: rows keep their order inside a block."""
    bs, L = 8, 21
    rng = np.random.default_rng(7)
    lk = [np.arange(L, dtype=np.float32).reshape(L, 1, 1) * np.ones((1, 2, 3), np.float32)]
    pool, tables = scatter(lk, bs, 6, rng, "f32")
    for g in range(2):
        got = oracle.gather(pool, tables, 0, L, g)
        assert np.array_equal(got[:, 0], np.arange(L, dtype=np.float64)), got[:, 0]


def pin_waste_bound():
    """'At most part of one block': 0 <= unused <= bs - 1, zero exactly when L fills its blocks."""
    rng = np.random.default_rng(11)
    for bs in (1, 8, 16, 32):
        for L in list(rng.integers(1, 5000, size=200)) + [1, bs, bs + 1, 2 * bs - 1]:
            L = int(L)
            alloc, unused = oracle.waste_per_sequence([L], bs)
            assert alloc == oracle.blocks_needed(L, bs) * bs
            assert 0 <= unused <= bs - 1, (L, bs, unused)
            assert (unused == 0) == (L % bs == 0)
            assert alloc - unused == L
    assert oracle.blocks_needed(0, 16) == 0
    assert oracle.waste_per_sequence([0], 16) == (0, 0)


def pin_waste_physical():
    """Sharing counts each physical block once; without sharing it equals the per-sequence sum."""
    bs = 16
    lens = [35, 16, 50]
    tables = np.asarray([[4, 1, 7, -1], [0, -1, -1, -1], [2, 3, 5, 6]], dtype=np.int32)
    assert oracle.waste_physical(tables, lens, bs, 8) == oracle.waste_per_sequence(lens, bs)
    # two sequences sharing a 32-token prefix (blocks 0, 1), then 5 and 20 own tokens
    tables = np.asarray([[0, 1, 2, -1], [0, 1, 3, 4]], dtype=np.int32)
    lens = [37, 52]
    alloc, unused = oracle.waste_physical(tables, lens, bs, 5)
    # unique blocks 0,1,2,3,4 -> 80 slots; tokens held: 32 shared + 5 + 20
    assert alloc == 80 and unused == 80 - (32 + 5 + 20), (alloc, unused)


def pin_gather_bit_exact():
    """The gathered contiguous view equals the logical arrays that were placed, bit for bit."""
    for dtype in ("f32", "bf16"):
        q, kp, vp, tables, lens, lk, lv = random_case(3, [35, 16, 1, 50, 0], 4, 2, 8, 16, dtype)
        for s, L in enumerate(lens):
            for g in range(2):
                got = oracle.gather(kp, tables, s, int(L), g)
                assert np.array_equal(got, values(lk[s])[:, g, :]), (dtype, s, g)
                got = oracle.gather(vp, tables, s, int(L), g)
                assert np.array_equal(got, values(lv[s])[:, g, :]), (dtype, s, g)


def pin_attention_brute():
    """Against softmax(scale q K^T) V over contiguous arrays (numpy fp64)."""
    cases = [
        (21, [35, 16, 1, 50], 4, 4, 64, 16, "f32", 0.125),
        (22, [7, 129, 64, 1], 8, 2, 32, 8, "bf16", 1 / math.sqrt(32)),
        (23, [300, 33], 4, 1, 16, 32, "f32", 0.3),
        (24, [17, 5, 90], 6, 3, 8, 4, "bf16", 0.7),
    ]
    for seed, lens, H, Hkv, D, bs, dtype, scale in cases:
        q, kp, vp, tables, lens_a, lk, lv = random_case(seed, lens, H, Hkv, D, bs, dtype)
        got = oracle.paged_attention(q, kp, vp, tables, lens_a, scale)
        ref = brute_all(q, lk, lv, scale, H, Hkv)
        err = np.abs(got - ref).max()
        assert err <= 1e-12, (seed, err)


def pin_ctx_one():
    """One token attended: the softmax weight is exactly 1, so out == v_0 exactly."""
    for dtype in ("f32", "bf16"):
        q, kp, vp, tables, lens, lk, lv = random_case(31, [1, 1], 4, 2, 16, 8, dtype)
        got = oracle.paged_attention(q, kp, vp, tables, lens, 0.25)
        for s in range(2):
            for h in range(4):
                assert np.array_equal(got[s, h], values(lv[s])[0, h // 2, :])


def pin_uniform_weights():
    """Equal keys, or scale 0, give the plain column mean of V."""
    rng = np.random.default_rng(41)
    L, D = 45, 16
    k_row = rng.standard_normal((1, 1, D)).astype(np.float32)
    lk = [np.repeat(k_row, L, axis=0)]
    lv = [rng.standard_normal((L, 1, D)).astype(np.float32)]
    perm = rng.permutation(8)
    kp, tables = scatter(lk, 8, 8, rng, "f32", perm=perm)
    vp, _ = scatter(lv, 8, 8, rng, "f32", perm=perm)
    q = rng.standard_normal((1, 1, D)).astype(np.float32)
    mean = lv[0][:, 0, :].astype(np.float64).mean(axis=0)
    got = oracle.paged_attention(q, kp, vp, tables, [L], 0.5)[0, 0]
    assert np.abs(got - mean).max() <= 1e-13
    lk = [rng.standard_normal((L, 1, D)).astype(np.float32)]
    kp, tables = scatter(lk, 8, 8, rng, "f32", perm=perm)
    got = oracle.paged_attention(q, kp, vp, tables, [L], 0.0)[0, 0]
    assert np.abs(got - mean).max() <= 1e-13


def pin_dominant_logit():
    """A logit far above the rest takes all the weight: out -> that value row.
    Logits reach ~1e4 here, so a softmax without the max shift overflows."""
    rng = np.random.default_rng(51)
    L, D, j = 40, 16, 23
    lk = [rng.standard_normal((L, 1, D)).astype(np.float32)]
    lv = [rng.standard_normal((L, 1, D)).astype(np.float32)]
    perm = rng.permutation(6)
    kp, tables = scatter(lk, 16, 6, rng, "f32", perm=perm)
    vp, _ = scatter(lv, 16, 6, rng, "f32", perm=perm)
    q = (lk[0][j, 0, :] * 4.0).reshape(1, 1, D)
    got = oracle.paged_attention(q, kp, vp, tables, [L], 300.0)[0, 0]
    assert np.all(np.isfinite(got))
    assert np.abs(got - lv[0][j, 0, :]).max() <= 1e-9


def pin_permutation_invariance():
    """'Physical blocks can be anywhere and in any order': moving the blocks
    (data and table together) leaves every output bit-identical."""
    for dtype in ("f32", "bf16"):
        q, kp, vp, tables, lens, lk, lv = random_case(61, [35, 16, 1, 50, 77], 4, 2, 16, 16, dtype)
        base = oracle.paged_attention(q, kp, vp, tables, lens, 0.25)
        rng = np.random.default_rng(62)
        perm = rng.permutation(kp.shape[0])  # new position of old block i is perm[i]
        kp2 = np.empty_like(kp)
        vp2 = np.empty_like(vp)
        kp2[perm] = kp
        vp2[perm] = vp
        t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1).astype(np.int32)
        got = oracle.paged_attention(q, kp2, vp2, t2, lens, 0.25)
        assert np.array_equal(got, base)


def pin_sharing_equals_private():
    """Two sequences pointing at the same physical prefix blocks give exactly
    the outputs they give with private byte-identical copies."""
    rng = np.random.default_rng(71)
    bs, D, Hkv, H = 8, 16, 2, 4
    prefix = rng.standard_normal((24, Hkv, D)).astype(np.float32)
    tails = [rng.standard_normal((n, Hkv, D)).astype(np.float32) for n in (5, 11)]
    lk = [np.concatenate([prefix, t]) for t in tails]
    lv = [np.concatenate([prefix[::-1] * 0.5, t * 2]) for t in tails]
    nblk = 12
    perm = rng.permutation(nblk)
    kp, tables = scatter(lk, bs, nblk, rng, "f32", perm=perm)
    vp, _ = scatter(lv, bs, nblk, rng, "f32", perm=perm)
    q = rng.standard_normal((2, H, D)).astype(np.float32)
    lens = [29, 35]
    private = oracle.paged_attention(q, kp, vp, tables, lens, 0.25)
    shared_tables = tables.copy()
    shared_tables[1, :3] = tables[0, :3]  # seq 1 now reads seq 0's prefix blocks
    shared = oracle.paged_attention(q, kp, vp, shared_tables, lens, 0.25)
    assert np.array_equal(private, shared)


def pin_gqa_equals_duplicated_mha():
    """Grouped-query attention equals multi-head attention over a cache whose
    kv heads are repeated group-size times, in order."""
    G = 4
    q, kp, vp, tables, lens, lk, lv = random_case(81, [19, 40, 3], 8, 2, 16, 8, "f32")
    got = oracle.paged_attention(q, kp, vp, tables, lens, 0.3)
    kp_m = np.ascontiguousarray(np.repeat(kp, G, axis=1))
    vp_m = np.ascontiguousarray(np.repeat(vp, G, axis=1))
    ref = oracle.paged_attention(q, kp_m, vp_m, tables, lens, 0.3)
    assert np.array_equal(got, ref)


def pin_ctx_zero():
    q, kp, vp, tables, lens, lk, lv = random_case(91, [0, 5], 2, 2, 8, 4, "f32")
    got = oracle.paged_attention(q, kp, vp, tables, lens, 0.5)
    assert np.array_equal(got[0], np.zeros((2, 8)))
    assert np.all(got[1] != 0)


def pin_rows_subset():
    q, kp, vp, tables, lens, lk, lv = random_case(92, [35, 16, 1, 50], 4, 2, 16, 16, "bf16")
    full = oracle.paged_attention(q, kp, vp, tables, lens, 0.25)
    rows = np.asarray([[3, 1], [0, 0], [2, 3], [3, 3]], dtype=np.int32)
    part = oracle.paged_attention(q, kp, vp, tables, lens, 0.25, rows=rows)
    for i, (s, h) in enumerate(rows):
        assert np.array_equal(part[i], full[s, h])


def pin_append_extends_logical():
    """'Grows by one entry for every new token': after appending rows at the
    slots of positions L .. L+n-1, the gathered view is the old one extended by
    exactly those rows.  A slot of -1 writes nothing."""
    for dtype in ("f32", "bf16"):
        rng = np.random.default_rng(101)
        bs, Hkv, D = 8, 2, 16
        lens = [13, 8]
        new = [4, 9]
        q, kp, vp, tables, lens_a, lk, lv = random_case(102, lens, 2, Hkv, D, bs, dtype, spare=6)
        used = set(int(x) for x in tables[tables >= 0])
        free = [p for p in range(kp.shape[0]) if p not in used]
        maxb = max(-(-(L + n) // bs) for L, n in zip(lens, new))
        t2 = np.full((2, maxb), -1, dtype=np.int32)
        t2[:, : tables.shape[1]] = tables
        slots, rows_k, rows_v, expect_k, expect_v = [], [], [], [], []
        for s, (L, n) in enumerate(zip(lens, new)):
            nk = to_dtype(rng.standard_normal((n, Hkv, D)).astype(np.float32), dtype)
            nv = to_dtype(rng.standard_normal((n, Hkv, D)).astype(np.float32), dtype)
            for i in range(n):
                t = L + i
                if t2[s, t // bs] < 0:
                    t2[s, t // bs] = free.pop(0)
                slots.append(int(t2[s, t // bs]) * bs + t % bs)
            rows_k.append(nk)
            rows_v.append(nv)
            expect_k.append(np.concatenate([lk[s], nk]))
            expect_v.append(np.concatenate([lv[s], nv]))
        slots.append(-1)
        rows_k.append(to_dtype(np.full((1, Hkv, D), 1e3, np.float32), dtype))
        rows_v.append(to_dtype(np.full((1, Hkv, D), 1e3, np.float32), dtype))
        k_all = np.ascontiguousarray(np.concatenate(rows_k))
        v_all = np.ascontiguousarray(np.concatenate(rows_v))
        before_k = kp.copy()
        oracle.kv_append(kp, vp, k_all, v_all, np.asarray(slots, dtype=np.int64))
        touched = set(s // bs for s in slots if s >= 0)
        for p in range(kp.shape[0]):
            if p not in touched:
                assert np.array_equal(kp[p].view(np.uint8), before_k[p].view(np.uint8))
        for s, (L, n) in enumerate(zip(lens, new)):
            for g in range(Hkv):
                got = oracle.gather(kp, t2, s, L + n, g)
                assert np.array_equal(got, values(expect_k[s])[:, g, :]), (dtype, s, g)
                got = oracle.gather(vp, t2, s, L + n, g)
                assert np.array_equal(got, values(expect_v[s])[:, g, :]), (dtype, s, g)


def pin_copy_on_write():
    """Copy-on-write: the writer copies the shared block first, its table is
    updated, then it appends.  The sibling's blocks and outputs are
    byte-identical to before; the writer's new block equals the source except
    at the appended slot."""
    for dtype in ("f32", "bf16"):
        rng = np.random.default_rng(111)
        bs, Hkv, D, H = 8, 2, 16, 4
        prompt = rng.standard_normal((20, Hkv, D)).astype(np.float32)
        perm = rng.permutation(8)
        kp, tables = scatter([prompt], bs, 8, rng, dtype, perm=perm)
        vp, _ = scatter([prompt * -1.5], bs, 8, rng, dtype, perm=perm)
        shared = tables[0, :3].copy()
        t_sib = np.asarray([shared], dtype=np.int32)
        t_wr = t_sib.copy()
        q = to_dtype(rng.standard_normal((2, H, D)).astype(np.float32), dtype)
        sib_before = oracle.paged_attention(q[:1], kp, vp, t_sib, [20], 0.25)
        k_before, v_before = kp.copy(), vp.copy()
        src = int(shared[2])  # partial block: slots 0..3 hold tokens 16..19
        dst = [p for p in range(8) if p not in set(shared.tolist())][0]
        oracle.copy_blocks(kp, vp, np.asarray([[src, dst]], dtype=np.int64))
        t_wr[0, 2] = dst
        nk = to_dtype(rng.standard_normal((1, Hkv, D)).astype(np.float32), dtype)
        nv = to_dtype(rng.standard_normal((1, Hkv, D)).astype(np.float32), dtype)
        oracle.kv_append(kp, vp, nk, nv, np.asarray([dst * bs + 4], dtype=np.int64))
        for p in shared:
            assert np.array_equal(kp[p].view(np.uint8), k_before[p].view(np.uint8))
            assert np.array_equal(vp[p].view(np.uint8), v_before[p].view(np.uint8))
        sib_after = oracle.paged_attention(q[:1], kp, vp, t_sib, [20], 0.25)
        assert np.array_equal(sib_before, sib_after)
        for pool, before, new in ((kp, k_before, nk), (vp, v_before, nv)):
            for slot in range(bs):
                if slot == 4:
                    assert np.array_equal(pool[dst, :, slot, :].view(np.uint8), new[0].view(np.uint8))
                else:
                    assert np.array_equal(pool[dst, :, slot, :].view(np.uint8),
                                          before[src, :, slot, :].view(np.uint8))
        # the writer now sees the prompt plus its new token
        got = oracle.gather(kp, t_wr, 0, 21, 1)
        assert np.array_equal(got[:20], values(k_before[shared].transpose(1, 0, 2, 3)
                                               .reshape(Hkv, 3 * bs, D)[1, :20]))
        assert np.array_equal(got[20], values(nk)[0, 1])


def pin_copy_blocks_pairs():
    """Each pair copies one whole block (every kv head, slot and element, K and V)."""
    for dtype in ("f32", "bf16"):
        rng = np.random.default_rng(121)
        kp = to_dtype(rng.standard_normal((10, 3, 4, 8)).astype(np.float32), dtype)
        vp = to_dtype(rng.standard_normal((10, 3, 4, 8)).astype(np.float32), dtype)
        k0, v0 = kp.copy(), vp.copy()
        pairs = np.asarray([[2, 7], [5, 0], [9, 3]], dtype=np.int64)
        oracle.copy_blocks(kp, vp, pairs)
        dsts = set(pairs[:, 1].tolist())
        for s, d in pairs:
            assert np.array_equal(kp[d].view(np.uint8), k0[s].view(np.uint8))
            assert np.array_equal(vp[d].view(np.uint8), v0[s].view(np.uint8))
        for p in range(10):
            if p not in dsts:
                assert np.array_equal(kp[p].view(np.uint8), k0[p].view(np.uint8))


def pin_swap_round_trip():
    """Swapping moves whole blocks between pools: out and back in (to other
    blocks) gives the same bytes; blocks not named stay as they were."""
    for dtype in ("f32", "bf16"):
        rng = np.random.default_rng(131)
        dk = to_dtype(rng.standard_normal((8, 2, 4, 8)).astype(np.float32), dtype)
        dv = to_dtype(rng.standard_normal((8, 2, 4, 8)).astype(np.float32), dtype)
        hk = np.zeros((5, 2, 4, 8), dtype=dk.dtype)
        hv = np.zeros((5, 2, 4, 8), dtype=dk.dtype)
        k0, v0 = dk.copy(), dv.copy()
        out_pairs = np.asarray([[6, 0], [1, 3], [4, 4]], dtype=np.int64)
        oracle.swap_blocks(hk, hv, dk, dv, out_pairs)
        for d, h in out_pairs:
            assert np.array_equal(hk[h].view(np.uint8), k0[d].view(np.uint8))
            assert np.array_equal(hv[h].view(np.uint8), v0[d].view(np.uint8))
        assert not hk[[1, 2]].any()
        back = np.asarray([[0, 2], [3, 7], [4, 5]], dtype=np.int64)
        oracle.swap_blocks(dk, dv, hk, hv, back)
        for (d, h), (h2, d2) in zip(out_pairs, back):
            assert np.array_equal(dk[d2].view(np.uint8), k0[d].view(np.uint8))
            assert np.array_equal(dv[d2].view(np.uint8), v0[d].view(np.uint8))
        for p in (0, 1, 3, 4, 6):
            assert np.array_equal(dk[p].view(np.uint8), k0[p].view(np.uint8))


def _torch_e4m3_codes(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_e4m3_decode():
    """Every e4m3 code's value equals torch's float8_e4m3fn conversion."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    got = np.asarray([oracle.e4m3_value(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9


def pin_e4m3_encode():
    """Round to nearest (ties to even) as torch does inside the finite range;
    saturation to +-448 beyond it (torch gives NaN there); NaN stays NaN;
    every finite code round-trips."""
    rng = np.random.default_rng(141)
    xs = np.concatenate([
        rng.uniform(-463, 463, 4000), rng.normal(0, 1, 4000), rng.normal(0, 1e-2, 2000),
        np.ldexp(rng.uniform(-1, 1, 2000), -8),
        # exact grid points and midpoints between neighbouring codes
        [oracle.e4m3_value(c) for c in range(0x7F)],
        [(oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2 for c in range(0x7E)],
    ]).astype(np.float32)
    ref = _torch_e4m3_codes(xs)
    got = np.asarray([oracle.e4m3_encode(float(x)) for x in xs], dtype=np.uint8)
    assert np.array_equal(got, ref), np.flatnonzero(got != ref)[:5]
    for y, code in ((464.0, 0x7E), (1e9, 0x7E), (-500.0, 0xFE), (float("inf"), 0x7E),
                    (float("-inf"), 0xFE)):
        assert oracle.e4m3_encode(y) == code, (y, oracle.e4m3_encode(y))
    assert oracle.e4m3_encode(float("nan")) & 0x7F == 0x7F
    for c in list(range(0x7F)) + list(range(0x80, 0xFF)):
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c


def _fp8_case(seed, lens, H, Hkv, D, bs, ks, vs):
    rng = np.random.default_rng(seed)
    nblk = sum(-(-L // bs) for L in lens) + 3
    kc = rng.integers(0, 256, size=(nblk, Hkv, bs, D)).astype(np.uint8)
    vc = rng.integers(0, 256, size=(nblk, Hkv, bs, D)).astype(np.uint8)
    for c in (kc, vc):  # no NaN codes
        c[(c & 0x7F) == 0x7F] = 0x7E
    perm = rng.permutation(nblk)
    bt = np.full((len(lens), max(-(-L // bs) for L in lens)), -1, dtype=np.int32)
    nxt = 0
    for s, L in enumerate(lens):
        for j in range(-(-L // bs)):
            bt[s, j] = perm[nxt]
            nxt += 1
    q = to_dtype(rng.standard_normal((len(lens), H, D)).astype(np.float32) * 0.05, "bf16")
    return q, kc, vc, np.asarray(ks, np.float32), np.asarray(vs, np.float32), bt, np.asarray(lens, np.int32)


def pin_fp8_attention():
    """With power-of-two scales every dequantised value is an fp32 number, and
    the fp8 oracle equals the plain oracle on the dequantised caches exactly;
    with other scales it matches a numpy brute force."""
    H, Hkv, D, bs = 4, 2, 16, 8
    q, kc, vc, ks, vs, bt, lens = _fp8_case(151, [19, 40, 3, 0], H, Hkv, D, bs, [0.25, 0.0625], [0.5, 2.0])
    got = oracle.paged_attention_fp8(q, kc, vc, ks, vs, bt, lens, 0.3)
    deq = np.vectorize(oracle.e4m3_value)
    kf = (deq(kc) * ks[None, :, None, None]).astype(np.float32)
    vf = (deq(vc) * vs[None, :, None, None]).astype(np.float32)
    qf = values(q).astype(np.float32)
    ref = oracle.paged_attention(qf, kf, vf, bt, lens, 0.3)
    assert np.array_equal(got, ref)
    q, kc, vc, ks, vs, bt, lens = _fp8_case(152, [33, 7], H, Hkv, D, bs, [0.013, 0.021], [0.017, 0.3])
    got = oracle.paged_attention_fp8(q, kc, vc, ks, vs, bt, lens, 0.25)
    for s, L in enumerate(lens):
        for h in range(H):
            g = h // (H // Hkv)
            rows = [bt[s, t // bs] for t in range(L)]
            K = np.stack([deq(kc[p, g, t % bs]) for t, p in enumerate(rows)]) * float(ks[g])
            V = np.stack([deq(vc[p, g, t % bs]) for t, p in enumerate(rows)]) * float(vs[g])
            ref = attention_contiguous(values(q)[s, h], K, V, 0.25)
            assert np.abs(got[s, h] - ref).max() <= 1e-12


def pin_fp8_append():
    """Appended rows hold torch's e4m3 codes of (fp32 x) / scale; -1 skips."""
    rng = np.random.default_rng(161)
    Hkv, D, bs = 2, 16, 4
    kc = np.zeros((6, Hkv, bs, D), np.uint8)
    vc = np.zeros((6, Hkv, bs, D), np.uint8)
    k = to_dtype(rng.standard_normal((3, Hkv, D)).astype(np.float32) * 3, "bf16")
    v = to_dtype(rng.standard_normal((3, Hkv, D)).astype(np.float32) * 3, "bf16")
    ks = np.asarray([0.02, 0.5], np.float32)
    vs = np.asarray([0.125, 0.03], np.float32)
    slots = np.asarray([5, -1, 17], np.int64)
    oracle.kv_append_fp8(kc, vc, ks, vs, k, v, slots)
    for i, slot in enumerate(slots):
        if slot < 0:
            continue
        for g in range(Hkv):
            kx = values(k)[i, g].astype(np.float32) / ks[g]
            vx = values(v)[i, g].astype(np.float32) / vs[g]
            assert np.array_equal(kc[slot // bs, g, slot % bs], _torch_e4m3_codes(np.clip(kx, -448, 448)))
            assert np.array_equal(vc[slot // bs, g, slot % bs], _torch_e4m3_codes(np.clip(vx, -448, 448)))
    assert not kc[[0, 2, 3, 5]].any()  # token 1 was skipped; only blocks 1 and 4 written


PINS = [
    pin_worked_example,
    pin_logical_block_ranges,
    pin_slot_within_block,
    pin_waste_bound,
    pin_waste_physical,
    pin_gather_bit_exact,
    pin_attention_brute,
    pin_ctx_one,
    pin_uniform_weights,
    pin_dominant_logit,
    pin_permutation_invariance,
    pin_sharing_equals_private,
    pin_gqa_equals_duplicated_mha,
    pin_ctx_zero,
    pin_rows_subset,
    pin_append_extends_logical,
    pin_copy_on_write,
    pin_copy_blocks_pairs,
    pin_swap_round_trip,
    pin_e4m3_decode,
    pin_e4m3_encode,
    pin_fp8_attention,
    pin_fp8_append,
]
