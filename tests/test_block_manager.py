"""The native block manager (host code, no GPU) against the pages' rules.

A small Python model written from the rules (allocate a block only when the
last one is full; forks share blocks by refcount; a writer whose partly
filled last block is shared copies it first; the last holder writes in
place; a finished request releases its blocks) runs the same seeded
operation sequences; tables, slots, copy pairs and counters must agree.
The waste counters are also checked against the oracle's accounting and the
pages' worked example.
"""
import numpy as np
import pytest

import oracle
from oracle_pins import read_golden_kv
from paged_kv_cache_323_b200 import build as pkv_build


@pytest.fixture(scope="module")
def pk():
    pkv_build.build()
    from paged_kv_cache_323_b200 import pagedkv

    return pagedkv


class ModelBM:
    """Plain model of the rules; free blocks are handed out in `order`, released ones first."""

    def __init__(self, num_blocks, bs, order):
        self.bs = bs
        self.free = list(reversed(list(order)))  # pop() takes the next
        self.ref = [0] * num_blocks
        self.seqs = {}

    def take(self):
        b = self.free.pop()
        self.ref[b] = 1
        return b

    def release(self, b):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def add(self, sid):
        self.seqs[sid] = {"blocks": [], "len": 0}

    def fork(self, parent, sid):
        p = self.seqs[parent]
        for b in p["blocks"]:
            self.ref[b] += 1
        self.seqs[sid] = {"blocks": list(p["blocks"]), "len": p["len"]}

    def append(self, sid, n):
        s = self.seqs[sid]
        bs = self.bs
        need = -(-(s["len"] + n) // bs)
        cow = s["len"] % bs != 0 and self.ref[s["blocks"][-1]] > 1
        if need - len(s["blocks"]) + (1 if cow else 0) > len(self.free):
            return None
        pairs = []
        if cow:
            src = s["blocks"][-1]
            dst = self.take()
            self.release(src)
            s["blocks"][-1] = dst
            pairs.append((src, dst))
        while len(s["blocks"]) < need:
            s["blocks"].append(self.take())
        slots = [s["blocks"][t // bs] * bs + t % bs for t in range(s["len"], s["len"] + n)]
        s["len"] += n
        return slots, pairs

    def free_seq(self, sid):
        for b in self.seqs.pop(sid)["blocks"]:
            self.release(b)


def test_worked_example_counters(pk):
    """35 tokens in 16-token blocks: 3 blocks, 48 allocated slots, 13 unused."""
    gold = read_golden_kv("worked_example_unused_block_space.txt")
    bm = pk.BlockManager(10, gold["block_size"])
    s = bm.add_sequence()
    slots, pairs = bm.append(s, gold["sequence_length"])
    st = bm.stats()
    assert st["used_blocks"] == gold["blocks"]
    assert st["allocated_slots"] == gold["allocated_slots"]
    assert st["allocated_slots"] - st["used_slots"] == gold["unused_slots"]
    assert len(pairs) == 0 and len(slots) == 35


def test_on_demand_allocation(pk):
    """A new block only when the last one is full."""
    bm = pk.BlockManager(8, 4)
    s = bm.add_sequence()
    seen = []
    for _ in range(9):
        bm.append(s, 1)
        seen.append(bm.stats()["used_blocks"])
    assert seen == [1, 1, 1, 1, 2, 2, 2, 2, 3]


def test_parallel_sampling_copy_on_write(pk):
    """Four samples of a 10-token prompt (bs 4): every writer but the last
    holder copies the shared partial block; full prompt blocks stay shared."""
    bm = pk.BlockManager(32, 4, free_order=np.arange(32))
    p = bm.add_sequence()
    bm.append(p, 10)  # blocks 0, 1, 2 (the last holds 2 tokens)
    kids = [bm.fork(p) for _ in range(3)]
    samples = [p] + kids
    pairs_all = []
    for s in samples:
        slots, pairs = bm.append(s, 3)
        pairs_all.append(pairs)
    assert [len(x) for x in pairs_all] == [1, 1, 1, 0]  # the last holder writes in place
    assert [tuple(x[0]) for x in pairs_all[:3]] == [(2, 3), (2, 5), (2, 7)]
    bt, lens = bm.tables(samples, 4)
    assert lens.tolist() == [13] * 4
    assert bt[:, :2].tolist() == [[0, 1]] * 4  # full prompt blocks still shared
    assert bt[3, 2] == 2  # the last holder kept the original partial block
    st = bm.stats()
    assert st["copy_on_write"] == 3
    a, u = oracle.waste_physical(bt, lens, 4, 32)
    assert (st["allocated_slots"], st["allocated_slots"] - st["used_slots"]) == (a, u)


def test_free_and_reuse(pk):
    bm = pk.BlockManager(6, 8, free_order=[5, 4, 3, 2, 1, 0])
    a = bm.add_sequence()
    bm.append(a, 20)  # blocks 5, 4, 3
    b = bm.fork(a)
    bm.free(a)
    assert bm.stats()["free_blocks"] == 3  # still referenced by b
    bm.free(b)
    assert bm.stats()["free_blocks"] == 6
    c = bm.add_sequence()
    slots, _ = bm.append(c, 1)
    assert slots[0] // 8 == 3  # released blocks are reused first, the last released first


def test_out_of_blocks_changes_nothing(pk):
    bm = pk.BlockManager(3, 4)
    s = bm.add_sequence()
    bm.append(s, 10)
    before = bm.stats()
    with pytest.raises(pk.PagedKVError) as e:
        bm.append(s, 5)
    assert e.value.status == pk.PKV_ERR_OUT_OF_BLOCKS
    assert bm.stats() == before and bm.length(s) == 10


def test_victim_and_swap_round_trip(pk):
    bm = pk.BlockManager(16, 4, num_host_blocks=8)
    ids = [bm.add_sequence() for _ in range(3)]
    for i, s in enumerate(ids):
        bm.append(s, 5 + i)
    victim = bm.pick_victim()
    assert victim == ids[-1]  # most recently arrived first
    bt_before, _ = bm.tables([victim], 4)
    out_pairs = bm.swap_out(victim)
    assert [int(x) for x in out_pairs[:, 0]] == [int(x) for x in bt_before[0, :2]]
    st = bm.stats()
    assert st["swapped_sequences"] == 1 and st["preemptions"] == 1 and st["host_free_blocks"] == 6
    assert bm.pick_victim() == ids[1]
    in_pairs = bm.swap_in(victim)
    assert in_pairs[:, 0].tolist() == out_pairs[:, 1].tolist()
    assert bm.length(victim) == 7 and bm.stats()["host_free_blocks"] == 8


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_against_model(pk, seed):
    """Random add / fork / append / free sequences agree with the model."""
    rng = np.random.default_rng(seed)
    nblk, bs = 200, int(rng.choice([4, 8, 16]))
    order = rng.permutation(nblk)
    bm = pk.BlockManager(nblk, bs, free_order=order)
    model = ModelBM(nblk, bs, order)
    live = []
    for _ in range(300):
        op = rng.random()
        if op < 0.15 or not live:
            sid = bm.add_sequence()
            model.add(sid)
            live.append(sid)
        elif op < 0.3:
            parent = int(rng.choice(live))
            sid = bm.fork(parent)
            model.fork(parent, sid)
            live.append(sid)
        elif op < 0.85:
            sid = int(rng.choice(live))
            n = int(rng.integers(1, 3 * bs))
            expect = model.append(sid, n)
            if expect is None:
                with pytest.raises(pk.PagedKVError):
                    bm.append(sid, n)
                continue
            slots, pairs = bm.append(sid, n)
            assert slots.tolist() == expect[0]
            assert [tuple(int(v) for v in p) for p in pairs] == expect[1]
        else:
            sid = int(rng.choice(live))
            bm.free(sid)
            model.free_seq(sid)
            live.remove(sid)
        if live:
            maxb = max(len(model.seqs[s]["blocks"]) for s in live) + 1
            bt, lens = bm.tables(live, maxb)
            for i, s in enumerate(live):
                nb = len(model.seqs[s]["blocks"])
                assert bt[i, :nb].tolist() == model.seqs[s]["blocks"]
                assert lens[i] == model.seqs[s]["len"]
            st = bm.stats()
            a, u = oracle.waste_physical(bt, lens, bs, nblk)
            assert st["allocated_slots"] == a and st["allocated_slots"] - st["used_slots"] == u
            assert st["free_blocks"] == len(model.free)


def test_bad_arguments(pk):
    L = pk.lib
    assert not L.pkv_bm_create(0, 16, 0, None)
    bad_order = np.array([0, 0, 1], dtype=np.int32)
    assert not L.pkv_bm_create(3, 16, 0, bad_order.ctypes.data)
    bm = pk.BlockManager(4, 16)
    with pytest.raises(pk.PagedKVError):
        bm.fork(7)
    with pytest.raises(pk.PagedKVError):
        bm.free(0)
