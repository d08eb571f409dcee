"""The multi-GPU plan on CPU: world size 2 over gloo.

The decode path shards by sequence with no data-path exchange, so each rank
owns its own batch (weak scaling).  These tests run the host logic of
bench.py on two gloo ranks: distinct per-rank batches, the MAX all-reduce of
the timed region, the whole-job value, and that a rank's shard computed
alone equals the same sequences inside a merged batch (the oracle, fp64).
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_path):
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    import oracle
    from paged_kv_cache_323_b200 import workload as wl

    seed = bench.rank_seed("mha", rank)
    w = wl.mha(seed=seed, num_seqs=3, num_blocks=400, heads=4, ctx_range=(40, 300))
    # each rank's step on its own shard (the oracle stands in for the GPU here)
    from steps import oracle_step

    out, _, _ = oracle_step(w)
    local_ms = 10.0 + rank  # rank 1 is the slower one
    ms = bench.max_over_ranks(world, local_ms)
    # the timed region's repeat count: every rank runs the same number (the
    # largest any rank needs), here 0.5 s of 1 ms regions on rank 0 and of
    # 2 ms regions on rank 1, so 500 capped at 200 on both
    reps = bench.repeat_count(world, 1.0 + rank, 0.5)
    reps_small = bench.repeat_count(world, 100.0 * (rank + 1), 0.5)  # 5 on rank 0, 3 on rank 1
    value = bench.job_value(world, w.kv_bytes_logical(), ms)
    gathered = [None] * world
    dist.all_gather_object(gathered, (seed, float(out.sum()), w.kv_bytes_logical(), reps, reps_small))
    if rank == 0:
        torch.save({"ms": ms, "value": value, "gathered": gathered}, out_path)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    out_path = str(tmp_path / "r.pt")
    mp.spawn(_worker, args=(2, _free_port(), out_path), nprocs=2, join=True)
    r = torch.load(out_path)
    assert r["ms"] == 11.0  # the slowest rank decides
    (s0, sum0, b0, n0, m0), (s1, sum1, b1, n1, m1) = r["gathered"]
    assert s0 != s1 and sum0 != sum1  # distinct batches per rank
    assert n0 == n1 == 200 and m0 == m1 == 5  # ranks agree on the timed regions they run
    assert abs(r["value"] - 2 * b0 / 11e-3 / 1e9) < 1e-9  # weak scaling: world x bytes / max time


def test_shard_equals_merged_batch():
    """A sequence's output does not depend on which other sequences share its
    batch, so splitting a batch across ranks by sequence needs no exchange."""
    import oracle
    from paged_kv_cache_323_b200 import workload as wl
    from steps import oracle_step, subset

    w = wl.mha(seed=9, num_seqs=4, num_blocks=500, heads=4, ctx_range=(40, 300))
    full, _, _ = oracle_step(w)
    for shard in ([0, 1], [2, 3]):
        part, _, _ = oracle_step(subset(w, shard))
        assert np.array_equal(part, full[shard])
