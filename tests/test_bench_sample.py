"""The sample the oracle arm and the CPU baseline time (bench.compact_subset,
bench.pick_sample) is the same work as those sequences inside the full step:
the oracle on the compact pool gives exactly the full step's output rows,
with copy-on-write pairs, multi-token appends and an fp8 cache."""
import numpy as np
import pytest

import bench
import oracle
from paged_kv_cache_323_b200 import workload as wl
from steps import oracle_step


def _run_sample(sub, scale):
    kc, vc = sub["kc"].copy(), sub["vc"].copy()
    if len(sub["pairs"]):
        oracle.copy_blocks(kc, vc, sub["pairs"])
    if sub["k_scales"] is not None:
        oracle.kv_append_fp8(kc, vc, sub["k_scales"], sub["v_scales"], sub["k_new"], sub["v_new"],
                             sub["slots"])
        return oracle.paged_attention_fp8(sub["q"], kc, vc, sub["k_scales"], sub["v_scales"],
                                          sub["bt"], sub["ctx"], scale)
    oracle.kv_append(kc, vc, sub["k_new"], sub["v_new"], sub["slots"])
    return oracle.paged_attention(sub["q"], kc, vc, sub["bt"], sub["ctx"], scale)


@pytest.mark.parametrize("make", [
    lambda: wl.tiny(),
    lambda: wl.gqa_sampling(groups=3, samples=3, prompt_median=120, prompt_max=300, heads=8,
                            kv_heads=2, head_dim=64),
    lambda: wl.gqa_sampling(groups=3, samples=3, prompt_median=120, prompt_max=300, heads=8,
                            kv_heads=2, head_dim=64, dtype="fp8"),
], ids=["tiny", "gqa_sampling", "gqa_sampling_fp8"])
def test_compact_subset_reproduces_rows(make):
    w = make()
    ref, _, _ = oracle_step(w)
    seqs = sorted({0, w.num_seqs // 2, w.num_seqs - 1})
    sub = bench.compact_subset(w, seqs)
    assert len(sub["pairs"]) == sum(1 for s in w.pair_seq.tolist() if s in seqs)
    if len(w.cow_pairs):
        assert len(sub["pairs"]) > 0  # the sample exercises the copy-on-write remap
    out = _run_sample(sub, w.scale)
    assert np.array_equal(out, ref[seqs])
    kv = int(w.context_lens[seqs].astype(np.int64).sum()) * w.num_kv_heads * w.head_dim * 2 * w.elt
    assert sub["kv_bytes"] == kv


def test_pick_sample_bounds_the_work():
    w = wl.gqa_sampling(groups=4, samples=2, prompt_median=100, prompt_max=200, heads=4,
                        kv_heads=2, head_dim=64)
    sub, n, dt, out = bench.pick_sample(w, target_s=0.0, threads=1)  # any work is enough
    assert n == 1 and len(sub["ctx"]) == 1 and dt >= 0 and out.shape[0] == 1
    sub, n, _, out = bench.pick_sample(w, target_s=1e9, threads=2)  # never enough: every sequence
    assert n == w.num_seqs and len(sub["ctx"]) == w.num_seqs
    # the rows it returns are the oracle's rows of those sequences in the full step
    ref, _, _ = oracle_step(w)
    assert sub["seqs"] == list(range(w.num_seqs)) and np.array_equal(out, ref)


def test_rows_match_bar():
    """The bench's per-row parity verdict applies the parity bars: bf16
    2e-2 + 1e-2 |ref| elementwise, fp32 1e-5 absolute, never a NaN."""
    import torch

    ref = np.zeros((2, 3, 4))
    ok = bench.rows_match(torch.full((2, 3, 4), 0.019, dtype=torch.bfloat16), ref, "bf16")
    assert ok["ok"] and ok["rows"] == 6
    assert not bench.rows_match(torch.full((2, 3, 4), 0.03), ref, "bf16")["ok"]
    assert not bench.rows_match(torch.full((2, 3, 4), 2e-5), ref, "f32")["ok"]
    nan = torch.zeros((2, 3, 4))
    nan[1, 2, 3] = float("nan")
    assert not bench.rows_match(nan, ref, "bf16")["ok"]
