"""fp8 (e4m3) KV cache on the GPU against the oracle: the quantising append
is bit-exact (codes), and decode attention over the dequantised cache meets
the bf16 bar (the oracle computes on exactly the same fp8 values)."""
import pytest
import torch

from paged_kv_cache_323_b200 import workload as wl
from steps import assert_close, assert_pool_equal, full_size_check, gpu_step, oracle_step

pytestmark = pytest.mark.gpu


def _full_check(w, partition_tokens=0):
    ref, kref, vref = oracle_step(w)
    out, kc, vc = gpu_step(w, partition_tokens=partition_tokens)
    assert_pool_equal(kc, kref, "k pool (codes)")
    assert_pool_equal(vc, vref, "v pool (codes)")
    return assert_close(out, ref, "bf16")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_fp8_shape_grid(D, bs, G):
    lens = [1, bs - 1, bs, 3 * bs + 5, 700, 1111]
    w = wl.custom(300 + G, lens, heads=2 * G, kv_heads=2, head_dim=D, block_size=bs, dtype="fp8",
                  maxb=-(-1111 // bs) + 2)
    _full_check(w, partition_tokens=256)


def test_fp8_mha_reduced():
    w = wl.mha(num_seqs=8, num_blocks=2048, dtype="fp8")
    _full_check(w)


def test_fp8_gqa_sampling_reduced():
    """Copy-on-write copies fp8 blocks byte for byte, then the append quantises."""
    w = wl.gqa_sampling(groups=4, prompt_median=300, prompt_max=1500, dtype="fp8")
    assert len(w.cow_pairs) > 0
    _full_check(w)


def test_fp8_mha_full():
    """The batch-64 MHA step with an fp8 cache: all 64 x 32 rows, codes bit-exact."""
    full_size_check(wl.mha(device="cuda", dtype="fp8"))


def test_fp8_head_dim_64_full():
    """The batch-64 MHA step with head_dim 64 over an fp8 cache (the
    tensor-core kernel on kv head pairs): every row."""
    full_size_check(wl.mha(device="cuda", head_dim=64, dtype="fp8"))


def test_fp8_saturates_large_values():
    """New tokens far beyond the e4m3 range store +-448 codes, as the oracle does."""
    w = wl.custom(5, [40, 17], heads=4, kv_heads=2, head_dim=128, block_size=16, dtype="fp8")
    w.k_new = (w.k_new.float() * 1e4).to(torch.bfloat16)
    _full_check(w)


@pytest.mark.parametrize("q_pow2", [-30, 20, 60])
def test_fp8_query_magnitudes(q_pow2):
    """Queries far outside f16's range, or deep below it, with the softmax
    scale compensating: the logits, and so the outputs, are those of the
    unscaled query.  One dimension is also made 2^12 times larger than the
    rest, so small elements of a head sit far below its largest."""
    w = wl.custom(21, [1, 37, 300, 999], heads=8, kv_heads=2, head_dim=128, block_size=16,
                  dtype="fp8")
    q = w.q.float()
    q[:, :, 5] *= 2.0 ** 12
    w.q = (q * 2.0 ** q_pow2).to(torch.bfloat16)
    w.scale = w.scale * 2.0 ** -(q_pow2 + 12)
    _full_check(w)
