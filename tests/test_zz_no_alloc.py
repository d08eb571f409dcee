"""paged_attention_decode_noalloc, the entry point for callers that cannot
allocate device memory (a KV pool that already fills the GPU, a host
framework that only allows its own allocator, or a decode loop that cannot
afford cudaMalloc's synchronisation).  Its split-K scratch is a fixed array
inside the library, so these tests check, through the C ABI, that two calls
in a row give exactly what paged_attention_decode_ex gives with a caller
workspace (the same kernel with the same reduction order, so bit for bit),
that the no-alloc path alone meets the oracle's bar, and that a batch too
large for the fixed scratch is refused.

The file name makes pytest collect it last; it needs no state from the
other tests and also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_323_b200 import workload as wl
from steps import BF16_ATOL, BF16_RTOL, oracle_step, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", ["mha_bf16", "gqa_bf16", "tiny_f32"])
def test_noalloc_matches_ex_twice(case):
    from paged_kv_cache_323_b200 import pagedkv as pk

    if case == "mha_bf16":
        w, pt = wl.mha(num_seqs=8, num_blocks=2048), 0  # 4 partitions per long sequence
    elif case == "gqa_bf16":
        w, pt = wl.gqa_sampling(groups=4, prompt_median=400, prompt_max=3000), 256
    else:
        w, pt = wl.tiny(), 16
    t = to_device(w)
    if len(w.cow_pairs):
        pk.copy_blocks(t["k_cache"], t["v_cache"], t["cow_pairs"])
    pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"], t["v_new"], t["slot_mapping"])
    need = pk.paged_attention_workspace_size(w.num_seqs, w.num_heads,
                                             w.max_blocks_per_seq * w.block_size, w.head_dim, pt)
    assert 0 < need <= pk.NOALLOC_SCRATCH_BYTES  # the case really uses split-K scratch
    ref = torch.empty_like(t["q"])
    pk.paged_attention_decode_ex(ref, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                 t["context_lens"], w.scale, num_blocks=w.num_blocks,
                                 partition_tokens=pt,
                                 workspace=torch.zeros(need, dtype=torch.uint8, device="cuda"))
    outs = []
    for _ in range(2):  # the second call sees the scratch the first one left
        o = torch.full_like(t["q"], float("nan"))
        pk.paged_attention_decode_noalloc(o, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                          t["context_lens"], w.scale, num_blocks=w.num_blocks,
                                          partition_tokens=pt)
        outs.append(o)
    torch.cuda.synchronize()
    assert pk.get_device_error() == 0
    for o in outs:
        assert torch.isfinite(o.float()).all()
        assert torch.equal(o, ref)  # same kernel, same reduction order: bit-identical


def test_noalloc_against_oracle():
    """The no-alloc path on its own also meets the oracle bar."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.long_context(num_seqs=2, ctx_range=(3000, 9000))
    ref, _, _ = oracle_step(w)
    t = to_device(w)
    pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"], t["v_new"], t["slot_mapping"])
    for _ in range(2):
        pk.paged_attention_decode_noalloc(t["out"], t["q"], t["k_cache"], t["v_cache"],
                                          t["block_tables"], t["context_lens"], w.scale,
                                          num_blocks=w.num_blocks, partition_tokens=512)
        torch.cuda.synchronize()
        got = t["out"].double().cpu().numpy()
        assert np.all(np.abs(got - ref) <= BF16_ATOL + BF16_RTOL * np.abs(ref))


def test_noalloc_refuses_oversize():
    """A batch whose scratch exceeds the fixed array is refused before any launch."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    B, H, D, bs, maxb = 64, 64, 128, 16, 4096  # 65536-token tables at 512-token partitions
    assert pk.paged_attention_workspace_size(B, H, maxb * bs, D, 512) > pk.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, H, D, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, 8, bs, D, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(B, maxb, dtype=torch.int32, device="cuda")
    ctx = torch.zeros(B, dtype=torch.int32, device="cuda")
    n0 = pk.launch_count()
    with pytest.raises(pk.PagedKVError) as e:
        pk.paged_attention_decode_noalloc(torch.empty_like(q), q, kc, kc, bt, ctx, 0.1,
                                          partition_tokens=512)
    assert e.value.status == pk.PKV_ERR_WORKSPACE
    assert pk.launch_count() == n0
