"""The split-K workspace across calls: a decode whose bounded waits run out
must leave the workspace valid for the next call, and one workspace must
serve calls of different shapes ("How PagedAttention works", item 5: the
decode kernel follows the block tables of whatever batch the step has).

The timeout is made, not faked: the library's test hook shortens the limit
of the decode pipeline's waits to a microsecond, far below a load's latency,
so real decode launches give up part-way (PKV_ERR_TIMEOUT), while the wait
that lets a stopped CTA's own copies land keeps its one-second bound.
Nothing faults or hangs.  The calls that follow, on the same caller
workspace and on the library's own, must then match the oracle.
"""
import pytest
import torch

from paged_kv_cache_323_b200 import workload as wl
from steps import assert_close, oracle_step, to_device

pytestmark = pytest.mark.gpu

KERNELS = {
    # batch-64-like MHA on the staged CUDA-core kernel (bulk copies and
    # mbarrier waits; the register-streamed kernel that serves this shape by
    # default has no waits), 4 partitions per long sequence
    "cuda_core": (lambda: wl.mha(num_seqs=8, num_blocks=2048), 512),
    # grouped-query heads on the tensor-core kernel, several partitions
    "tensor_core": (lambda: wl.gqa_sampling(groups=4, prompt_median=600, prompt_max=3000), 256),
    # fp8 cache on the tensor-core fp8 kernel, one CTA per unit
    "tensor_core_fp8": (lambda: wl.mha(num_seqs=8, num_blocks=2048, dtype="fp8"), 512),
    # the same in persistent form: a stopped CTA also drains the work queue
    "tensor_core_fp8_persistent": (lambda: wl.mha(num_seqs=8, num_blocks=2048, dtype="fp8"), 512),
    # persistent, one partition per sequence: first-wave units in index order, the rest queued
    "tensor_core_fp8_persistent_one_partition": (lambda: wl.mha(num_seqs=64, num_blocks=16384, dtype="fp8"),
                                                 2048),
    # head_dim 64 over an fp8 cache: one CTA per pair of kv heads
    "tensor_core_fp8_d64": (lambda: wl.mha(num_seqs=8, num_blocks=2048, head_dim=64, dtype="fp8"), 512),
}


def _decode(pk, w, t, pt, ws):
    if w.dtype == "fp8":
        ks = torch.from_numpy(w.k_scales).cuda()
        vs = torch.from_numpy(w.v_scales).cuda()
        pk.paged_attention_decode_fp8(t["out"], t["q"], t["k_cache"], t["v_cache"], ks, vs,
                                      t["block_tables"], t["context_lens"], w.scale,
                                      num_blocks=w.num_blocks, partition_tokens=pt, workspace=ws)
    else:
        pk.paged_attention_decode_ex(t["out"], t["q"], t["k_cache"], t["v_cache"],
                                     t["block_tables"], t["context_lens"], w.scale,
                                     num_blocks=w.num_blocks, partition_tokens=pt, workspace=ws)


def _appended(pk, w):
    """Device tensors after the step's copies and append (the decode's input)."""
    t = to_device(w)
    if len(w.cow_pairs):
        pk.copy_blocks(t["k_cache"], t["v_cache"], t["cow_pairs"])
    if w.dtype == "fp8":
        pk.kv_cache_append_fp8(t["k_cache"], t["v_cache"], torch.from_numpy(w.k_scales).cuda(),
                               torch.from_numpy(w.v_scales).cuda(), t["k_new"], t["v_new"],
                               t["slot_mapping"])
    else:
        pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"], t["v_new"], t["slot_mapping"])
    torch.cuda.synchronize()
    return t


def _time_out(pk, run, tries=10):
    """Run `run` with a 1 us pipeline wait limit until a launch reports
    PKV_ERR_TIMEOUT; restore the default.  A launch usually times out, but a
    1 us limit sits near one load's latency and the timer's granularity, so
    several launches in a row can finish in time."""
    assert pk.get_device_error() == 0
    prev = pk.set_wait_limit_us(1)
    try:
        assert prev == 1000000  # the default: one second
        for _ in range(tries):
            run()
            code = pk.get_device_error()
            if code == pk.PKV_ERR_TIMEOUT:
                return
            assert code == 0, code
    finally:
        pk.set_wait_limit_us(0)
    pytest.fail("no decode launch timed out with a 1 us wait limit")


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_timeout_then_parity_on_the_same_workspace(kernel):
    """A stopped CTA still takes its turn on its merge counter, so the
    caller's workspace is valid right after PKV_ERR_TIMEOUT: the next
    decodes on it match the oracle."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    make, pt = KERNELS[kernel]
    prev = pk._set_fp8_persistent(kernel != "tensor_core_fp8")
    prev_reg = pk._set_reg_stream(False)
    try:
        _timeout_then_parity(pk, make(), pt)
    finally:
        pk._set_fp8_persistent(prev)
        pk._set_reg_stream(prev_reg)


def _timeout_then_parity(pk, w, pt):
    ref, _, _ = oracle_step(w)
    t = _appended(pk, w)
    need = pk.paged_attention_workspace_size(w.num_seqs, w.num_heads,
                                             w.max_blocks_per_seq * w.block_size, w.head_dim, pt)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    _time_out(pk, lambda: _decode(pk, w, t, pt, ws))
    assert torch.isfinite(t["out"].float()).all()  # a stopped launch still writes finite rows
    for _ in range(2):
        t["out"].fill_(float("nan"))
        _decode(pk, w, t, pt, ws)
        torch.cuda.synchronize()
        assert pk.get_device_error() == 0
        assert_close(t["out"], ref, "bf16" if w.dtype == "fp8" else w.dtype)


def test_timeout_then_parity_library_workspace():
    """The same through paged_attention_decode, whose workspace the library
    owns: a timed-out call leaves it valid for the next call on the stream."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.mha(num_seqs=8, num_blocks=2048)  # contexts up to 2048: split into 2 partitions
    ref, _, _ = oracle_step(w)
    t = _appended(pk, w)

    def plain():
        pk.paged_attention_decode(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                  t["context_lens"], w.scale)

    prev_reg = pk._set_reg_stream(False)  # the staged kernel, which waits on its copies
    try:
        plain()  # the library's workspace for this stream exists before the timeout
        torch.cuda.synchronize()
        assert pk.get_device_error() == 0
        _time_out(pk, plain)
        for _ in range(2):
            t["out"].fill_(float("nan"))
            plain()
            torch.cuda.synchronize()
            assert pk.get_device_error() == 0
            assert_close(t["out"], ref, w.dtype)
    finally:
        pk._set_reg_stream(prev_reg)


def test_register_kernel_has_no_waits():
    """The register-streamed kernel (bf16 MHA) loads straight into registers
    and waits on nothing: with the 1 us limit its launches never report a
    timeout and still match the oracle."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.mha(num_seqs=8, num_blocks=2048)
    ref, _, _ = oracle_step(w)
    t = _appended(pk, w)
    need = pk.paged_attention_workspace_size(w.num_seqs, w.num_heads,
                                             w.max_blocks_per_seq * w.block_size, w.head_dim, 512)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    assert pk.get_device_error() == 0
    prev = pk.set_wait_limit_us(1)
    try:
        for _ in range(3):
            t["out"].fill_(float("nan"))
            _decode(pk, w, t, 512, ws)
            torch.cuda.synchronize()
            assert pk.get_device_error() == 0
            assert_close(t["out"], ref, w.dtype)
    finally:
        pk.set_wait_limit_us(0)


def _shapes():
    """Three batches whose split-K layouts all differ (sequences, heads,
    partitions), each with its oracle result."""
    ws = [wl.mha(seed=31, num_seqs=64, num_blocks=6000, heads=8),
          wl.mha(seed=32, num_seqs=8, num_blocks=2048, heads=4),
          wl.gqa_sampling(seed=33, groups=4, prompt_median=600, prompt_max=3000)]
    return [(w, oracle_step(w)[0]) for w in ws]


def test_plain_decode_across_batch_shapes():
    """paged_attention_decode at batch 64, then 8, then a grouped-query
    batch, then 64 again, on one stream: the library's workspace serves every
    shape and each result matches the oracle."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    cases = _shapes()
    devs = [_appended(pk, w) for w, _ in cases]
    for i in (0, 1, 2, 0, 1):
        (w, ref), t = cases[i], devs[i]
        t["out"].fill_(float("nan"))
        pk.paged_attention_decode(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                  t["context_lens"], w.scale)
        torch.cuda.synchronize()
        assert pk.get_device_error() == 0
        assert_close(t["out"], ref, w.dtype, what=f"call on shape {i}")


@pytest.mark.parametrize("pt", [0, 256])
def test_ex_one_workspace_across_batch_shapes(pt):
    """One caller workspace, zeroed once, serves decode_ex calls of three
    shapes in turn (and back), each matching the oracle."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    cases = _shapes()
    devs = [_appended(pk, w) for w, _ in cases]
    need = max(pk.paged_attention_workspace_size(w.num_seqs, w.num_heads,
                                                 w.max_blocks_per_seq * w.block_size,
                                                 w.head_dim, pt) for w, _ in cases)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for i in (0, 1, 2, 0, 2, 1):
        (w, ref), t = cases[i], devs[i]
        t["out"].fill_(float("nan"))
        _decode(pk, w, t, pt, ws)
        torch.cuda.synchronize()
        assert pk.get_device_error() == 0
        assert_close(t["out"], ref, w.dtype, what=f"call on shape {i}")


def test_binding_reuses_its_workspace():
    """Calls that pass no workspace reuse one buffer per stream instead of
    allocating one per call."""
    from paged_kv_cache_323_b200 import pagedkv as pk

    w = wl.mha(seed=34, num_seqs=8, num_blocks=2048)
    ref, _, _ = oracle_step(w)
    t = _appended(pk, w)
    for _ in range(3):
        pk.paged_attention_decode_ex(t["out"], t["q"], t["k_cache"], t["v_cache"],
                                     t["block_tables"], t["context_lens"], w.scale,
                                     num_blocks=w.num_blocks, partition_tokens=256)
        torch.cuda.synchronize()
        assert_close(t["out"], ref, w.dtype)
    key = (t["q"].device.index, torch.cuda.current_stream().cuda_stream)
    first = pk._workspaces[key].data_ptr()
    pk.paged_attention_decode_ex(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                 t["context_lens"], w.scale, num_blocks=w.num_blocks,
                                 partition_tokens=256)
    assert pk._workspaces[key].data_ptr() == first
