"""The Python binding's argument checks, on the CPU.

Each wrapper checks device, layout, element type and shape before it hands
raw pointers to the C ABI: a tensor that is not where the kernel expects it
would otherwise be read as device memory.  Here host tensors stand in for
CUDA tensors (they report a CUDA device) and a recording fake stands in for
the library, so the wrappers' host logic runs without a GPU: the shapes the
GPU tests use pass through with the right sizes, and each malformed argument
raises before anything is called.
"""
import contextlib
import types

import numpy as np
import pytest
import torch

from paged_kv_cache_323_b200 import workload as wl


class Dev:
    """A host tensor the binding takes for a CUDA tensor on cuda:<index>."""

    def __init__(self, t, index=0, contiguous=True, cuda=True, pinned=False):
        self.t = t
        self.is_cuda = cuda
        self.device = torch.device("cuda", index) if cuda else torch.device("cpu")
        self._contiguous = contiguous
        self._pinned = pinned

    shape = property(lambda self: self.t.shape)
    dtype = property(lambda self: self.t.dtype)

    def dim(self):
        return self.t.dim()

    def is_contiguous(self):
        return self._contiguous

    def is_pinned(self):
        return self._pinned

    def data_ptr(self):
        return self.t.data_ptr()

    def numel(self):
        return self.t.numel()

    def element_size(self):
        return self.t.element_size()


class FakeLib:
    """Records every call; every entry point returns PKV_OK (0), the
    workspace-size query returns 0."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def f(*args):
            self.calls.append((name, args))
            return 0

        return f


@pytest.fixture
def pk(monkeypatch):
    from paged_kv_cache_323_b200 import pagedkv

    fake = FakeLib()
    monkeypatch.setattr(pagedkv, "lib", fake)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_stream",
                        lambda device=None: types.SimpleNamespace(cuda_stream=0))
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(pagedkv, "fake", fake, raising=False)
    return pagedkv


def _step_tensors(dtype="bf16"):
    w = wl.custom(3, [35, 16, 1, 50], heads=8, kv_heads=2, head_dim=64, block_size=16,
                  dtype=dtype)
    pools = (w.k_cache, w.v_cache)
    if dtype == "fp8":
        pools = tuple(p.view(torch.float8_e4m3fn) for p in pools)
    t = {
        "q": Dev(w.q), "out": Dev(torch.empty_like(w.q)), "k_cache": Dev(pools[0]),
        "v_cache": Dev(pools[1]), "k_new": Dev(w.k_new), "v_new": Dev(w.v_new),
        "bt": Dev(torch.from_numpy(w.block_tables)), "ctx": Dev(torch.from_numpy(w.context_lens)),
        "slots": Dev(torch.from_numpy(w.slot_mapping)), "pairs": Dev(torch.from_numpy(w.cow_pairs)),
    }
    if dtype == "fp8":
        t["ks"] = Dev(torch.from_numpy(w.k_scales))
        t["vs"] = Dev(torch.from_numpy(w.v_scales))
    return w, t


def test_decode_ex_passes_sizes(pk):
    w, t = _step_tensors()
    ws = Dev(torch.zeros(4096, dtype=torch.uint8))
    pk.paged_attention_decode_ex(t["out"], t["q"], t["k_cache"], t["v_cache"], t["bt"], t["ctx"],
                                 w.scale, num_blocks=w.num_blocks, workspace=ws)
    name, args = pk.fake.calls[-1]
    assert name == "paged_attention_decode_ex"
    assert args[:4] == (t["out"].data_ptr(), t["q"].data_ptr(), t["k_cache"].data_ptr(),
                        t["v_cache"].data_ptr())
    assert args[6:12] == (w.num_seqs, 8, 2, 64, 16, w.max_blocks_per_seq)
    assert args[13:] == (w.num_blocks, pk.PKV_BF16, 0, ws.data_ptr(), 4096, 0)


def test_every_wrapper_accepts_the_test_shapes(pk):
    w, t = _step_tensors()
    pk.copy_blocks(t["k_cache"], t["v_cache"], t["pairs"])
    pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"], t["v_new"], t["slots"])
    pk.paged_attention_decode(t["out"], t["q"], t["k_cache"], t["v_cache"], t["bt"], t["ctx"],
                              w.scale)
    pk.paged_attention_decode_noalloc(t["out"], t["q"], t["k_cache"], t["v_cache"], t["bt"],
                                      t["ctx"], w.scale)
    # empty calls: a zero-length batch, no tokens, no pairs
    empty = Dev(torch.empty(0, dtype=torch.int64))
    pk.kv_cache_append(t["k_cache"], t["v_cache"], Dev(w.k_new[:0]), Dev(w.v_new[:0]), empty)
    pk.copy_blocks(t["k_cache"], t["v_cache"], Dev(torch.empty(0, 2, dtype=torch.int64)))
    pk.paged_attention_decode_ex(Dev(w.q[:0].clone()), Dev(w.q[:0]), t["k_cache"], t["v_cache"],
                                 Dev(torch.from_numpy(w.block_tables[:0])),
                                 Dev(torch.from_numpy(w.context_lens[:0])), w.scale)
    wf, f = _step_tensors("fp8")
    pk.kv_cache_append_fp8(f["k_cache"], f["v_cache"], f["ks"], f["vs"], f["k_new"], f["v_new"],
                           f["slots"])
    pk.paged_attention_decode_fp8(f["out"], f["q"], f["k_cache"], f["v_cache"], f["ks"], f["vs"],
                                  f["bt"], f["ctx"], wf.scale, num_blocks=wf.num_blocks)
    calls = [c for c in pk.fake.calls if c[0] != "paged_attention_workspace_size"]
    assert [c[0] for c in calls] == [
        "copy_blocks", "kv_cache_append", "paged_attention_decode", "paged_attention_decode_noalloc",
        "kv_cache_append", "copy_blocks", "paged_attention_decode_ex", "kv_cache_append_fp8",
        "paged_attention_decode_fp8"]
    # empty calls hand the library no pointers for the empty arrays
    assert calls[4][1][2:5] == (None, None, None) and calls[4][1][5] == 0  # append: k, v, slots
    assert calls[5][1][2] is None and calls[5][1][3] == 0  # copy: pairs
    assert calls[6][1][6] == 0  # decode: no sequences


def test_swap_accepts_pinned_host_pools(pk):
    dk = Dev(torch.zeros(6, 2, 16, 64, dtype=torch.bfloat16))
    hk = Dev(torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16), cuda=False, pinned=True)
    pairs = Dev(torch.tensor([[1, 0], [5, 3]], dtype=torch.int64))
    pk.swap_blocks(hk, hk, dk, dk, pairs)
    name, args = pk.fake.calls[-1]
    assert name == "swap_blocks" and args[5:12] == (2, 2, 64, 16, 6, 4, pk.PKV_BF16)
    host_pairs = Dev(pairs.t, cuda=False, pinned=True)
    pk.swap_blocks(dk, dk, hk, hk, host_pairs)
    with pytest.raises(ValueError, match="pinned"):
        pk.swap_blocks(Dev(hk.t, cuda=False), hk, dk, dk, pairs)  # pageable host pool
    with pytest.raises(ValueError, match="shape"):
        pk.swap_blocks(hk, hk, dk, dk, Dev(torch.zeros(2, 3, dtype=torch.int64)))


@pytest.mark.parametrize("case", [
    "workspace_on_host", "workspace_dtype", "other_device", "non_contiguous", "ctx_length",
    "table_rows", "table_dims", "out_shape", "stream_device",
])
def test_decode_rejects(pk, monkeypatch, case):
    w, t = _step_tensors()
    kw = dict(num_blocks=w.num_blocks)
    args = [t["out"], t["q"], t["k_cache"], t["v_cache"], t["bt"], t["ctx"], w.scale]
    exc = ValueError
    if case == "workspace_on_host":
        kw["workspace"] = Dev(torch.zeros(4096, dtype=torch.uint8), cuda=False)
    elif case == "workspace_dtype":
        kw["workspace"] = Dev(torch.zeros(1024, dtype=torch.float32))
        exc = TypeError
    elif case == "other_device":
        args[2] = Dev(args[2].t, index=1)
    elif case == "non_contiguous":
        args[1] = Dev(args[1].t, contiguous=False)
    elif case == "ctx_length":
        args[5] = Dev(torch.from_numpy(w.context_lens[:-1]))
    elif case == "table_rows":
        args[4] = Dev(torch.from_numpy(w.block_tables[:-1]))
    elif case == "table_dims":
        args[4] = Dev(torch.from_numpy(w.block_tables.reshape(-1)))
    elif case == "out_shape":
        args[0] = Dev(torch.empty(w.num_seqs, 8, 32, dtype=torch.bfloat16))
    elif case == "stream_device":
        class Stream:  # a stream of another device
            device = torch.device("cuda", 1)
            cuda_stream = 7

        monkeypatch.setattr(torch.cuda, "Stream", Stream)
        kw["stream"] = Stream()
    with pytest.raises(exc):
        pk.paged_attention_decode_ex(*args, **kw)
    assert [c for c in pk.fake.calls if c[0] == "paged_attention_decode_ex"] == []


@pytest.mark.parametrize("case", ["scales_length", "scales_dtype", "k_new_shape"])
def test_fp8_rejects(pk, case):
    w, f = _step_tensors("fp8")
    ks, vs, k_new = f["ks"], f["vs"], f["k_new"]
    exc = ValueError
    if case == "scales_length":
        ks = Dev(torch.from_numpy(np.ones(1, np.float32)))
    elif case == "scales_dtype":
        vs = Dev(torch.from_numpy(w.v_scales.astype(np.float64)))
        exc = TypeError
    elif case == "k_new_shape":
        k_new = Dev(w.k_new[:, :1])
    with pytest.raises(exc):
        pk.kv_cache_append_fp8(f["k_cache"], f["v_cache"], ks, vs, k_new, f["v_new"], f["slots"])
    if case != "k_new_shape":
        with pytest.raises(exc):
            pk.paged_attention_decode_fp8(f["out"], f["q"], f["k_cache"], f["v_cache"], ks, vs,
                                          f["bt"], f["ctx"], w.scale)
    assert pk.fake.calls == []


def test_append_and_copy_reject(pk):
    w, t = _step_tensors()
    with pytest.raises(ValueError):  # one slot short
        pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"], t["v_new"],
                           Dev(torch.from_numpy(np.ascontiguousarray(w.slot_mapping[:-1]))))
    with pytest.raises(ValueError):  # pairs not [n][2]
        pk.copy_blocks(t["k_cache"], t["v_cache"], Dev(torch.zeros(3, dtype=torch.int64)))
    with pytest.raises(ValueError):  # pools of different shapes
        pk.copy_blocks(t["k_cache"], Dev(t["v_cache"].t[:-1]), t["pairs"])
    with pytest.raises(ValueError):  # a pool on another device
        pk.kv_cache_append(t["k_cache"], Dev(t["v_cache"].t, index=1), t["k_new"], t["v_new"],
                           t["slots"])
    assert pk.fake.calls == []
