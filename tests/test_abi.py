"""The C-ABI library loads and exports every symbol include/pagedkv.h
declares, and its host-side validation returns the documented status codes
before touching the GPU (no GPU needed: these calls never reach CUDA)."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_323_b200 import build as pkv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


@pytest.fixture(scope="module")
def pk():
    pkv_build.build()
    from paged_kv_cache_323_b200 import pagedkv

    return pagedkv


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^PKV_API\s+[\w\s\*]+?\b(\w+)\(", text, re.M)
    return names


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("paged_attention_decode", "paged_attention_decode_ex", "kv_cache_append",
              "copy_blocks", "pkv_get_device_error", "pkv_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(pk):
    lib = ctypes.CDLL(pk.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared but not exported"
        assert name in pk.SIGNATURES, f"{name} has no binding signature"


FAKE = 0x7F0000001000  # aligned, never dereferenced: validation fails first
MIS = FAKE + 8  # 8-byte aligned only


def _decode(pk, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, ctx=FAKE, B=4, H=8, Hkv=2, D=128, bs=16,
             maxb=8, scale=0.125, nblk=64, dtype=pk.PKV_BF16, pt=0, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return pk.lib.paged_attention_decode_ex(a["out"], a["q"], a["k"], a["v"], a["bt"], a["ctx"],
                                            a["B"], a["H"], a["Hkv"], a["D"], a["bs"], a["maxb"],
                                            a["scale"], a["nblk"], a["dtype"], a["pt"], a["ws"],
                                            a["wsb"], None)


def test_decode_validation(pk):
    assert _decode(pk, B=0, out=None, q=None) == pk.PKV_OK  # no-op
    assert _decode(pk, B=-1) == pk.PKV_ERR_INVALID
    for name in ("out", "q", "k", "v", "bt", "ctx"):
        assert _decode(pk, **{name: None}) == pk.PKV_ERR_NULL, name
    assert _decode(pk, H=6, Hkv=4) == pk.PKV_ERR_INVALID  # heads not a multiple of kv heads
    assert _decode(pk, Hkv=0) == pk.PKV_ERR_INVALID
    assert _decode(pk, D=96) == pk.PKV_ERR_UNSUPPORTED
    assert _decode(pk, bs=12) == pk.PKV_ERR_UNSUPPORTED
    assert _decode(pk, H=6, Hkv=2) == pk.PKV_ERR_UNSUPPORTED  # group of 3
    assert _decode(pk, D=0) == pk.PKV_ERR_INVALID
    assert _decode(pk, maxb=0) == pk.PKV_ERR_INVALID
    assert _decode(pk, nblk=0) == pk.PKV_ERR_INVALID
    assert _decode(pk, dtype=7) == pk.PKV_ERR_INVALID
    assert _decode(pk, scale=float("nan")) == pk.PKV_ERR_INVALID
    assert _decode(pk, pt=24) == pk.PKV_ERR_INVALID  # not a multiple of the block size
    assert _decode(pk, pt=8192) == pk.PKV_ERR_INVALID
    assert _decode(pk, pt=-16) == pk.PKV_ERR_INVALID
    assert _decode(pk, k=MIS) == pk.PKV_ERR_INVALID  # pools must be 16-byte aligned
    assert _decode(pk, q=MIS) == pk.PKV_ERR_INVALID
    # long tables need a split-K workspace
    assert _decode(pk, maxb=200, ws=None, wsb=0) == pk.PKV_ERR_WORKSPACE
    assert _decode(pk, maxb=200, wsb=16) == pk.PKV_ERR_WORKSPACE
    assert _decode(pk, maxb=200, ws=FAKE + 16) == pk.PKV_ERR_WORKSPACE  # not 256-aligned


def test_workspace_size(pk):
    ws = pk.paged_attention_workspace_size
    one = ws(4, 8, 512, 128, 0)  # one partition: the merge counters' region and the schedule
    assert one == ws(4, 8, 512, 128, 512) and one >= 65536 * 4 + 4 * 4
    n = ws(4, 8, 513, 128, 0)  # two partitions: plus the partial results
    assert n >= one + 4 * 8 * 2 * (128 + 2) * 4
    assert ws(4, 8, 4096, 128, 256) >= 4 * 8 * 16 * 128 * 4
    assert ws(0, 8, 4096, 128, 0) == 0
    # the counters' region grows with batches of more than 65536 (sequence, head) units
    assert ws(1024, 128, 512, 128, 0) >= 1024 * 128 * 4


def test_append_and_copy_validation(pk):
    L = pk.lib
    assert L.kv_cache_append(None, None, None, None, None, 0, 8, 128, 16, 10, 1, None) == pk.PKV_OK
    assert L.kv_cache_append(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 8, 128, 16, 10, 1, None) == pk.PKV_ERR_INVALID
    assert L.kv_cache_append(FAKE, None, FAKE, FAKE, FAKE, 3, 8, 128, 16, 10, 1, None) == pk.PKV_ERR_NULL
    assert L.kv_cache_append(FAKE, FAKE, FAKE, FAKE, FAKE, 3, 8, 4, 16, 10, 1, None) == pk.PKV_ERR_UNSUPPORTED
    assert L.kv_cache_append(FAKE, FAKE, MIS, FAKE, FAKE, 3, 8, 128, 16, 10, 1, None) == pk.PKV_ERR_INVALID
    assert L.kv_cache_append(FAKE, FAKE, FAKE, FAKE, FAKE, 3, 8, 128, 16, 10, 5, None) == pk.PKV_ERR_INVALID
    assert L.copy_blocks(None, None, None, 0, 8, 128, 16, 10, 1, None) == pk.PKV_OK
    assert L.copy_blocks(FAKE, FAKE, None, 2, 8, 128, 16, 10, 1, None) == pk.PKV_ERR_NULL
    assert L.copy_blocks(FAKE, FAKE, FAKE, -2, 8, 128, 16, 10, 1, None) == pk.PKV_ERR_INVALID
    assert L.copy_blocks(FAKE, FAKE, FAKE, 2, 0, 128, 16, 10, 1, None) == pk.PKV_ERR_INVALID


def test_status_strings_and_version(pk):
    for code in range(0, -9, -1):
        assert pk.status_string(code) and pk.status_string(code) != "unknown status"
    assert pk.status_string(-99) == "unknown status"
    assert pk.lib.pkv_version() == 100
    assert pk.lib.pkv_get_device_error(None, None) == pk.PKV_ERR_NULL


def test_noalloc_validation(pk):
    """The fixed-scratch entry point refuses oversize batches before touching the GPU."""
    L = pk.lib
    args = [FAKE] * 6
    assert L.paged_attention_decode_noalloc(*args, 0, 8, 2, 128, 16, 8, 0.1, 64, 1, 0, None) == pk.PKV_OK
    assert L.paged_attention_decode_noalloc(*args, -1, 8, 2, 128, 16, 8, 0.1, 64, 1, 0, None) == pk.PKV_ERR_INVALID
    # 64 sequences x 64 heads x 128 partitions x 128 dims of fp32 partials >> 16 MiB
    assert L.paged_attention_decode_noalloc(*args, 64, 64, 8, 128, 16, 4096, 0.1, 64, 1, 512,
                                            None) == pk.PKV_ERR_WORKSPACE


def test_partition_tokens(pk):
    pt = pk.paged_attention_partition_tokens
    bf = pk.PKV_BF16
    assert pt(64, 32, 32, 128, 16, 2048, bf, 0) == 1024  # batch-64 MHA, CUDA-core kernel
    # tokens of at most 256 bytes per kv head (here bf16 at head_dim 64): twice as long
    assert pt(64, 32, 32, 64, 16, 2048, bf, 0) == 2048
    assert pt(4, 8, 8, 64, 16, 64, pk.PKV_F32, 0) == 1024  # fp32 at head_dim 64: 512-byte tokens
    assert pt(64, 32, 32, 128, 16, 2048, bf, 256) == 256  # explicit sizes pass through
    # grouped-query heads on the tensor-core kernel: long partitions unless the grid gets small
    assert pt(256, 32, 8, 128, 16, 8256, bf, 0) == 4096
    assert pt(8, 64, 8, 128, 32, 131072, bf, 0) == 4096  # 2048 CTAs: still 4 waves
    assert pt(1, 32, 8, 128, 16, 1024, bf, 0) == 512
    # fp8 caches: the tensor-core kernel for MHA too, in persistent form, whose
    # partitions hold at most 128 blocks
    f8 = pk.PKV_FP8_E4M3
    assert pt(64, 32, 32, 128, 16, 2048, f8, 0) == 2048
    assert pt(8, 64, 8, 128, 32, 131072, f8, 0) == 4096
    assert pt(64, 32, 32, 128, 8, 2048, f8, 0) == 1024
    # head_dim 64: one CTA per pair of kv heads, partitions halved until one wave
    assert pt(64, 32, 32, 64, 16, 2048, f8, 0) == 4096
    assert pt(8, 32, 32, 64, 16, 2048, f8, 0) == 512
    prev = pk._set_fp8_persistent(False)
    try:
        assert pt(64, 32, 32, 128, 16, 2048, f8, 0) == 4096  # one CTA per unit
    finally:
        pk._set_fp8_persistent(prev)
    prev = pk.set_tensor_core_gqa(False)
    try:
        big = pt(8, 64, 8, 128, 32, 131072, bf, 0)  # CUDA-core kernel: fewer, larger partitions
        assert 1024 < big <= 4096 and 131072 // big <= 64
    finally:
        pk.set_tensor_core_gqa(prev)
    assert pt(0, 8, 8, 128, 16, 1024, bf, 0) == 0
