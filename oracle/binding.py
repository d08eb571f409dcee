"""ctypes wrapper around ``pkv_oracle.c`` (test infrastructure only).

Arrays are passed as numpy buffers.  bf16 data is passed as its raw 16-bit
patterns (``uint16``); the C side widens each value to double exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

ORACLE_F32 = 0
ORACLE_BF16 = 1
ORACLE_FP8 = 2  # e4m3 codes (uint8): byte moves only; attention has its own fp8 entry

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB = os.path.join(_HERE, "libpkv_oracle.so")
_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _LIB


def compile_source(src: str, out: str) -> str:
    """Compile an oracle source file with gcc (no fast-math, no FMA contraction)."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared",
         "-fPIC", "-o", tmp, src, "-lpthread", "-lm"]
    )
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def open_library(path: str):
    """Load an oracle build and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_blocks_needed.argtypes = [i64, i64]
    lib.oracle_blocks_needed.restype = i64
    lib.oracle_waste_per_sequence.argtypes = [P, i32, i32, P, P]
    lib.oracle_waste_physical.argtypes = [P, P, i32, i32, i32, i32, P, P]
    lib.oracle_gather.argtypes = [P, P, i32, P, i32, i32, i32, i32, i32, i32, i32]
    lib.oracle_paged_attention.argtypes = [
        P, P, P, P, i32, P, P, i32, i32, i32, i32, i32, i32, dbl, P, i32, i32]
    lib.oracle_paged_attention.restype = i32
    lib.oracle_kv_append.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32]
    lib.oracle_copy_blocks.argtypes = [P, P, P, i32, i32, i32, i32, i32]
    lib.oracle_swap_blocks.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32]
    lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_value.restype = dbl
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_kv_append_fp8.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32]
    lib.oracle_paged_attention_fp8.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                               i32, dbl]
    lib.oracle_paged_attention_fp8.restype = i32
    return lib


_override = None  # a mutant build loaded by the tests that check the pins


def use_library(lib) -> None:
    """Route the module functions to ``lib`` (None restores the real build)."""
    global _override
    _override = lib


def _load():
    global _lib
    if _override is not None:
        return _override
    with _lock:
        if _lib is None:
            build()
            _lib = open_library(_LIB)
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return ORACLE_F32
    if a.dtype == np.uint16:
        return ORACLE_BF16
    if a.dtype == np.uint8:
        return ORACLE_FP8
    raise TypeError(f"oracle takes float32 or bf16 bit patterns (uint16), got {a.dtype}")


def blocks_needed(L: int, bs: int) -> int:
    return int(_load().oracle_blocks_needed(L, bs))


def waste_per_sequence(lens, bs: int):
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    a, u = ctypes.c_int64(), ctypes.c_int64()
    _load().oracle_waste_per_sequence(_ptr(lens), len(lens), bs, ctypes.byref(a), ctypes.byref(u))
    return a.value, u.value


def waste_physical(block_tables, lens, bs: int, num_blocks: int):
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    a, u = ctypes.c_int64(), ctypes.c_int64()
    _load().oracle_waste_physical(_ptr(bt), _ptr(lens), len(lens), bt.shape[1], bs, num_blocks,
                                  ctypes.byref(a), ctypes.byref(u))
    return a.value, u.value


def gather(cache: np.ndarray, block_tables, s: int, L: int, g: int) -> np.ndarray:
    """Contiguous [L][head_dim] fp64 view of sequence s, kv head g."""
    cache = np.ascontiguousarray(cache)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    _, hkv, bs, d = cache.shape
    out = np.empty((L, d), dtype=np.float64)
    _load().oracle_gather(_ptr(out), _ptr(cache), _dtype_code(cache), _ptr(bt), s, L, g, hkv, d,
                          bs, bt.shape[1])
    return out


def paged_attention(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                    rows=None, nthreads: int | None = None) -> np.ndarray:
    """fp64 decode attention.  q is [B][H][D]; caches are [N][Hkv][bs][D].

    With ``rows`` (an int array of (s, h) pairs) only those outputs are
    computed and the result is [len(rows)][D]; otherwise [B][H][D]."""
    q = np.ascontiguousarray(q)
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    code = _dtype_code(k_cache)
    assert _dtype_code(q) == code and _dtype_code(v_cache) == code
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, H, D = q.shape
    _, hkv, bs, d2 = k_cache.shape
    assert d2 == D
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 2)
        out = np.zeros((rows.shape[0], D), dtype=np.float64)
        rp, nr = _ptr(rows), rows.shape[0]
    else:
        out = np.zeros((B, H, D), dtype=np.float64)
        rp, nr = None, 0
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().oracle_paged_attention(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), code,
                                        _ptr(bt), _ptr(ctx), B, H, hkv, D, bs, bt.shape[1],
                                        float(scale), rp, nr, int(nthreads))
    if rc != 0:
        raise ValueError("oracle_paged_attention rejected its arguments")
    return out


def kv_append(k_cache: np.ndarray, v_cache: np.ndarray, k: np.ndarray, v: np.ndarray,
              slot_mapping) -> None:
    """In place on the numpy caches."""
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    code = _dtype_code(k_cache)
    assert k.dtype == k_cache.dtype and v.dtype == v_cache.dtype
    _, hkv, bs, d = k_cache.shape
    _load().oracle_kv_append(_ptr(k_cache), _ptr(v_cache), _ptr(k), _ptr(v), _ptr(sm), len(sm),
                             hkv, d, bs, code)


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, pairs) -> None:
    """In place on the numpy caches."""
    pairs = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    code = _dtype_code(k_cache)
    _, hkv, bs, d = k_cache.shape
    _load().oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pairs), pairs.shape[0], hkv, d,
                               bs, code)


def swap_blocks(dst_k: np.ndarray, dst_v: np.ndarray, src_k: np.ndarray, src_v: np.ndarray,
                pairs) -> None:
    """In place on the destination pools."""
    pairs = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    code = _dtype_code(src_k)
    assert dst_k.dtype == src_k.dtype and dst_k.shape[1:] == src_k.shape[1:]
    _, hkv, bs, d = src_k.shape
    _load().oracle_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(np.ascontiguousarray(src_k)),
                               _ptr(np.ascontiguousarray(src_v)), _ptr(pairs), pairs.shape[0], hkv,
                               d, bs, code)


def e4m3_value(code: int) -> float:
    return float(_load().oracle_e4m3_value(int(code)))


def e4m3_encode(y: float) -> int:
    return int(_load().oracle_e4m3_encode(float(y)))


def kv_append_fp8(k_cache: np.ndarray, v_cache: np.ndarray, k_scales, v_scales, k: np.ndarray,
                  v: np.ndarray, slot_mapping) -> None:
    """In place on uint8 (e4m3 code) caches; k, v are bf16 bit patterns."""
    assert k_cache.dtype == np.uint8 and k.dtype == np.uint16
    ks = np.ascontiguousarray(k_scales, dtype=np.float32)
    vs = np.ascontiguousarray(v_scales, dtype=np.float32)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    _, hkv, bs, d = k_cache.shape
    _load().oracle_kv_append_fp8(_ptr(k_cache), _ptr(v_cache), _ptr(ks), _ptr(vs), _ptr(k), _ptr(v),
                                 _ptr(sm), len(sm), hkv, d, bs)


def paged_attention_fp8(q, k_cache, v_cache, k_scales, v_scales, block_tables, context_lens,
                        scale: float) -> np.ndarray:
    """fp64 decode attention over e4m3 caches with per-kv-head scales; q is bf16 bits."""
    q = np.ascontiguousarray(q)
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    assert q.dtype == np.uint16 and k_cache.dtype == np.uint8
    ks = np.ascontiguousarray(k_scales, dtype=np.float32)
    vs = np.ascontiguousarray(v_scales, dtype=np.float32)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, H, D = q.shape
    _, hkv, bs, _ = k_cache.shape
    out = np.zeros((B, H, D), dtype=np.float64)
    rc = _load().oracle_paged_attention_fp8(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                            _ptr(ks), _ptr(vs), _ptr(bt), _ptr(ctx), B, H, hkv, D,
                                            bs, bt.shape[1], float(scale))
    if rc != 0:
        raise ValueError("oracle_paged_attention_fp8 rejected its arguments")
    return out
