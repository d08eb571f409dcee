"""Thin ctypes binding of libpagedkv.so (the C ABI in include/pagedkv.h).

Argument marshalling only: each function takes torch tensors that already
live on the GPU, reads their shapes and device pointers, and calls the C
entry point of the same name on the current torch stream.  Every step of the
decode path runs in the library's CUDA kernels; there is no fallback, and
importing this module fails when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# PKV_LIBRARY=debug loads the build whose kernels check every derived index
# (python -m paged_kv_cache_323_b200.build --debug)
DEBUG = os.environ.get("PKV_LIBRARY", "") == "debug"
LIB_PATH = os.path.join(_HERE, "libpagedkv_debug.so" if DEBUG else "libpagedkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_323_b200.build"
        f"{' --debug' if DEBUG else ''}` (nvcc, sm_100a); the decode path has no other "
        "implementation")

lib = ctypes.CDLL(LIB_PATH)

PKV_OK = 0
PKV_ERR_NULL = -1
PKV_ERR_INVALID = -2
PKV_ERR_UNSUPPORTED = -3
PKV_ERR_CUDA = -4
PKV_ERR_WORKSPACE = -5
PKV_ERR_DEVICE_BOUNDS = -6
PKV_ERR_TIMEOUT = -7
PKV_ERR_OUT_OF_BLOCKS = -8
PKV_F32 = 0
PKV_BF16 = 1
PKV_FP8_E4M3 = 2
KERNEL_DECODE = 0
KERNEL_APPEND = 1
KERNEL_COPY_BLOCKS = 2
KERNEL_SWAP_BLOCKS = 3

_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); the order mirrors include/pagedkv.h
SIGNATURES = {
    "paged_attention_decode": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P]),
    "paged_attention_decode_ex": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float,
                                       _I, _I, _I, _P, _SZ, _P]),
    "paged_attention_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "paged_attention_decode_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                        ctypes.c_float, _I, _I, _P, _SZ, _P]),
    "kv_cache_append_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "paged_attention_partition_tokens": (_I, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "paged_attention_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                            ctypes.c_float, _I, _I, _I, _P]),
    "kv_cache_append": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "copy_blocks": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "swap_blocks": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P]),
    "pkv_bm_create": (_P, [_I, _I, _I, _P]),
    "pkv_bm_destroy": (None, [_P]),
    "pkv_bm_add_sequence": (_I, [_P]),
    "pkv_bm_fork": (_I, [_P, _I]),
    "pkv_bm_append": (_I, [_P, _I, _I, _P, _P, _I, ctypes.POINTER(_I)]),
    "pkv_bm_free": (_I, [_P, _I]),
    "pkv_bm_tables": (_I, [_P, _P, _I, _I, _P, _P]),
    "pkv_bm_length": (_I, [_P, _I]),
    "pkv_bm_pick_victim": (_I, [_P]),
    "pkv_bm_swap_out": (_I, [_P, _I, _P, _I, ctypes.POINTER(_I)]),
    "pkv_bm_swap_in": (_I, [_P, _I, _P, _I, ctypes.POINTER(_I)]),
    "pkv_bm_get_stats": (_I, [_P, _P]),
    "pkv_get_device_error": (_I, [_P, ctypes.POINTER(_I)]),
    "pkv_selftest_bounded_wait": (_I, [_I, _P]),
    "pkv_set_wait_limit_us": (_I, [_I]),
    "pkv_debug_build": (_I, []),
    "pkv_debug_failed_line": (_I, [_P, ctypes.POINTER(_I)]),
    "pkv_status_string": (ctypes.c_char_p, [_I]),
    "pkv_profile_enable": (_I, [_I]),
    "pkv_profile_read": (_I, [_I, ctypes.POINTER(ctypes.c_longlong), ctypes.POINTER(ctypes.c_double)]),
    "pkv_profile_reset": (_I, []),
    "pkv_launch_count": (ctypes.c_ulonglong, []),
    "pkv_set_tensor_core_gqa": (_I, [_I]),
    "pkv_set_longest_first": (_I, [_I]),
    "pkv_version": (_I, []),
}
for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args
# not in the header: selects the fp8 tensor-core decode's persistent form
lib.pkv_internal_set_fp8_persistent.restype = _I
lib.pkv_internal_set_fp8_persistent.argtypes = [_I]
lib.pkv_internal_set_reg_stream.restype = _I
lib.pkv_internal_set_reg_stream.argtypes = [_I]


class PagedKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def status_string(status: int) -> str:
    return lib.pkv_status_string(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != PKV_OK:
        raise PagedKVError(rc, where)


def _stream(stream, device=None) -> int:
    """cudaStream_t of `stream` (None: the current stream of `device`)."""
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        if device is not None and stream.device != device:
            raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
        return stream.cuda_stream
    return int(stream)


def _device(*tensors) -> torch.device:
    """The device of the first CUDA tensor given (else the current device):
    the call runs there, and every other device tensor must be on it."""
    for t in tensors:
        if t is not None and t.is_cuda:
            return t.device
    return torch.device("cuda", torch.cuda.current_device())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return PKV_F32
    if t.dtype == torch.bfloat16:
        return PKV_BF16
    if t.dtype == torch.float8_e4m3fn:
        return PKV_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t: torch.Tensor, name: str, dtype=None, *, device=None, shape=None) -> int:
    """Device pointer of a contiguous CUDA tensor, after checking its device,
    element type and shape where given."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the other tensors on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


# Split-K workspaces the binding keeps for calls that pass none: one zeroed
# uint8 buffer per (device index, stream handle), grown when a call needs
# more.  Each buffer is allocated on its own stream, so torch's allocator
# reuses the memory of a replaced one only after the work queued on that
# stream before the replacement.  Calls on one stream are ordered, so
# sharing the buffer between them is safe; different streams get different
# buffers.
_workspaces: dict = {}


def _torch_stream(stream_handle: int, dev: torch.device):
    if stream_handle == torch.cuda.current_stream(dev).cuda_stream:
        return torch.cuda.current_stream(dev)
    return torch.cuda.ExternalStream(stream_handle, device=dev)


def _workspace_for(need: int, dev: torch.device, stream_handle: int) -> torch.Tensor:
    key = (dev.index, stream_handle)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < need:
        with torch.cuda.stream(_torch_stream(stream_handle, dev)):
            ws = torch.zeros(need + need // 4, dtype=torch.uint8, device=dev)
        _workspaces[key] = ws
    return ws


def _tables(block_tables, context_lens, B: int) -> int:
    """max_blocks_per_seq of a [B][max_blocks] table; context_lens must be [B]."""
    if block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError(f"block_tables must be [{B}][max_blocks_per_seq], got {tuple(block_tables.shape)}")
    if tuple(context_lens.shape) != (B,):
        raise ValueError(f"context_lens must be [{B}], got {tuple(context_lens.shape)}")
    return block_tables.shape[1]


def paged_attention_workspace_size(num_seqs: int, num_heads: int, max_context: int, head_dim: int,
                                   partition_tokens: int = 0) -> int:
    return int(lib.paged_attention_workspace_size(num_seqs, num_heads, max_context, head_dim,
                                                  partition_tokens))


def paged_attention_partition_tokens(num_seqs: int, num_heads: int, num_kv_heads: int,
                                     head_dim: int, block_size: int, max_context: int,
                                     dtype: int = PKV_BF16, partition_tokens: int = 0) -> int:
    return int(lib.paged_attention_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim,
                                                    block_size, max_context, dtype,
                                                    partition_tokens))


def paged_attention_decode_ex(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                              *, num_blocks: int | None = None, partition_tokens: int = 0,
                              workspace: torch.Tensor | None = None, stream=None) -> None:
    """out, q: [B][H][D]; caches: [N][Hkv][bs][D]; block_tables int32 [B][maxb];
    context_lens int32 [B].  ``workspace`` is a zero-initialised uint8 CUDA
    tensor of at least :func:`paged_attention_workspace_size` bytes, reusable
    across calls of any shape; when None, a buffer this module keeps per
    (device, stream) is used."""
    B, H, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (B, H, D) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between q, out and the caches")
    maxb = _tables(block_tables, context_lens, B)
    if num_blocks is None:
        num_blocks = N
    dev = _device(q)
    code = _dtype_code(q)
    args = (_dev(out, "out", q.dtype, device=dev), _dev(q, "q", device=dev),
            _dev(k_cache, "k_cache", q.dtype, device=dev), _dev(v_cache, "v_cache", q.dtype, device=dev),
            _dev(block_tables, "block_tables", torch.int32, device=dev),
            _dev(context_lens, "context_lens", torch.int32, device=dev))
    need = paged_attention_workspace_size(B, H, maxb * bs, D, partition_tokens)
    st = _stream(stream, dev)
    if workspace is None and need > 0:
        workspace = _workspace_for(need, dev, st)
    ws_ptr = _dev(workspace, "workspace", torch.uint8, device=dev) if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    with torch.cuda.device(dev):
        rc = lib.paged_attention_decode_ex(*args, B, H, Hkv, D, bs, maxb, float(scale),
                                           int(num_blocks), code, int(partition_tokens), ws_ptr,
                                           ws_bytes, st)
    _check(rc, "paged_attention_decode_ex")


def paged_attention_decode_fp8(out, q, k_cache, v_cache, k_scales, v_scales, block_tables,
                               context_lens, scale: float, *, num_blocks: int | None = None,
                               partition_tokens: int = 0, workspace: torch.Tensor | None = None,
                               stream=None) -> None:
    """fp8 (float8_e4m3fn) caches with per-kv-head float32 scales (CUDA
    tensors [num_kv_heads]); q and out bf16."""
    B, H, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (B, H, D) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between q, out and the caches")
    maxb = _tables(block_tables, context_lens, B)
    dev = _device(q)
    args = (_dev(out, "out", torch.bfloat16, device=dev), _dev(q, "q", torch.bfloat16, device=dev),
            _dev(k_cache, "k_cache", torch.float8_e4m3fn, device=dev),
            _dev(v_cache, "v_cache", torch.float8_e4m3fn, device=dev),
            _dev(k_scales, "k_scales", torch.float32, device=dev, shape=(Hkv,)),
            _dev(v_scales, "v_scales", torch.float32, device=dev, shape=(Hkv,)),
            _dev(block_tables, "block_tables", torch.int32, device=dev),
            _dev(context_lens, "context_lens", torch.int32, device=dev))
    need = paged_attention_workspace_size(B, H, maxb * bs, D, partition_tokens)
    st = _stream(stream, dev)
    if workspace is None and need > 0:
        workspace = _workspace_for(need, dev, st)
    ws_ptr = _dev(workspace, "workspace", torch.uint8, device=dev) if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    with torch.cuda.device(dev):
        rc = lib.paged_attention_decode_fp8(*args, B, H, Hkv, D, bs, maxb, float(scale),
                                            N if num_blocks is None else int(num_blocks),
                                            int(partition_tokens), ws_ptr, ws_bytes, st)
    _check(rc, "paged_attention_decode_fp8")


def kv_cache_append_fp8(k_cache, v_cache, k_scales, v_scales, k, v, slot_mapping, stream=None) -> None:
    """Quantise bf16 rows k, v [T][Hkv][D] into the fp8 pools."""
    T = slot_mapping.shape[0]
    N, Hkv, bs, D = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache and v_cache must have the same shape")
    if T and (tuple(k.shape) != (T, Hkv, D) or tuple(v.shape) != (T, Hkv, D)):
        raise ValueError("k / v must be [num_tokens][num_kv_heads][head_dim]")
    dev = _device(k_cache)
    args = (_dev(k_cache, "k_cache", torch.float8_e4m3fn, device=dev),
            _dev(v_cache, "v_cache", torch.float8_e4m3fn, device=dev),
            _dev(k_scales, "k_scales", torch.float32, device=dev, shape=(Hkv,)),
            _dev(v_scales, "v_scales", torch.float32, device=dev, shape=(Hkv,)),
            _dev(k, "k", torch.bfloat16, device=dev) if T else None,
            _dev(v, "v", torch.bfloat16, device=dev) if T else None,
            _dev(slot_mapping, "slot_mapping", torch.int64, device=dev, shape=(T,)) if T else None)
    with torch.cuda.device(dev):
        rc = lib.kv_cache_append_fp8(*args, T, Hkv, D, bs, N, _stream(stream, dev))
    _check(rc, "kv_cache_append_fp8")


# Size of the fixed device scratch of paged_attention_decode_noalloc.
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def paged_attention_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens,
                                   scale: float, *, num_blocks: int | None = None,
                                   partition_tokens: int = 0, stream=None) -> None:
    """Same result as :func:`paged_attention_decode_ex`, for callers that
    cannot allocate device memory (a KV pool that fills the GPU, a host
    allocator that must account for every byte, or a loop that cannot afford
    cudaMalloc's synchronisation): the split-K scratch lives in a fixed
    NOALLOC_SCRATCH_BYTES device array inside the library, shared by every
    call, so calls must not overlap on the GPU.  Batches that need more
    scratch raise PagedKVError (PKV_ERR_WORKSPACE).  Nothing is allocated."""
    B, H, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (B, H, D) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between q, out and the caches")
    maxb = _tables(block_tables, context_lens, B)
    dev = _device(q)
    args = (_dev(out, "out", q.dtype, device=dev), _dev(q, "q", device=dev),
            _dev(k_cache, "k_cache", q.dtype, device=dev), _dev(v_cache, "v_cache", q.dtype, device=dev),
            _dev(block_tables, "block_tables", torch.int32, device=dev),
            _dev(context_lens, "context_lens", torch.int32, device=dev))
    with torch.cuda.device(dev):
        rc = lib.paged_attention_decode_noalloc(*args, B, H, Hkv, D, bs, maxb, float(scale),
                                                N if num_blocks is None else int(num_blocks),
                                                _dtype_code(q), int(partition_tokens),
                                                _stream(stream, dev))
    _check(rc, "paged_attention_decode_noalloc")


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                           stream=None) -> None:
    """bf16 form with the library-owned workspace (see include/pagedkv.h)."""
    B, H, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (B, H, D) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between q, out and the caches")
    maxb = _tables(block_tables, context_lens, B)
    dev = _device(q)
    args = (_dev(out, "out", torch.bfloat16, device=dev), _dev(q, "q", torch.bfloat16, device=dev),
            _dev(k_cache, "k_cache", torch.bfloat16, device=dev),
            _dev(v_cache, "v_cache", torch.bfloat16, device=dev),
            _dev(block_tables, "block_tables", torch.int32, device=dev),
            _dev(context_lens, "context_lens", torch.int32, device=dev))
    with torch.cuda.device(dev):
        rc = lib.paged_attention_decode(*args, B, H, Hkv, D, bs, maxb, float(scale),
                                        _stream(stream, dev))
    _check(rc, "paged_attention_decode")


def kv_cache_append(k_cache, v_cache, k, v, slot_mapping, stream=None) -> None:
    """k, v: [T][Hkv][D]; slot_mapping int64 [T] (-1 = skip)."""
    T = slot_mapping.shape[0]
    N, Hkv, bs, D = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache and v_cache must have the same shape")
    if T and (tuple(k.shape) != (T, Hkv, D) or tuple(v.shape) != (T, Hkv, D)):
        raise ValueError("k / v must be [num_tokens][num_kv_heads][head_dim]")
    dev = _device(k_cache)
    args = (_dev(k_cache, "k_cache", device=dev), _dev(v_cache, "v_cache", k_cache.dtype, device=dev),
            _dev(k, "k", k_cache.dtype, device=dev) if T else None,
            _dev(v, "v", k_cache.dtype, device=dev) if T else None,
            _dev(slot_mapping, "slot_mapping", torch.int64, device=dev, shape=(T,)) if T else None)
    with torch.cuda.device(dev):
        rc = lib.kv_cache_append(*args, T, Hkv, D, bs, N, _dtype_code(k_cache), _stream(stream, dev))
    _check(rc, "kv_cache_append")


def copy_blocks(k_cache, v_cache, src_dst_pairs, stream=None) -> None:
    """src_dst_pairs: int64 [n][2] of (src, dst) physical blocks."""
    n = src_dst_pairs.shape[0]
    N, Hkv, bs, D = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache and v_cache must have the same shape")
    dev = _device(k_cache)
    args = (_dev(k_cache, "k_cache", device=dev), _dev(v_cache, "v_cache", k_cache.dtype, device=dev),
            _dev(src_dst_pairs, "src_dst_pairs", torch.int64, device=dev, shape=(n, 2)) if n else None)
    with torch.cuda.device(dev):
        rc = lib.copy_blocks(*args, n, Hkv, D, bs, N, _dtype_code(k_cache), _stream(stream, dev))
    _check(rc, "copy_blocks")


def _reachable(t: torch.Tensor, name: str, dtype=None, *, device=None, shape=None) -> int:
    """Pointer of a device tensor (on `device`) or of a pinned host tensor (swap pools)."""
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    if t.is_cuda and device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the other device tensors on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def swap_blocks(dst_k, dst_v, src_k, src_v, src_dst_pairs, stream=None) -> None:
    """Copy whole blocks between pools, either of which may be pinned host
    memory (preemption by swapping); src_dst_pairs int64 [n][2]."""
    n = src_dst_pairs.shape[0]
    Ns, Hkv, bs, D = src_k.shape
    Nd = dst_k.shape[0]
    if tuple(dst_k.shape[1:]) != (Hkv, bs, D):
        raise ValueError("source and destination pools must share the block layout")
    if tuple(src_v.shape) != tuple(src_k.shape) or tuple(dst_v.shape) != tuple(dst_k.shape):
        raise ValueError("K and V pools must have the same shape")
    dev = _device(dst_k, src_k, src_dst_pairs)
    args = (_reachable(dst_k, "dst_k", device=dev), _reachable(dst_v, "dst_v", dst_k.dtype, device=dev),
            _reachable(src_k, "src_k", dst_k.dtype, device=dev),
            _reachable(src_v, "src_v", dst_k.dtype, device=dev),
            _reachable(src_dst_pairs, "src_dst_pairs", torch.int64, device=dev, shape=(n, 2))
            if n else None)
    with torch.cuda.device(dev):
        rc = lib.swap_blocks(*args, n, Hkv, D, bs, Ns, Nd, _dtype_code(dst_k), _stream(stream, dev))
    _check(rc, "swap_blocks")


class _BmStats(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int64) for name in (
        "num_blocks", "free_blocks", "used_blocks", "allocated_slots", "used_slots",
        "logical_allocated", "logical_used", "live_sequences", "swapped_sequences",
        "host_free_blocks", "preemptions", "copy_on_write")]


class BlockManager:
    """The native block manager (include/pkv_block_manager.h): free lists,
    block tables, refcounts, forks, copy-on-write pairs, swapping, counters."""

    def __init__(self, num_blocks: int, block_size: int, num_host_blocks: int = 0, free_order=None):
        import numpy as np

        self._np = np
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
        self.block_size = block_size
        # the instance keeps the library: at interpreter exit the module's
        # globals may be cleared before this object is collected
        self._lib = lib
        self._h = lib.pkv_bm_create(num_blocks, block_size, num_host_blocks,
                                    order.ctypes.data if order is not None else None)
        if not self._h:
            raise ValueError("pkv_bm_create rejected its arguments")

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def _id(self, rc: int, where: str) -> int:
        if rc < 0:
            raise PagedKVError(rc, where)
        return rc

    def add_sequence(self) -> int:
        return self._id(lib.pkv_bm_add_sequence(self._h), "pkv_bm_add_sequence")

    def fork(self, parent: int) -> int:
        return self._id(lib.pkv_bm_fork(self._h, parent), "pkv_bm_fork")

    def append(self, seq: int, n: int):
        """Slots of n new tokens (int64 [n]) and copy-on-write pairs (int64 [k][2])."""
        np = self._np
        slots = np.empty(max(n, 1), dtype=np.int64)
        pairs = np.empty((1, 2), dtype=np.int64)
        k = ctypes.c_int(0)
        _check(lib.pkv_bm_append(self._h, seq, n, slots.ctypes.data, pairs.ctypes.data, 1,
                                 ctypes.byref(k)), "pkv_bm_append")
        return slots[:n].copy(), pairs[: k.value].copy()

    def free(self, seq: int) -> None:
        _check(lib.pkv_bm_free(self._h, seq), "pkv_bm_free")

    def tables(self, seqs, max_blocks: int):
        np = self._np
        seqs = np.ascontiguousarray(seqs, dtype=np.int32)
        bt = np.empty((len(seqs), max_blocks), dtype=np.int32)
        lens = np.empty(len(seqs), dtype=np.int32)
        _check(lib.pkv_bm_tables(self._h, seqs.ctypes.data, len(seqs), max_blocks, bt.ctypes.data,
                                 lens.ctypes.data), "pkv_bm_tables")
        return bt, lens

    def length(self, seq: int) -> int:
        return self._id(lib.pkv_bm_length(self._h, seq), "pkv_bm_length")

    def pick_victim(self) -> int:
        return int(lib.pkv_bm_pick_victim(self._h))

    def _swap(self, fn, seq: int, where: str):
        np = self._np
        cap = 1 << 16
        pairs = np.empty((cap, 2), dtype=np.int64)
        k = ctypes.c_int(0)
        _check(fn(self._h, seq, pairs.ctypes.data, cap, ctypes.byref(k)), where)
        return pairs[: k.value].copy()

    def swap_out(self, seq: int):
        """(device_block, host_block) pairs to copy device -> host."""
        return self._swap(lib.pkv_bm_swap_out, seq, "pkv_bm_swap_out")

    def swap_in(self, seq: int):
        """(host_block, device_block) pairs to copy host -> device."""
        return self._swap(lib.pkv_bm_swap_in, seq, "pkv_bm_swap_in")

    def stats(self) -> dict:
        st = _BmStats()
        _check(lib.pkv_bm_get_stats(self._h, ctypes.byref(st)), "pkv_bm_get_stats")
        return {name: int(getattr(st, name)) for name, _ in _BmStats._fields_}


def get_device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    _check(lib.pkv_get_device_error(_stream(stream), ctypes.byref(code)), "pkv_get_device_error")
    return code.value


def debug_failed_line(stream=None) -> int:
    """Source line of the first failed index check of a debug build (0: none)."""
    line = ctypes.c_int(0)
    _check(lib.pkv_debug_failed_line(_stream(stream), ctypes.byref(line)), "pkv_debug_failed_line")
    return line.value


def selftest_bounded_wait(timeout_us: int, stream=None) -> None:
    """Launch a wait that runs out after timeout_us (see include/pagedkv.h)."""
    _check(lib.pkv_selftest_bounded_wait(int(timeout_us), _stream(stream)), "pkv_selftest_bounded_wait")


def set_wait_limit_us(microseconds: int) -> int:
    """Failure-path test hook: limit of the decode kernels' pipeline waits
    (0 restores the one-second default); returns the previous limit."""
    rc = int(lib.pkv_set_wait_limit_us(int(microseconds)))
    if rc < 0:
        raise PagedKVError(rc, "pkv_set_wait_limit_us")
    return rc


def profile_enable(on: bool = True) -> None:
    _check(lib.pkv_profile_enable(1 if on else 0), "pkv_profile_enable")


def profile_read(kind: int) -> tuple[int, float]:
    n = ctypes.c_longlong(0)
    ms = ctypes.c_double(0.0)
    _check(lib.pkv_profile_read(kind, ctypes.byref(n), ctypes.byref(ms)), "pkv_profile_read")
    return n.value, ms.value


def profile_reset() -> None:
    _check(lib.pkv_profile_reset(), "pkv_profile_reset")


def launch_count() -> int:
    return int(lib.pkv_launch_count())


def set_tensor_core_gqa(enable: bool) -> bool:
    """Select the tensor-core (True) or CUDA-core (False) decode kernels
    where a tensor-core one applies (bf16 caches with grouped query heads,
    fp8 caches); returns the previous setting."""
    return bool(lib.pkv_set_tensor_core_gqa(1 if enable else 0))


def _set_fp8_persistent(enable: bool) -> bool:
    """The fp8 tensor-core decode in persistent form (the default: one CTA
    per resident slot taking units from a queue in the workspace, longest
    first) where it applies -- a workspace is given and partitions are at
    most 128 blocks -- or one CTA per unit (False).  Returns the previous
    setting."""
    return bool(lib.pkv_internal_set_fp8_persistent(1 if enable else 0))


def _set_reg_stream(enable: bool) -> bool:
    """bf16 MHA decode over 8-token blocks with K and V streamed through
    registers (the default) or staged in shared memory by bulk copies
    (False).  Returns the previous setting."""
    return bool(lib.pkv_internal_set_reg_stream(1 if enable else 0))


def set_longest_first(mode: int) -> int:
    """Schedule of the decode grid: 1 (the default) longest first where it
    pays, 2 always, 0 never; all give the same bits.  Returns the previous
    mode."""
    rc = int(lib.pkv_set_longest_first(int(mode)))
    if rc < 0:
        raise PagedKVError(rc, "pkv_set_longest_first")
    return rc
