"""The debug build (libpagedkv_debug.so, -DPKV_DEBUG): the same sources with
a check on every index the kernels derive from their inputs, standing in for
a device sanitizer.

On the CPU: it compiles for sm_100a, loads, exports every symbol the header
declares, and says which build it is.  On the GPU: one step of every kernel
family (the register-streamed bf16 MHA decode, the staged CUDA-core decode at
block sizes 8 / 16 / 32 over fp32, bf16 and fp8 caches, the tensor-core
decode over bf16 and fp8 caches, split-K with the
fused merge, the longest-first schedule, the fp8 tensor-core kernel in both
forms, the no-alloc entry, append and
copy-on-write) runs through the debug library in a child process, matches
the oracle, and no check fails.
"""
import ctypes
import os
import subprocess
import sys

import pytest

from paged_kv_cache_323_b200 import build as pkv_build
from test_abi import declared_functions

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def debug_lib():
    return ctypes.CDLL(pkv_build.build(debug=True))


def test_debug_build_exports_and_flag(debug_lib):
    for name in declared_functions():
        assert hasattr(debug_lib, name), f"{name} declared but not exported by the debug build"
    assert debug_lib.pkv_debug_build() == 1
    release = ctypes.CDLL(pkv_build.build())
    assert release.pkv_debug_build() == 0


CHILD = r"""
import torch
from paged_kv_cache_323_b200 import pagedkv as pk
from paged_kv_cache_323_b200 import workload as wl
from steps import gpu_step, oracle_step, assert_close, assert_pool_equal, to_device
assert pk.DEBUG and pk.lib.pkv_debug_build() == 1
pk.set_longest_first(2)  # plan every launch, so the schedule's checks run too
cases = [
    ("register-streamed bs8 split-K", wl.mha(num_seqs=6, num_blocks=1200, heads=4, block_size=8), 256),
    ("register-streamed bs16", wl.mha(num_seqs=6, num_blocks=600, heads=4), 0),
    ("cuda-core bs32 fp32", wl.custom(3, [1, 31, 33, 700], heads=4, kv_heads=2, head_dim=64,
                                     block_size=32, dtype="f32"), 128),
    ("tensor-core bf16 copy-on-write", wl.gqa_sampling(groups=3, prompt_median=300, prompt_max=1500), 256),
    ("tensor-core fp8 (persistent)", wl.custom(5, [1, 129, 640, 3000], heads=16, kv_heads=2,
                                              head_dim=128, block_size=16, dtype="fp8"), 512),
    ("tensor-core fp8 head_dim 64 (kv head pairs)", wl.custom(6, [5, 77, 900], heads=4, kv_heads=2,
                                                              head_dim=64, block_size=16, dtype="fp8"), 256),
    ("tensor-core fp8 head_dim 64, 4 heads per kv head, block size 32",
     wl.custom(7, [5, 77, 900], heads=16, kv_heads=4, head_dim=64, block_size=32, dtype="fp8"), 256),
    ("cuda-core fp8 head_dim 64, 8 heads per kv head", wl.custom(8, [5, 77, 900], heads=16, kv_heads=2,
                                                                 head_dim=64, block_size=16,
                                                                 dtype="fp8"), 256),
    ("cuda-core fp8 head_dim 64, odd kv heads", wl.custom(9, [5, 77, 900], heads=3, kv_heads=3,
                                                          head_dim=64, block_size=16, dtype="fp8"), 256),
]
for name, w, pt in cases:
    ref, kref, vref = oracle_step(w)
    out, kc, vc = gpu_step(w, partition_tokens=pt)
    assert_pool_equal(kc, kref, name + ": k pool")
    assert_close(out, ref, "bf16" if w.dtype == "fp8" else w.dtype, name)
    line = pk.debug_failed_line()
    assert line == 0, f"{name}: index check failed at line {line}"
pk._set_fp8_persistent(False)  # the fp8 tensor-core kernel with one CTA per unit
name, w, pt = cases[4]  # the head_dim-128 fp8 case
ref, kref, vref = oracle_step(w)
out, kc, vc = gpu_step(w, partition_tokens=pt)
assert_close(out, ref, "bf16", name + ", one CTA per unit")
assert pk.debug_failed_line() == 0, "one CTA per unit: index check failed"
pk._set_fp8_persistent(True)
pk._set_reg_stream(False)  # bf16 MHA on the staged kernel (bulk copies into shared memory)
for name, w, pt in cases[:2]:
    ref, _, _ = oracle_step(w)
    out, _, _ = gpu_step(w, partition_tokens=pt)
    assert_close(out, ref, w.dtype, name + ", staged")
    assert pk.debug_failed_line() == 0, name + ", staged: index check failed"
pk._set_reg_stream(True)
w = wl.mha(num_seqs=8, num_blocks=2048)
ref, _, _ = oracle_step(w)
t = to_device(w)
pk.kv_cache_append(t["k_cache"], t["v_cache"], t["k_new"], t["v_new"], t["slot_mapping"])
pk.paged_attention_decode_noalloc(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                  t["context_lens"], w.scale, num_blocks=w.num_blocks)
torch.cuda.synchronize()
assert pk.get_device_error() == 0
assert_close(t["out"], ref, w.dtype, "no-alloc")
assert pk.debug_failed_line() == 0
print("DEBUG_BUILD_OK")
"""


@pytest.mark.gpu
def test_debug_build_runs_every_kernel_clean():
    pkv_build.build(debug=True)
    env = dict(os.environ, PKV_LIBRARY="debug",
               PYTHONPATH=os.pathsep.join([ROOT, os.path.join(ROOT, "tests"),
                                           os.environ.get("PYTHONPATH", "")]))
    p = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert p.returncode == 0 and "DEBUG_BUILD_OK" in p.stdout, (p.stdout[-3000:] + p.stderr[-3000:])
