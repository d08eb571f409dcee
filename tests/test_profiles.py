"""The committed DRAM-traffic figures (profiles/*.traffic.txt) that bench.py
folds into its roofline must belong to the kernel sources as they are: each
file's hash is the current source hash of the kernel family that serves its
workload.  A kernel change without a new capture fails here."""
import glob
import os

import pytest

import bench
from paged_kv_cache_323_b200 import workload as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# which decode kernel serves each bench workload (by shape and cache type)
FAMILY = {
    "mha": "reg", "gqa_sampling": "tc_bf16", "long_context": "tc_bf16",
    "prefix_bs8": "tc_bf16", "prefix_bs16": "tc_bf16", "prefix_bs32": "tc_bf16",
    "mha_fp8": "tc_fp8", "gqa_sampling_fp8": "tc_fp8", "long_context_fp8": "tc_fp8",
    "mha_d64_fp8": "tc_fp8_d64", "mha_bs8": "reg", "mha_d64": "reg",
}


def _read(path):
    kv = {}
    for line in open(path):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=", 1)
            kv[k.strip()] = v.strip()
    return kv


@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(ROOT, "profiles", "decode_*.traffic.txt"))),
                         ids=os.path.basename)
def test_traffic_file_matches_current_kernel_sources(path):
    workload = os.path.basename(path)[len("decode_"):-len(".traffic.txt")]
    assert workload in bench.WORKLOADS, workload
    kv = _read(path)
    assert kv["kernel_source_sha256"] == bench.kernel_source_sha(FAMILY[workload])
    assert int(kv["dram_bytes_per_launch"]) > 0
    assert bench.committed_traffic("decode", workload, bench.kernel_source_sha(FAMILY[workload])) == \
        float(kv["dram_bytes_per_launch"])


@pytest.mark.parametrize("heads,kv_heads,dtype,head_dim,family", [
    (32, 32, "bf16", 128, "reg"), (32, 8, "bf16", 128, "tc_bf16"), (64, 8, "bf16", 128, "tc_bf16"),
    (32, 32, "fp8", 128, "tc_fp8"), (32, 8, "fp8", 128, "tc_fp8"), (8, 8, "f32", 128, "cuda_core"),
    (32, 32, "fp8", 64, "tc_fp8_d64"), (32, 8, "fp8", 64, "tc_fp8_d64"), (6, 3, "fp8", 64, "cuda_core"),
    (64, 8, "fp8", 64, "cuda_core"), (32, 8, "bf16", 64, "cuda_core"),
])
def test_kernel_family_by_shape(heads, kv_heads, dtype, head_dim, family):
    w = wl.custom(1, [40, 7], heads=heads, kv_heads=kv_heads, head_dim=head_dim, block_size=16,
                  dtype=dtype)
    assert bench.decode_kernel_family(w) == family


@pytest.mark.parametrize("bs,D,dtype,family", [(8, 128, "bf16", "reg"), (16, 128, "bf16", "reg"),
                                              (32, 128, "bf16", "reg"), (16, 64, "bf16", "reg"),
                                              (8, 128, "f32", "cuda_core")])
def test_kernel_family_mha_by_block_size(bs, D, dtype, family):
    w = wl.custom(1, [40, 7], heads=8, kv_heads=8, head_dim=D, block_size=bs, dtype=dtype)
    assert bench.decode_kernel_family(w) == family


@pytest.mark.parametrize("heads,kv_heads,dtype,head_dim,family", [
    (32, 32, "bf16", 128, "reg"), (32, 8, "bf16", 128, "cuda_core"), (32, 32, "fp8", 128, "cuda_core"),
    (32, 32, "bf16", 64, "reg"), (32, 32, "fp8", 64, "cuda_core"),
])
def test_kernel_family_with_tensor_cores_off(heads, kv_heads, dtype, head_dim, family):
    """bench.py --cuda-cores: bf16 MHA keeps the register-streamed kernel, the
    rest falls to the staged CUDA-core kernel."""
    w = wl.custom(1, [40, 7], heads=heads, kv_heads=kv_heads, head_dim=head_dim, block_size=16,
                  dtype=dtype)
    assert bench.decode_kernel_family(w, tensor_cores=False) == family
