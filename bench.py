"""Benchmark of the paged decode step on B200.

A step is one pass of the whole hot path over one batch: copy-on-write block
copies (when the workload has forks), the append of the step's new tokens,
and block-table decode attention (partition kernel + split-K reduce).  The
default workload is MHA decode: batch 64, 32 query = 32 KV heads, head_dim
128, bf16, block_size 16, context lengths U[128, 2048], pool of 16384 blocks
placed by a seeded permutation, one new token per sequence.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle, bounded sample

Prints one JSON line (rank 0).  Under torchrun each rank runs its own batch
(weak scaling, no data-path collective); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_323_b200 import workload as wl  # noqa: E402

METRIC = "paged decode-attention KV-read HBM GB/s (% of B200 peak) and tokens/s"
FALLBACK_HBM_GBS = 6650.0

WORKLOADS = {
    "mha": ("mha_decode_b64_h32_kv32_d128_bs16_ctxU128-2048_bf16",
            lambda dev, seed: wl.mha(seed=seed, device=dev)),
    "gqa_sampling": ("gqa_sampling_b256_g64x4_h32_kv8_d128_bs16_bf16",
                     lambda dev, seed: wl.gqa_sampling(seed=seed, device=dev)),
    "long_context": ("long_context_b8_h64_kv8_d128_bs32_ctxU32768-131072_bf16",
                     lambda dev, seed: wl.long_context(seed=seed, device=dev)),
    "prefix_bs8": ("prefix_sweep_b1024_prefix2048_h32_kv8_d128_bs8_bf16",
                   lambda dev, seed: wl.prefix_sweep(8, seed=seed, device=dev)),
    "prefix_bs16": ("prefix_sweep_b1024_prefix2048_h32_kv8_d128_bs16_bf16",
                    lambda dev, seed: wl.prefix_sweep(16, seed=seed, device=dev)),
    "prefix_bs32": ("prefix_sweep_b1024_prefix2048_h32_kv8_d128_bs32_bf16",
                    lambda dev, seed: wl.prefix_sweep(32, seed=seed, device=dev)),
    "tiny": ("tiny_b4_ctx35-16-1-50_h4_d64_bs16_f32", lambda dev, seed: wl.tiny(seed=seed, device=dev)),
    # the gather's cost: the same MHA batch at block sizes 8 / 16 / 32, blocks placed at random
    # (paged) or consecutively per sequence (the layout of a contiguous per-request cache)
    "mha_bs8": ("mha_decode_b64_h32_kv32_d128_bs8_ctxU128-2048_bf16",
                lambda dev, seed: wl.mha(seed=seed, device=dev, block_size=8)),
    "mha_bs32": ("mha_decode_b64_h32_kv32_d128_bs32_ctxU128-2048_bf16",
                 lambda dev, seed: wl.mha(seed=seed, device=dev, block_size=32)),
    "mha_contig_bs8": ("mha_decode_b64_h32_kv32_d128_bs8_contiguous_bf16",
                       lambda dev, seed: wl.mha(seed=seed, device=dev, block_size=8, contiguous=True)),
    "mha_contig_bs16": ("mha_decode_b64_h32_kv32_d128_bs16_contiguous_bf16",
                        lambda dev, seed: wl.mha(seed=seed, device=dev, contiguous=True)),
    "mha_contig_bs32": ("mha_decode_b64_h32_kv32_d128_bs32_contiguous_bf16",
                        lambda dev, seed: wl.mha(seed=seed, device=dev, block_size=32, contiguous=True)),
    # the same MHA batch with an fp8 (e4m3) cache and per-kv-head scales: half the KV bytes
    "mha_fp8": ("mha_decode_b64_h32_kv32_d128_bs16_ctxU128-2048_fp8e4m3_cache",
                lambda dev, seed: wl.mha(seed=seed, device=dev, dtype="fp8")),
    # a smaller MHA batch for profiler captures: 16 sequences, 4096-block pool (1 GB), ~0.3 GB KV per step
    "mha_small": ("mha_decode_b16_h32_kv32_d128_bs16_ctxU128-2048_bf16_pool4096",
                  lambda dev, seed: wl.mha(seed=seed, device=dev, num_seqs=16, num_blocks=4096)),
    # fp8 (e4m3) caches on the grouped-query workloads
    "gqa_sampling_fp8": ("gqa_sampling_b256_g64x4_h32_kv8_d128_bs16_fp8e4m3_cache",
                         lambda dev, seed: wl.gqa_sampling(seed=seed, device=dev, dtype="fp8")),
    "long_context_fp8": ("long_context_b8_h64_kv8_d128_bs32_ctxU32768-131072_fp8e4m3_cache",
                         lambda dev, seed: wl.long_context(seed=seed, device=dev, dtype="fp8")),
    # head_dim 64, bf16 cache (the register-streamed kernel)
    "mha_d64": ("mha_decode_b64_h32_kv32_d64_bs16_ctxU128-2048_bf16",
                lambda dev, seed: wl.mha(seed=seed, device=dev, head_dim=64)),
    # head_dim 64 over an fp8 cache (the tensor-core kernel on kv head pairs)
    "mha_d64_fp8": ("mha_decode_b64_h32_kv32_d64_bs16_ctxU128-2048_fp8e4m3_cache",
                    lambda dev, seed: wl.mha(seed=seed, device=dev, head_dim=64, dtype="fp8")),
    "mha_d64_fp8_small": ("mha_decode_b16_h32_kv32_d64_bs16_ctxU128-2048_fp8e4m3_cache_pool4096",
                          lambda dev, seed: wl.mha(seed=seed, device=dev, num_seqs=16, num_blocks=4096,
                                                   head_dim=64, dtype="fp8")),
    "mha_bs8_small": ("mha_decode_b16_h32_kv32_d128_bs8_ctxU128-2048_bf16_pool8192",
                      lambda dev, seed: wl.mha(seed=seed, device=dev, num_seqs=16, num_blocks=8192,
                                               block_size=8)),
    "mha_fp8_small": ("mha_decode_b16_h32_kv32_d128_bs16_ctxU128-2048_fp8e4m3_cache_pool4096",
                      lambda dev, seed: wl.mha(seed=seed, device=dev, num_seqs=16, num_blocks=4096,
                                               dtype="fp8")),
}
DEFAULT_SEED = {"mha": 2, "gqa_sampling": 3, "long_context": 4, "prefix_bs8": 5, "prefix_bs16": 5,
                "prefix_bs32": 5, "tiny": 1, "mha_small": 2, "mha_bs8": 2, "mha_bs32": 2,
                "mha_contig_bs8": 2, "mha_contig_bs16": 2, "mha_contig_bs32": 2, "mha_fp8": 2,
                "mha_fp8_small": 2, "mha_bs8_small": 2, "gqa_sampling_fp8": 3, "long_context_fp8": 4,
                "mha_d64_fp8": 2, "mha_d64_fp8_small": 2, "mha_d64": 2}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def committed_traffic(kernel: str, workload: str, source_sha: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=", 1)
            kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha256") != source_sha:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# source files of each decode kernel family (what the DRAM-traffic counters
# in profiles/ were taken on)
KERNEL_SOURCES = {
    "cuda_core": ("common.cuh", "decode_common.cuh", "decode_attn.cuh", "decode_launch.cuh"),
    "tc_bf16": ("common.cuh", "decode_common.cuh", "decode_tc.cuh", "decode_tc.cu"),
    "tc_fp8": ("common.cuh", "decode_common.cuh", "decode_tc.cuh", "decode_tc_fp8.cuh", "decode_tc_fp8p.cuh",
               "decode_tc_fp8p.cu", "persist.cuh", "plan.cuh"),
    "tc_fp8_d64": ("common.cuh", "decode_common.cuh", "decode_tc.cuh", "decode_tc_fp8.cuh", "decode_tc_fp8_d64.cuh",
                   "decode_tc_fp8_d64.cu", "plan.cuh"),
    "reg": ("common.cuh", "decode_common.cuh", "decode_attn.cuh", "decode_reg.cuh", "decode_reg.cu"),
}


def decode_kernel_family(w, tensor_cores: bool = True) -> str:
    """Which decode kernel the library runs for this workload (tensor-core
    kernels on, as by default, or off)."""
    group = w.num_heads // w.num_kv_heads
    if w.head_dim in (64, 128) and w.dtype == "bf16" and group == 1:
        return "reg"
    if not tensor_cores:
        return "cuda_core"
    if w.head_dim == 128 and w.dtype == "fp8" and group in (1, 2, 4, 8):
        return "tc_fp8"
    if w.head_dim == 64 and w.dtype == "fp8" and group in (1, 2, 4) and w.num_kv_heads % 2 == 0:
        return "tc_fp8_d64"
    if w.head_dim == 128 and w.dtype == "bf16" and group in (2, 4, 8):
        return "tc_bf16"
    return "cuda_core"


def kernel_source_sha(family: str = "cuda_core") -> str:
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_323_b200", "csrc")
    for name in KERNEL_SOURCES[family]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons of this process's GPU,
    sampled by NVML (read-only queries) every ~2 ms in a background thread
    while the timed region runs."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device: int):
        self.device = device
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._nvml = None

    def start(self):
        import threading

        try:
            import pynvml as nv

            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._h = nv.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self._nvml = nv
        except Exception as e:  # no NVML: report no clocks rather than guess
            self._err = repr(e)
            return
        self._stop = threading.Event()

        def loop():
            nv = self._nvml
            while not self._stop.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
                self._stop.wait(0.002)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def stop(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": "NVML unavailable: " + getattr(self, "_err", "")}
        self._stop.set()
        self._thread.join()
        nv = self._nvml
        mhz = [m for m, _ in self.samples]
        reasons = sorted({name for _, rs in self.samples for name, attr in self.REASONS
                          if rs & getattr(nv, attr, 0)})
        try:
            nv.nvmlShutdown()
        except Exception:
            pass
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


def dist_setup(n_gpus: int, cuda: bool = True):
    """One process per GPU under torchrun (NCCL); `cuda` False (the oracle arm
    on a host without a GPU) joins the ranks over gloo instead."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        if cuda:
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif cuda:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(world, x: float) -> float:
    """The slowest rank's time: every rank's number goes through one MAX all-reduce."""
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(workload: str, rank: int) -> int:
    """Each rank draws its own batch (weak scaling): seed offset by rank."""
    return DEFAULT_SEED[workload] + 1000 * rank


def job_value(world: int, kv_bytes_per_rank: int, ms_per_step: float) -> float:
    """Whole-job KV GB/s: the bytes all ranks read per step over the slowest rank's step time."""
    return world * kv_bytes_per_rank / (ms_per_step / 1e3) / 1e9


def compact_subset(w: wl.Workload, seqs):
    """The step restricted to ``seqs`` on a compact host pool (oracle input)."""
    bs = w.block_size
    seqs = list(seqs)
    sel_pairs = [i for i, s in enumerate(w.pair_seq.tolist()) if s in seqs]
    blocks = set()
    for s in seqs:
        nb = -(-int(w.context_lens[s]) // bs)
        blocks.update(int(x) for x in w.block_tables[s][:nb])
    for i in sel_pairs:
        blocks.update(int(x) for x in w.cow_pairs[i])
    order = sorted(blocks)
    remap = {b: i for i, b in enumerate(order)}
    idx = torch.tensor(order, dtype=torch.long, device=w.k_cache.device)
    if w.dtype == "fp8":  # gather the codes as bytes
        kc = w.k_cache.view(torch.uint8).index_select(0, idx).cpu().numpy()
        vc = w.v_cache.view(torch.uint8).index_select(0, idx).cpu().numpy()
    else:
        kc = wl.to_numpy_bits(w.k_cache.index_select(0, idx))
        vc = wl.to_numpy_bits(w.v_cache.index_select(0, idx))
    bt = np.full((len(seqs), w.max_blocks_per_seq), -1, dtype=np.int32)
    for i, s in enumerate(seqs):
        nb = -(-int(w.context_lens[s]) // bs)
        bt[i, :nb] = [remap[int(x)] for x in w.block_tables[s][:nb]]
    toks = [i for i, s in enumerate(w.token_seq.tolist()) if s in seqs]
    slots = np.asarray([remap[int(w.slot_mapping[i]) // bs] * bs + int(w.slot_mapping[i]) % bs
                        for i in toks], dtype=np.int64)
    tok_idx = torch.tensor(toks, dtype=torch.long, device=w.k_new.device)
    pairs = np.asarray([[remap[int(w.cow_pairs[i][0])], remap[int(w.cow_pairs[i][1])]]
                        for i in sel_pairs], dtype=np.int64).reshape(-1, 2)
    q = wl.to_numpy_bits(w.q.index_select(0, torch.tensor(seqs, device=w.q.device)))
    return dict(q=q, kc=kc, vc=vc, bt=bt, ctx=w.context_lens[seqs].copy(), slots=slots,
                k_new=wl.to_numpy_bits(w.k_new.index_select(0, tok_idx)),
                v_new=wl.to_numpy_bits(w.v_new.index_select(0, tok_idx)), pairs=pairs,
                k_scales=w.k_scales, v_scales=w.v_scales,
                kv_bytes=int(w.context_lens[seqs].astype(np.int64).sum()) * w.num_kv_heads
                * w.head_dim * 2 * w.elt)


def oracle_sample_step(sub, scale, threads):
    """One step of the oracle on a compact sample: (seconds, fp64 output rows)."""
    import oracle

    kc = sub["kc"].copy()
    vc = sub["vc"].copy()
    t0 = time.perf_counter()
    if len(sub["pairs"]):
        oracle.copy_blocks(kc, vc, sub["pairs"])
    if sub["k_scales"] is not None:  # fp8 cache
        oracle.kv_append_fp8(kc, vc, sub["k_scales"], sub["v_scales"], sub["k_new"], sub["v_new"],
                             sub["slots"])
        out = oracle.paged_attention_fp8(sub["q"], kc, vc, sub["k_scales"], sub["v_scales"],
                                         sub["bt"], sub["ctx"], scale)
        return time.perf_counter() - t0, out
    oracle.kv_append(kc, vc, sub["k_new"], sub["v_new"], sub["slots"])
    out = oracle.paged_attention(sub["q"], kc, vc, sub["bt"], sub["ctx"], scale, nthreads=threads)
    return time.perf_counter() - t0, out


def pick_sample(w: wl.Workload, target_s: float, threads: int):
    """Grow a seeded sample of sequences until one oracle step costs about
    target_s; returns (sample, sequences, seconds, the sample's output rows)."""
    rng = np.random.default_rng(1234)
    order = rng.permutation(w.num_seqs).tolist()
    n = min(len(order), max(1, threads))
    while True:
        seqs = sorted(order[:n])
        sub = compact_subset(w, seqs)
        dt, out = oracle_sample_step(sub, w.scale, threads)
        if dt >= target_s / 4 or n >= len(order):
            break
        n = min(len(order), max(n + 1, int(n * min(8.0, target_s / 4 / max(dt, 1e-3)))))
    sub["seqs"] = seqs
    return sub, n, dt, out


# Parity bar of bf16 (and fp8-cache) outputs against the fp64 oracle:
# |gpu - ref| <= 2e-2 + 1e-2 |ref| per element; fp32: |gpu - ref| <= 1e-5.
def rows_match(gpu_rows: torch.Tensor, ref: np.ndarray, dtype: str) -> dict:
    g = gpu_rows.detach().float().cpu().double().numpy().reshape(ref.shape)
    err = np.abs(g - ref)
    ok = bool(np.all(np.isfinite(g))) and (
        bool(err.max() <= 1e-5) if dtype == "f32" else bool(np.all(err <= 2e-2 + 1e-2 * np.abs(ref))))
    return {"rows": int(ref.shape[0] * ref.shape[1]), "max_abs_err": float(err.max()), "ok": ok,
            "bar": "max abs 1e-5" if dtype == "f32" else "|gpu - ref| <= 2e-2 + 1e-2 |ref|"}


def measure_swap(pk, w, stream, nblocks: int = 1024, reps: int = 5) -> dict:
    """Preemption by swapping: host-link bandwidth of swap_blocks moving
    `nblocks` whole blocks of the pool to a pinned host pool and back (CUDA
    events on the launch stream, best of `reps`)."""
    nblocks = min(nblocks, w.num_blocks)
    shape = (nblocks,) + tuple(w.k_cache.shape[1:])
    hk = torch.empty(shape, dtype=w.k_cache.dtype, pin_memory=True)
    hv = torch.empty(shape, dtype=w.k_cache.dtype, pin_memory=True)
    rng = np.random.default_rng(99)
    dev_blocks = torch.from_numpy(rng.choice(w.num_blocks, nblocks, replace=False).astype(np.int64))
    host_blocks = torch.arange(nblocks, dtype=torch.int64)
    out_pairs = torch.stack([dev_blocks, host_blocks], 1).cuda()
    in_pairs = torch.stack([host_blocks, dev_blocks], 1).cuda()
    nbytes = 2 * nblocks * w.k_cache[0].numel() * w.k_cache.element_size()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    res = {}
    for name, args in (("device_to_host", (hk, hv, w.k_cache, w.v_cache, out_pairs)),
                       ("host_to_device", (w.k_cache, w.v_cache, hk, hv, in_pairs))):
        best = float("inf")
        for _ in range(reps):
            e0.record(stream)
            pk.swap_blocks(*args)
            e1.record(stream)
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        res[name + "_gbs"] = nbytes / (best * 1e-3) / 1e9
    res.update({"blocks": nblocks, "bytes": nbytes, "unit": "GB/s"})
    return res


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, world, rank):
    """The oracle as it stands, timed on host cores, on a bounded sample."""
    if rank != 0:
        return
    name, make = WORKLOADS[args.workload]
    # the generator runs on the GPU where there is one (faster for the large
    # pools); the timed work is the oracle on host cores either way
    w = make("cuda" if torch.cuda.is_available() else "cpu", DEFAULT_SEED[args.workload])
    threads = cpu_threads()
    sub, n, _, _ = pick_sample(w, target_s=8.0 / max(1, args.steps), threads=threads)
    for _ in range(min(args.warmup, 1)):
        oracle_sample_step(sub, w.scale, threads)
    times = [oracle_sample_step(sub, w.scale, threads)[0] for _ in range(args.steps)]
    t = sum(times) / len(times)
    value = sub["kv_bytes"] / t / 1e9
    sample = f"{n} of {w.num_seqs} sequences (seeded), all heads, per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": name},
        "tokens_per_s": n / t,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# Configurations measured beside the headline in the default run: the
# parallel-sampling GQA batch, the long-context split-K batch and the
# prefix-sharing block-size sweep.
# configs 3-5, then the block-size-8 MHA step and the fp8-cache rows (the quantised cache)
DEFAULT_CONFIGS = ("gqa_sampling", "long_context", "prefix_bs8", "prefix_bs16", "prefix_bs32", "mha_bs8",
                   "mha_fp8", "gqa_sampling_fp8", "mha_d64_fp8")
L2_FLUSH_BYTES = 512 << 20  # written before each cold step: four times the 126 MB L2


def device_inputs(w, dev) -> dict:
    return {
        "q": w.q, "k_cache": w.k_cache, "v_cache": w.v_cache, "k_new": w.k_new, "v_new": w.v_new,
        "bt": torch.from_numpy(w.block_tables).to(dev),
        "ctx": torch.from_numpy(w.context_lens).to(dev),
        "slots": torch.from_numpy(w.slot_mapping).to(dev),
        "pairs": torch.from_numpy(w.cow_pairs).to(dev),
    }


class Step:
    """One pass of the hot path on a workload through the binding: the
    copy-on-write copies (if any), the append, the decode with a caller
    workspace.  Calling it with a set of per-step inputs (q, new K/V, slots,
    tables, lengths) writes the decode output into ``self.out``."""

    def __init__(self, pk, w, t, dev, partition_tokens):
        self.pk, self.w, self.t, self.pt = pk, w, t, partition_tokens
        self.out = torch.empty_like(w.q)
        self.ws_bytes = pk.paged_attention_workspace_size(
            w.num_seqs, w.num_heads, w.max_blocks_per_seq * w.block_size, w.head_dim,
            partition_tokens)
        self.ws = torch.zeros(max(self.ws_bytes, 1), dtype=torch.uint8, device=dev)
        self.fp8 = w.dtype == "fp8"
        if self.fp8:
            self.ks = torch.from_numpy(w.k_scales).to(dev)
            self.vs = torch.from_numpy(w.v_scales).to(dev)
        self.dev_args = (t["q"], t["k_new"], t["v_new"], t["bt"], t["ctx"], t["slots"])

    def __call__(self, q, k_new, v_new, bt, ctx, slots, out=None):
        pk, w, t = self.pk, self.w, self.t
        out = self.out if out is None else out
        ws = self.ws if self.ws_bytes else None
        if len(w.cow_pairs):
            pk.copy_blocks(t["k_cache"], t["v_cache"], t["pairs"])
        if self.fp8:
            pk.kv_cache_append_fp8(t["k_cache"], t["v_cache"], self.ks, self.vs, k_new, v_new, slots)
            pk.paged_attention_decode_fp8(out, q, t["k_cache"], t["v_cache"], self.ks, self.vs, bt,
                                          ctx, w.scale, num_blocks=w.num_blocks,
                                          partition_tokens=self.pt, workspace=ws)
            return
        pk.kv_cache_append(t["k_cache"], t["v_cache"], k_new, v_new, slots)
        pk.paged_attention_decode_ex(out, q, t["k_cache"], t["v_cache"], bt, ctx, w.scale,
                                     num_blocks=w.num_blocks, partition_tokens=self.pt,
                                     workspace=ws)


def timed_region(step, steps, world, stream) -> float:
    """Exactly `steps` steps between a barrier + synchronize on both sides,
    timed by CUDA events on the launching stream; the slowest rank's ms."""
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        step(*step.dev_args)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(world, ev0.elapsed_time(ev1))


def repeat_count(world: int, first_ms: float, min_s: float, cap: int = 200) -> int:
    """Repeats of the timed region so that they span at least `min_s`
    seconds, given the first one took `first_ms`; the same on every rank
    (the largest any rank needs), since each repeat holds barriers."""
    reps = int(min(cap, max(1, -(-min_s * 1e3 // max(first_ms, 1e-3)))))
    return int(max_over_ranks(world, float(reps)))


def repeated_regions(step, steps, world, stream, min_s: float):
    """The timed region repeated until the repeats span at least `min_s`
    seconds (every rank runs the same number); returns the ms of each."""
    first = timed_region(step, steps, world, stream)
    reps = repeat_count(world, first, min_s)
    return [first] + [timed_region(step, steps, world, stream) for _ in range(reps - 1)]


def profiled_region(pk, step, steps, world, stream):
    """The same steps with the library's per-launch events on (they cost a
    few percent, so this region stays out of the headline): the mean device
    time of each kernel and per-step percentiles."""
    pk.profile_reset()
    pk.profile_enable(True)
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    barrier(world)
    torch.cuda.synchronize()
    step_ev[0].record(stream)
    for i in range(steps):
        step(*step.dev_args)
        step_ev[i + 1].record(stream)
    torch.cuda.synchronize()
    pk.profile_enable(False)
    barrier(world)
    step_ms = sorted(step_ev[i].elapsed_time(step_ev[i + 1]) for i in range(steps))
    per_kernel = {}
    for kind, kname in ((pk.KERNEL_DECODE, "decode"), (pk.KERNEL_APPEND, "kv_append"),
                        (pk.KERNEL_COPY_BLOCKS, "copy_blocks")):
        n, kms = pk.profile_read(kind)
        if n:
            per_kernel[kname] = {"launches": n, "avg_us": kms / n * 1e3}
    pk.profile_reset()
    pct = {"p10": step_ms[len(step_ms) // 10], "p50": step_ms[len(step_ms) // 2],
           "p90": step_ms[(9 * len(step_ms)) // 10]}
    return per_kernel, pct


def cold_l2_steps(step, steps, stream, flush) -> float:
    """Median ms of single steps, each timed alone right after a 512 MB write
    (outside its events) has pushed every earlier byte out of L2."""
    times = []
    for _ in range(steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step(*step.dev_args)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def waste_of(w) -> dict:
    wst = w.padded_slot_waste()
    return {"per_sequence": wst["per_sequence_unused"] / max(1, wst["per_sequence_allocated"]),
            "physical": wst["physical_unused"] / max(1, wst["physical_allocated"])}


def partition_of(pk, w, partition_tokens) -> int:
    return pk.paged_attention_partition_tokens(
        w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size,
        w.max_blocks_per_seq * w.block_size,
        {"f32": pk.PKV_F32, "bf16": pk.PKV_BF16, "fp8": pk.PKV_FP8_E4M3}[w.dtype], partition_tokens)


def oracle_check(w, step, target_s: float, threads: int) -> dict:
    """CPU baseline of a configuration: the oracle as it stands, timed on
    this host's cores over a seeded sample of the batch, and its rows
    compared with the GPU step's rows for the same sequences."""
    sub, n, dt, ref = pick_sample(w, target_s=target_s, threads=threads)
    got = step.out.index_select(0, torch.tensor(sub["seqs"], device=step.out.device))
    return {"value": sub["kv_bytes"] / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} of {w.num_seqs} sequences (seeded), all heads, one step in {dt:.2f} s",
            "parity": rows_match(got, ref, w.dtype)}


def measure_config(pk, key, args, world, rank, stream, peak, flush) -> dict:
    """One configuration of the default run's `configs` map."""
    name, make = WORKLOADS[key]
    w = make("cuda", rank_seed(key, rank))
    dev = torch.device("cuda", torch.cuda.current_device())
    step = Step(pk, w, device_inputs(w, dev), dev, args.partition_tokens)
    for _ in range(args.warmup):
        step(*step.dev_args)
    torch.cuda.synchronize()
    code = pk.get_device_error()
    if code != 0:
        raise RuntimeError(f"{key}: device error word {code} after warm-up")
    runs = repeated_regions(step, args.steps, world, stream, min_s=args.min_region_s / 2)
    ms = statistics.median(runs) / args.steps
    per_kernel, pct = profiled_region(pk, step, args.steps, world, stream)
    cold_ms = max_over_ranks(world, cold_l2_steps(step, min(args.steps, 10), stream, flush))
    logical, unique = w.kv_bytes_logical(), w.kv_bytes_unique()
    dec_us = per_kernel.get("decode", {}).get("avg_us")
    fam = decode_kernel_family(w)
    traffic = committed_traffic("decode", key, kernel_source_sha(fam))
    shared = unique < logical
    e = {
        "workload": name, "kernel": fam, "partition_tokens": partition_of(pk, w, args.partition_tokens),
        "step_us": ms * 1e3, "step_us_pct": {k: v * 1e3 for k, v in pct.items()},
        "step_us_cold_l2": cold_ms * 1e3, "decode_us": dec_us,
        "tokens_per_s": world * w.num_seqs / (ms / 1e3),
        "kv_bytes_per_step": {"logical": logical, "unique": unique},
        # logical: every sequence's context bytes; unique: each physical block once
        "kv_gbs_logical": job_value(world, logical, ms), "kv_gbs_unique": job_value(world, unique, ms),
        "pct_of_peak_hbm": 100.0 * job_value(world, logical, ms) / peak,
        "decode_kernel": None if dec_us is None else {
            "logical_gbs": logical / (dec_us * 1e-6) / 1e9,
            "frac_logical": logical / (dec_us * 1e-6) / 1e9 / peak,
            "unique_gbs": unique / (dec_us * 1e-6) / 1e9,
            "dram_gbs": None if traffic is None else traffic / (dec_us * 1e-6) / 1e9,
            "frac_dram": None if traffic is None else traffic / (dec_us * 1e-6) / 1e9 / peak,
            "dram_bytes_per_launch": traffic},
        "l2": ("warm: steps back to back; the shared prefix blocks stay in L2 across sequences"
               if shared else "warm: steps back to back; the KV read per step is larger than L2")
              + "; step_us_cold_l2 flushes L2 (512 MB write) before each step",
        "padded_slot_waste": waste_of(w),
    }
    if world == 1 and not args.no_cpu_baseline:
        e["cpu_baseline"] = oracle_check(w, step, target_s=1.5, threads=cpu_threads())
    del step, w
    torch.cuda.empty_cache()
    return e


def run_gpu(args, world, rank, local):
    from paged_kv_cache_323_b200 import pagedkv as pk

    pk.set_longest_first(args.schedule)
    pk.set_tensor_core_gqa(not args.cuda_cores)
    name, make = WORKLOADS[args.workload]
    w = make("cuda", rank_seed(args.workload, rank))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    step = Step(pk, w, device_inputs(w, dev), dev, args.partition_tokens)
    for _ in range(args.warmup):
        step(*step.dev_args)
    torch.cuda.synchronize()
    code = pk.get_device_error()
    if code != 0:
        raise RuntimeError(f"device error word {code} after warm-up")

    # ------------------------------------------------ device-resident timing
    # The headline region runs exactly `steps` steps bare; it is repeated
    # until the repeats span half a second (so the clock sampler sees the
    # load) and the median repeat is reported.  Per-kernel durations come
    # from a second region of the same steps in which the library brackets
    # every launch with CUDA events on its stream.
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    launches0 = pk.launch_count()
    runs = repeated_regions(step, args.steps, world, stream, min_s=args.min_region_s)
    launches = (pk.launch_count() - launches0) // len(runs)
    ms = statistics.median(runs)
    per_kernel, pct = profiled_region(pk, step, args.steps, world, stream)
    clock_info = clocks.stop()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    cold_ms = max_over_ranks(world, cold_l2_steps(step, min(args.steps, 20), stream, flush))

    # -------------------------------------------- end to end from host memory
    # Every step uploads its inputs (q, new K/V, slots, tables, lengths) from
    # pinned host memory and reads its output back.  Uploads and read-backs
    # run on copy streams with double-buffered device staging, so step i+1's
    # upload and step i-1's read-back overlap step i's kernels: the figure is
    # pipelined throughput, not the latency of one step.  The KV pool stays
    # resident (it is the cache itself).
    names = ("q", "k_new", "v_new", "bt", "ctx", "slots")
    host = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True).copy_(v)
            for k, v in zip(names, step.dev_args)}
    staged = [{k: torch.empty_like(v) for k, v in zip(names, step.dev_args)} for _ in range(2)]
    outs = [torch.empty_like(step.out) for _ in range(2)]
    out_host = [torch.empty(step.out.shape, dtype=step.out.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    up_stream = torch.cuda.Stream()    # host -> device
    down_stream = torch.cuda.Stream()  # device -> host
    ev_up = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b uploaded
    ev_used = [torch.cuda.Event() for _ in range(2)]   # step on buffer b finished
    ev_back = [torch.cuda.Event() for _ in range(2)]   # output of buffer b read back

    def upload(b):
        with torch.cuda.stream(up_stream):
            for k in names:
                staged[b][k].copy_(host[k], non_blocking=True)
            ev_up[b].record(up_stream)

    def e2e_run(n):
        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                if i >= 1:
                    up_stream.wait_event(ev_used[1 - b])  # step i-1 is done with buffer 1-b
                upload(1 - b)
            stream.wait_event(ev_up[b])
            if i >= 2:
                stream.wait_event(ev_back[b])  # outs[b] was read back
            sb = staged[b]
            step(sb["q"], sb["k_new"], sb["v_new"], sb["bt"], sb["ctx"], sb["slots"], out=outs[b])
            ev_used[b].record(stream)
            down_stream.wait_event(ev_used[b])
            with torch.cuda.stream(down_stream):
                out_host[b].copy_(outs[b], non_blocking=True)
                ev_back[b].record(down_stream)
        stream.wait_stream(up_stream)
        stream.wait_stream(down_stream)

    e2e_run(args.warmup)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(stream)
    e2e_run(args.steps)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_e2e = max_over_ranks(world, ev0.elapsed_time(ev1))
    if not torch.equal(out_host[(args.steps - 1) % 2], step.out.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident run")
    code = pk.get_device_error()
    if code != 0:
        raise RuntimeError(f"device error word {code} after the timed steps")

    peak, peak_src = measured_peak()
    kv_bytes = w.kv_bytes_logical()
    kv_unique = w.kv_bytes_unique()
    step_ms = ms / args.steps
    value = job_value(world, kv_bytes, step_ms)
    part = per_kernel.get("decode")
    roofline = None
    if part:
        achieved = kv_bytes / (part["avg_us"] * 1e-6) / 1e9
        fam = decode_kernel_family(w, not args.cuda_cores)
        traffic = committed_traffic("decode", args.workload, kernel_source_sha(fam))
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "traffic": traffic,
                    "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                    else "fallback 6650 GB/s"}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": name, "num_seqs_per_gpu": w.num_seqs, "num_heads": w.num_heads,
                   "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
                   "block_size": w.block_size, "kv_bytes_per_step_per_gpu": kv_bytes,
                   "kv_bytes_unique_per_step_per_gpu": kv_unique,
                   "padded_slot_waste": waste_of(w),
                   "partition_tokens": partition_of(pk, w, args.partition_tokens),
                   "accumulate": "f32",
                   "schedule": {0: "index order", 1: "longest first where it pays",
                                2: "longest first"}[args.schedule],
                   "kernel": decode_kernel_family(w, not args.cuda_cores),
                   "l2": "inputs larger than L2 (KV read per step >> 126 MB), no flush; "
                         "step_us_cold_l2 flushes L2 before each step",
                   "parallelism": f"{world} independent batches, one per GPU"},
        "timing": {"repeats": len(runs), "steps_per_repeat": args.steps,
                   "region_s": sum(runs) / 1e3, "statistic": "median repeat",
                   "repeat_ms_per_step": {"min": min(runs) / args.steps,
                                          "max": max(runs) / args.steps}},
        "tokens_per_s": world * w.num_seqs / (step_ms / 1e3),
        # shared blocks counted once (equal to `value` when nothing is shared)
        "unique_kv_gbs": job_value(world, kv_unique, step_ms),
        "pct_of_peak_hbm": 100.0 * value / peak,
        "per_kernel_us": per_kernel,
        "ms_per_step_profiled_pct": pct,
        "step_us_cold_l2": cold_ms * 1e3,
        "roofline": roofline,
        "gpu_launches": launches,
        "e2e": {"value": job_value(world, kv_bytes, ms_e2e / args.steps), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": ms_e2e / args.steps,
                "mode": "pipelined: each step's uploads and read-back run on copy streams and "
                        "overlap the neighbouring steps' kernels (throughput, not one step's latency)"},
        "clocks": clock_info,
    }
    if world == 1:
        line["swap"] = measure_swap(pk, w, stream)
    if world == 1 and not args.no_cpu_baseline:
        # the oracle as it stands, on this host's cores: a seeded sample of the
        # batch, stepped repeatedly for about 10 s of CPU time; its rows are
        # also compared with the GPU step's
        threads = cpu_threads()
        sub, n, _, ref = pick_sample(w, target_s=10.0, threads=threads)
        got = step.out.index_select(0, torch.tensor(sub["seqs"], device=dev))
        steps_run, spent = 0, 0.0
        while spent < 10.0 and steps_run < 1000:
            spent += oracle_sample_step(sub, w.scale, threads)[0]
            steps_run += 1
        line["cpu_baseline"] = {"value": sub["kv_bytes"] * steps_run / spent / 1e9, "unit": "GB/s",
                                "cores": threads, "kind": "oracle",
                                "sample": f"{n} of {w.num_seqs} sequences (seeded), all heads; "
                                          f"{steps_run} steps in {spent:.1f} s",
                                "parity": rows_match(got, ref, w.dtype)}
        # and on one core, over a smaller sample (about 3 s)
        sub1, n1, t1, _ = pick_sample(w, target_s=3.0, threads=1)
        line["cpu_baseline"]["value_1_core"] = sub1["kv_bytes"] / t1 / 1e9
        line["cpu_baseline"]["sample_1_core"] = f"{n1} of {w.num_seqs} sequences (seeded), one step"
    configs = [] if args.no_configs or args.workload != "mha" else list(DEFAULT_CONFIGS)
    if configs:
        del step, staged, outs, w
        torch.cuda.empty_cache()
        line["configs"] = {k: measure_config(pk, k, args, world, rank, stream, peak, flush)
                           for k in configs}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="pagedkv", choices=["pagedkv", "reference"])
    ap.add_argument("--workload", default="mha", choices=sorted(WORKLOADS))
    ap.add_argument("--partition-tokens", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cuda-cores", action="store_true",
                    help="decode on the CUDA-core kernel even where a tensor-core one applies")
    ap.add_argument("--schedule", type=int, default=1, choices=[0, 1, 2],
                    help="decode grid schedule: 0 index order, 1 longest first where it pays "
                         "(default), 2 longest first always")
    ap.add_argument("--min-region-s", type=float, default=0.5,
                    help="repeat the timed region of K steps until the repeats span this long")
    ap.add_argument("--no-configs", action="store_true",
                    help="headline workload only (the default mha run also measures "
                         + ", ".join(DEFAULT_CONFIGS) + ")")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_setup(args.gpus, cuda=args.impl != "reference" or torch.cuda.is_available())
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
