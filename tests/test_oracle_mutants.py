"""Planted mistakes in copies of the CPU oracle must each fail at least one pin.

Every mutant below is a plausible slip in the oracle (a dropped term, a wrong
sign, index or operand, a wrong conversion).  Each is compiled from a copy of
``oracle/pkv_oracle.c`` with one text substitution, loaded in a child process
(a mutant may crash; that counts as caught) and run against the pins of
``oracle_pins.py``.  The real oracle is never modified.
"""
from __future__ import annotations

import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "pkv_oracle.c")

MUTANTS = {
    "dropped_scale": ("x[t] = scale * acc;", "x[t] = acc;"),
    "exp_sign": ("x[t] = exp(x[t] - m);", "x[t] = exp(m - x[t]);"),
    "no_max_shift": ("double m = x[0];\n    for (int t = 1; t < L; ++t)\n        if (x[t] > m) m = x[t];",
                     "double m = 0.0;"),
    "no_normalise": ("double w = x[t] / Z;", "double w = x[t];"),
    "k_for_v": ("o[d] += w * Vc[(int64_t)t * D + d];", "o[d] += w * Kc[(int64_t)t * D + d];"),
    "block_index": ("max_blocks_per_seq + t / block_size];", "max_blocks_per_seq + t / (block_size + 1)];"),
    "slot_index": ("int slot = t % block_size;", "int slot = (t + 1) % block_size;"),
    "gqa_map": ("const int g = h / group;\n    const int L", "const int g = h % job->num_kv_heads;\n    const int L"),
    "q_row": ("((int64_t)s * job->num_heads + h) * D + d", "((int64_t)s * job->num_heads) * D + d"),
    "last_token_dropped": ("for (int t = 0; t < L; ++t) {\n        double acc",
                           "for (int t = 0; t < L; ++t) {\n        if (t == L - 1 && L > 1) { x[t] = -1e300; continue; }\n        double acc"),
    "bf16_widen": ("((uint32_t)bits16) << 16", "((uint32_t)bits16) << 15"),
    "blocks_needed": ("return (L + bs - 1) / bs;", "return L / bs + 1;"),
    "append_slot": ("int64_t blk = slot / block_size, off = slot % block_size;",
                    "int64_t blk = slot / block_size, off = (slot + 1) % block_size;"),
    "append_skip": ("if (slot < 0) continue;", "if (slot < 0) slot = 0;"),
    "append_head": ("int64_t src = ((int64_t)i * num_kv_heads + g) * row_bytes;",
                    "int64_t src = ((int64_t)i * num_kv_heads) * row_bytes;"),
    "copy_direction": ("int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];",
                       "int64_t dst = pairs[2 * i], src = pairs[2 * i + 1];"),
    "copy_one_head": ("(int64_t)num_kv_heads * block_size * head_dim * elem_bytes(dtype);",
                      "(int64_t)block_size * head_dim * elem_bytes(dtype);"),
    "swap_direction": ("memcpy((char*)dst_k + dst * block_bytes, (const char*)src_k + src * block_bytes,",
                       "memcpy((char*)dst_k + src * block_bytes, (const char*)src_k + dst * block_bytes,"),
    "e4m3_subnormal": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "e4m3_bias": ("v = ldexp(8.0 + m, e - 10);", "v = ldexp(8.0 + m, e - 9);"),
    "e4m3_tie_odd": ("(err == best_err && (c & 1) == 0 && (best & 1) == 1)",
                     "(err == best_err && (c & 1) == 1 && (best & 1) == 0)"),
    "e4m3_no_saturation": ("if (a >= 448.0) return sign | 0x7E;", "if (a >= 448.0) return sign | 0x7F;"),
    "fp8_k_scale_dropped": ("Kc[(int64_t)t * D + d] = oracle_e4m3_value(k_cache[row + d]) * (double)k_scales[g];",
                            "Kc[(int64_t)t * D + d] = oracle_e4m3_value(k_cache[row + d]);"),
    "fp8_v_uses_k_scale": ("Vc[(int64_t)t * D + d] = oracle_e4m3_value(v_cache[row + d]) * (double)v_scales[g];",
                           "Vc[(int64_t)t * D + d] = oracle_e4m3_value(v_cache[row + d]) * (double)k_scales[g];"),
    "fp8_gqa_map": ("const int g = h / group; /* contiguous query-head groups */",
                    "const int g = h % num_kv_heads; /* contiguous query-head groups */"),
    "fp8_block_index": ("const int32_t blk = table_row[t / block_size];",
                        "const int32_t blk = table_row[t / (block_size + 1)];"),
    "fp8_append_multiplies": ("k_cache[dst + d] = oracle_e4m3_encode(kx / k_scales[g]);",
                              "k_cache[dst + d] = oracle_e4m3_encode(kx * k_scales[g]);"),
    "physical_double_count": ("if (here > filled[p]) filled[p] = (int32_t)here;",
                              "filled[p] += (int32_t)here;"),
}

CHILD = r"""
import sys, traceback
sys.path.insert(0, {root!r}); sys.path.insert(0, {here!r})
import oracle
from oracle import binding
binding.use_library(binding.open_library({lib!r}))
import oracle_pins
failed = []
for pin in oracle_pins.PINS:
    try:
        pin()
    except Exception:
        failed.append(pin.__name__)
print("FAILED_PINS", ",".join(failed))
"""


def _run_mutant(name: str, tmp: str) -> tuple[str, bool, str]:
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique in the oracle"
    msrc = os.path.join(tmp, f"mut_{name}.c")
    with open(msrc, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(tmp, f"libmut_{name}.so")
    from oracle.binding import compile_source

    compile_source(msrc, lib)
    code = CHILD.format(root=ROOT, here=HERE, lib=lib)
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    if p.returncode != 0:
        return name, True, f"child exited {p.returncode}"
    line = [x for x in p.stdout.splitlines() if x.startswith("FAILED_PINS")][-1]
    failed = line.split(" ", 1)[1] if " " in line else ""
    return name, bool(failed.strip()), failed


def test_every_mutant_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda n: _run_mutant(n, tmp), sorted(MUTANTS)))
    missed = [n for n, caught, _ in results if not caught]
    assert not missed, f"pins did not catch: {missed}"


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutation_site_exists(name):
    assert open(SRC).read().count(MUTANTS[name][0]) == 1
