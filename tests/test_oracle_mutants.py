"""Plant plausible mistakes in the oracle's C source and check that the pins in
tests/test_oracle.py and tests/test_oracle_multi_query.py catch every one.

Each mutant is one textual edit of oracle/pa_oracle.c (a wrong head mapping, a
dropped scale, a transposed pool layout, ...).  It is compiled with gcc into a
temporary library and the pin suite runs against it in a child process (so a
mutant that misbehaves cannot disturb this process).  CPU only.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "pa_oracle.c")

MUTANTS = {
    "gqa_mapping_modulo": ("const int kv = h / G;",
                           "const int kv = h % job->num_kv_heads;"),
    "block_offset_off_by_one": ("int off = t % job->block_size;",
                                "int off = (t + 1) % job->block_size;"),
    "scale_dropped": ("z[t] = job->scale * dot;", "z[t] = dot;"),
    "normalisation_dropped": ("o[d] /= wsum;", "o[d] /= 1.0;"),
    "softmax_sign_flipped": ("z[t] = exp(z[t] - zmax);",
                             "z[t] = exp(zmax - z[t]);"),
    "last_token_dropped": ("const int L = job->context_lens[s];",
                           "const int L = job->context_lens[s] - 1;"),
    "pool_layout_head_major": (
        "return ((blk * block_size + off) * num_kv_heads + head) * head_size + d;",
        "return ((blk * num_kv_heads + head) * block_size + off) * head_size + d;"),
    "query_uses_kv_head": (
        "job->q + ((int64_t)s * job->num_heads + h) * D;",
        "job->q + ((int64_t)s * job->num_heads + kv) * D;"),
    "values_read_from_keys": (
        "o[d] += z[t] * bf16_bits_to_double(job->v_cache[idx]);",
        "o[d] += z[t] * bf16_bits_to_double(job->k_cache[idx]);"),
    "bf16_widening_shift": ("((uint32_t)bits) << 16;", "((uint32_t)bits) << 15;"),
    "cache_write_key_value_swapped": (
        "k_cache[dst] = key[(int64_t)i * key_token_stride +",
        "k_cache[dst] = value[(int64_t)i * value_token_stride +"),
    "padding_rule_includes_slot_zero": ("if (slot < 0) continue;",
                                        "if (slot <= 0) continue;"),
    "causal_limit_off_by_one": ("const int last = L - k + j;",
                                "const int last = L - k + j - 1;"),
    "query_row_not_advanced": (
        "const uint16_t* qv = job->q + ((int64_t)(q0 + j) * job->num_heads + h) * D;",
        "const uint16_t* qv = job->q + ((int64_t)(q0) * job->num_heads + h) * D;"),
    "query_count_off_by_one": ("const int k = job->query_start_loc[s + 1] - q0;",
                               "const int k = job->query_start_loc[s + 1] - q0 - 1;"),
    "swap_direction_reversed": (
        "memcpy(dst_caches[c] + dst * block_bytes,\n                   src_caches[c] + src * block_bytes, (size_t)block_bytes);",
        "memcpy(dst_caches[c] + src * block_bytes,\n                   src_caches[c] + dst * block_bytes, (size_t)block_bytes);"),
    "copy_direction_swapped": (
        "int64_t src = block_mapping[2 * p];\n        int64_t dst = block_mapping[2 * p + 1];",
        "int64_t src = block_mapping[2 * p + 1];\n        int64_t dst = block_mapping[2 * p];"),
}


def _compile(src_text: str, workdir: str, name: str) -> str:
    c = os.path.join(workdir, name + ".c")
    so = os.path.join(workdir, name + ".so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread",
                    c, "-o", so, "-lm"], check=True)
    return so


def _run_pins(lib_path: str) -> int:
    env = dict(os.environ, PA_ORACLE_LIB=lib_path)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q",
                        "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py"),
                        os.path.join(ROOT, "tests", "test_oracle_multi_query.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return r.returncode


def test_pins_catch_every_planted_mistake():
    with open(SRC) as f:
        original = f.read()
    with tempfile.TemporaryDirectory() as tmp:
        jobs = {"unmutated": _compile(original, tmp, "unmutated")}
        for name, (old, new) in MUTANTS.items():
            assert original.count(old) >= 1, f"mutant {name}: pattern not found"
            jobs[name] = _compile(original.replace(old, new), tmp, name)
        workers = max(1, min(8, len(os.sched_getaffinity(0))))
        with cf.ThreadPoolExecutor(workers) as ex:
            rcs = dict(zip(jobs, ex.map(_run_pins, jobs.values())))
    assert rcs.pop("unmutated") == 0, "pins fail on the unmutated oracle"
    survivors = [n for n, rc in rcs.items() if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
