"""Every plausible mistake planted in the oracle must fail at least one pin.

Each mutant is a copy of ``oracle/pa_oracle.c`` with one textual change
(a dropped term, a wrong sign, a wrong index or layout, a transposed
operand), compiled with gcc into a temporary library and run against the pin
suite.  A mutant that passes every pin would mean the pins cannot tell that
mistake from the correct oracle.  Only the CPU oracle is mutated.

The pins run in a child process: a mutant with a wrong index may read or
write out of bounds, and a crash there must not take the test run with it.
A crashed child counts as a caught mutant (it did not pass the pins).
"""
import os
import subprocess
import sys

import pytest

import oracle

_CHILD = """
import sys
sys.path[:0] = [{tests!r}, {root!r}]
import oracle
from pins import ALL_PINS
orc = oracle.load({lib!r})
for pin in ALL_PINS:
    try:
        pin(orc)
    except (AssertionError, oracle.OracleError):
        print("CAUGHT", pin.__name__)
        sys.exit(0)
print("PASSED_ALL")
"""

SRC = os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.c")

ROW = "((blk * num_kv_heads + kvh) * block_size + j % block_size) * head_dim"
MUTANTS = {
    "drop_scale": ("x[j] = scale * dot;", "x[j] = dot;"),
    "gqa_head_map": ("const int32_t kvh = h / group;", "const int32_t kvh = h % num_kv_heads;"),
    "table_index_shift": ("block_tables[(int64_t)s * max_blocks_per_seq + j / block_size]",
                          "block_tables[(int64_t)s * max_blocks_per_seq + (j / block_size + 1) % "
                          "max_blocks_per_seq]"),
    "token_major_layout": (ROW, "((blk * block_size + j % block_size) * num_kv_heads + kvh) * head_dim"),
    "no_max_subtraction": ("x[j] = exp(x[j] - m);", "x[j] = exp(x[j]);"),
    "exp_sign": ("x[j] = exp(x[j] - m);", "x[j] = exp(m - x[j]);"),
    "normalise_by_length": ("double w = x[j] / z;", "double w = x[j] / n;"),
    "read_past_length": ("const int32_t n = context_lens[s];",
                         "const int32_t n = context_lens[s] + (context_lens[s] % block_size != 0);"),
    "f16_exponent_bias": ("e - 25);", "e - 24);"),
    "f16_subnormal_scale": ("ldexp((double)m, -24)", "ldexp((double)m, -25)"),
    "bf16_shift": ("(uint32_t)h << 16;", "(uint32_t)h << 15;"),
    "values_from_key_cache": ("o[d] += w * widen(v_cache[row + d], dtype);",
                              "o[d] += w * widen(k_cache[row + d], dtype);"),
    "query_head_zero": ("qd[d] = widen(q[p * head_dim + d], dtype);",
                        "qd[d] = widen(q[(p - h) * head_dim + d], dtype);"),
    "max_not_updated": ("if (x[j] > m) m = x[j];", "if (x[j] < m) m = x[j];"),
    "write_slot_shift": ("int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;",
                         "int64_t dst = ((blk * num_kv_heads + h) * block_size + (off + 1) % block_size)"
                         " * head_dim;"),
    "write_key_into_value": ("v_cache[dst + d] = value[src + d];", "v_cache[dst + d] = key[src + d];"),
    "copy_only_k": ("memmove(v_caches[l] + dst * elems, v_caches[l] + src * elems, sizeof(uint16_t) * elems);",
                    ""),
    "copy_reversed": ("memmove(k_caches[l] + dst * elems, k_caches[l] + src * elems",
                      "memmove(k_caches[l] + src * elems, k_caches[l] + dst * elems"),
    "swap_only_k": ("memcpy(dst_v + dst * elems, src_v + src * elems, sizeof(uint16_t) * elems);", ""),
    "swap_direction": ("memcpy(dst_k + dst * elems, src_k + src * elems", "memcpy(dst_k + src * elems, src_k + dst * elems"),
    "e4m3_exponent_bias": ("v = ldexp((double)(m + 8), e - 10);", "v = ldexp((double)(m + 8), e - 9);"),
    "e4m3_ties_to_odd": ("(err == best_err && (c & 1) == 0)", "(err == best_err && (c & 1) == 1)"),
    "e4m3_subnormal_scale": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "e4m3_zero_sign_dropped": ("(signbit(y) ? 0x80 : 0)", "(y < 0 ? 0x80 : 0)"),
    "fp8_k_scale_dropped": ("* (widen_e4m3(k_cache[row + d]) * k_scale);", "* widen_e4m3(k_cache[row + d]);"),
    "fp8_scales_swapped": ("o[d] += w * (widen_e4m3(v_cache[row + d]) * v_scale);",
                           "o[d] += w * (widen_e4m3(v_cache[row + d]) * k_scale);"),
    "fp8_write_scale_multiplied": ("quantize_e4m3((float)widen(key[src + d], dtype) / k_scale, &tab)",
                                   "quantize_e4m3((float)widen(key[src + d], dtype) * k_scale, &tab)"),
    "ext_window_off_by_one": ("const int32_t lo = window > 0 && hi - window + 1 > 0 ? hi - window + 1 : 0;",
                              "const int32_t lo = window > 0 && hi - window > 0 ? hi - window : 0;"),
    "ext_window_ignored": ("const int32_t lo = window > 0 && hi - window + 1 > 0 ? hi - window + 1 : 0;",
                           "const int32_t lo = 0;"),
    "ext_causal_shift": ("const int32_t hi = context_lens[s] - q_len + i;",
                         "const int32_t hi = context_lens[s] - q_len + i - (i > 0);"),
    "ext_first_query_row_for_all": ("qd[d] = widen(q[r * head_dim + d], dtype);",
                                    "qd[d] = widen(q[(r - (int64_t)i * num_heads) * head_dim + d], dtype);"),
    "ext_k_scale_dropped": ("dot += qd[d] * (kv * k_scale);", "dot += qd[d] * kv;"),
    "ext_v_scale_dropped": ("o[d] += w * (vv * v_scale);", "o[d] += w * vv;"),
    "zero_length_not_zeroed": ("for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;\n        if (n == 0) continue;",
                               "if (n == 0) { o[0] = 1.0; continue; }\n        "
                               "for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;"),
}


def _run_mutant(name: str, workdir: str) -> tuple:
    """Build mutant `name` and run the pins on it in a child process:
    returns (returncode, stdout, stderr)."""
    old, new = MUTANTS[name]
    src = open(SRC).read()
    if old not in src:
        return (None, "", f"mutant {name}: pattern no longer in the oracle source")
    path = os.path.join(workdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.build(path, os.path.join(workdir, f"lib{name}.so"))
    tests = os.path.dirname(os.path.abspath(__file__))
    code = _CHILD.format(tests=tests, root=os.path.dirname(tests), lib=lib)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600,
                       env={**os.environ, "OMP_NUM_THREADS": "2"})
    return (r.returncode, r.stdout, r.stderr)


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Every mutant's child run, several at once (each in its own process)."""
    import concurrent.futures as cf
    workdir = str(tmp_path_factory.mktemp("mutants"))
    jobs = max(1, min(8, (os.cpu_count() or 2) // 2))
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        futs = {name: ex.submit(_run_mutant, name, workdir) for name in MUTANTS}
        return {name: f.result() for name, f in futs.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, mutant_results):
    rc, out, err = mutant_results[name]
    assert rc is not None, err
    if rc < 0:
        return  # killed by a signal (an out-of-bounds access): caught
    assert rc == 0, err[-2000:]
    assert "PASSED_ALL" not in out, f"mutant {name} passed every pin"
