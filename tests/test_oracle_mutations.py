"""Plant plausible slips in a copy of the oracle's C source and check that each
one fails at least one pin. The mutants are built and run on the CPU only."""
import os
import shutil
import tempfile

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.c")

# (name, original text, replacement)
MUTANTS = [
    ("dropped scale", "w[t] = scale * dot;", "w[t] = dot;"),
    ("sign of the score", "dot += qd[i] * K[(size_t)t * head_dim + i];",
     "dot -= qd[i] * K[(size_t)t * head_dim + i];"),
    ("kv-head grouping", "const int32_t kh = h / group;", "const int32_t kh = h % num_kv_heads;"),
    ("block / offset swapped", "int32_t phys = table_row[t / block_size];",
     "int32_t phys = table_row[t % block_size];"),
    ("layout transposed in decode",
     "int64_t base = (((int64_t)phys * num_kv_heads + kh) * block_size + t % block_size) *",
     "int64_t base = (((int64_t)phys * block_size + t % block_size) * num_kv_heads + kh) *"),
    ("layout transposed in append",
     "size_t dst = (((size_t)block * num_kv_heads + h) * block_size + offset) * vec;",
     "size_t dst = (((size_t)block * block_size + offset) * num_kv_heads + h) * vec;"),
    ("context off by one", "context_lens[s], s, h,", "context_lens[s] - (context_lens[s] > 1), s, h,"),
    ("no max shift", "w[t] = exp(w[t] - m);", "w[t] = exp(w[t]);"),
    ("bf16 widening", "u = ((uint32_t)h) << 16;", "u = ((uint32_t)h) << 15;"),
    ("normalisation", "o[i] /= l;", "o[i] /= (l + 1e-3);"),
    ("copy direction", "size_t src = (size_t)pairs[2 * p] * block_bytes;",
     "size_t src = (size_t)pairs[2 * p + 1] * block_bytes;"),
    ("padding test", "if (slot < 0) continue;", "if (slot <= 0) continue;"),
    ("causal end", "int32_t pos = context_lens[s] - n + (row - query_start[s]);",
     "int32_t pos = context_lens[s] - n + (row - query_start[s]) - (n > 1);"),
    ("e4m3 exponent bias", "else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("int8 rounding", "return (int8_t)lrintf(c);", "return (int8_t)c;"),
    ("quant tie break", "(err == best_err && (c & 1) == 0)", "(err == best_err && (c & 1) == 1)"),
    ("k scale dropped", "load_elem(k_cache, base + i, dtype) * ks;", "load_elem(k_cache, base + i, dtype);"),
    ("swap K from V", "memcpy((char*)dst_k + to, (const char*)src_k + from, block_bytes);",
     "memcpy((char*)dst_k + to, (const char*)src_v + from, block_bytes);"),
    ("query row", "qd[i] = load_elem(q, ((int64_t)s * num_heads + h) * head_dim + i, q_dtype);",
     "qd[i] = load_elem(q, ((int64_t)s * num_heads + (h / group) * group) * head_dim + i, q_dtype);"),
]

PINS = [
    pins.test_golden_append_layout,
    pins.test_golden_block_copy,
    lambda: pins.test_block_table_worked_example(40),
    pins.test_golden_closed_form,
    lambda: pins.test_decode_equals_contiguous_sdpa("bf16", 16, 8, 2),
    lambda: pins.test_decode_equals_contiguous_sdpa("f32", 2, 4, 4),
    pins.test_large_logits_stable,
    pins.test_bf16_widening_known_bits,
    pins.test_zero_query_gives_mean_of_v,
    pins.test_prefix_sharing_bitwise,
    pins.test_tiny_workload_step_matches_sdpa,
    pins.test_block_swap_equals_indexed_assignment,
    lambda: pins.test_decode_multi_equals_masked_sdpa("bf16", 16, 8, 2),
    pins.test_e4m3_values_match_torch_for_every_code,
    pins.test_e4m3_encoding_matches_torch_round_to_nearest_even,
    pins.test_int8_codes,
    lambda: pins.test_decode_quant_equals_sdpa_on_dequantised_values("fp8", 16, 8, 2),
]


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mut_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def test_unmutated_source_passes_all_pins(workdir):
    lib = oracle.compile_source(SRC, os.path.join(workdir, "orig.so"))
    with oracle.use_library(lib):
        for pin in PINS:
            pin()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_fails_a_pin(workdir, name, old, new):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    path = os.path.join(workdir, name.replace(" ", "_").replace("/", "_") + ".c")
    with open(path, "w", encoding="utf-8") as f:
        f.write(src.replace(old, new))
    lib = oracle.compile_source(path, path[:-2] + ".so")
    failed = []
    with oracle.use_library(lib):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, oracle.OracleError):
                failed.append(getattr(pin, "__name__", "pin"))
    assert failed, f"mutant '{name}' passed every pin"
