"""Plant plausible mistakes in copies of the oracle; each must trip at least one pin.

Each mutant is a one-line textual change of ``oracle/oracle.c`` (a dropped
term, a wrong index, a wrong sign, a transposed operand), compiled into a
temporary shared object.  The pins of ``oracle_pins`` are then run against it:
if none of them fails, the pins would not have caught that mistake in the
oracle itself.  Everything here runs on the CPU.
"""
import json
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "drop_scale": ("s[j] = scale * acc;", "s[j] = acc;"),
    "gqa_modulo": ("int g = h / G; /* consecutive", "int g = h % H_kv; /* consecutive"),
    "causal_ignores_row": ("int last = ctx_b - q_b + i; /* causal", "int last = ctx_b - q_b; /* causal"),
    "causal_off_by_one": ("int last = ctx_b - q_b + i; /* causal", "int last = ctx_b - q_b + i + 1; /* causal"),
    "page_index_transposed": (
        "const uint16_t *krow = key_cache + ((block * H_kv + g) * ORACLE_BLOCK + off) * d;",
        "const uint16_t *krow = key_cache + ((off * H_kv + g) * ORACLE_BLOCK + block) * d;",
    ),
    "values_from_keys": (
        "const uint16_t *vrow = value_cache + ((block * H_kv + g) * ORACLE_BLOCK + off) * d;",
        "const uint16_t *vrow = key_cache + ((block * H_kv + g) * ORACLE_BLOCK + off) * d;",
    ),
    "no_max_subtraction": ("s[j] = exp(s[j] - m);\n        z += s[j];", "s[j] = exp(s[j]);\n        z += s[j];"),
    "no_normalisation": ("double w = s[j] / z;", "double w = s[j];"),
    "bf16_bias": ("v = ldexp(1.0 + (double)f / 128.0, e - 127);", "v = ldexp(1.0 + (double)f / 128.0, e - 126);"),
    "f16_fraction": ("v = ldexp(1.0 + (double)f / 1024.0, e - 15);", "v = ldexp(1.0 + (double)f / 512.0, e - 15);"),
    "write_offset": (
        "int64_t dst = ((block * H_kv + h) * ORACLE_BLOCK + offset) * d + k;",
        "int64_t dst = ((offset * H_kv + h) * ORACLE_BLOCK + block) * d + k;",
    ),
    "copy_direction": (
        "key_cache[dst * per_block + e] = key_cache[src * per_block + e];",
        "key_cache[src * per_block + e] = key_cache[dst * per_block + e];",
    ),
    "swap_in_reads_keys_for_values": (
        "value_cache[dev * per_block + e] = host_value[hst * per_block + e];",
        "value_cache[dev * per_block + e] = host_key[hst * per_block + e];",
    ),
    "swap_out_wrong_host_block": (
        "host_key[hst * per_block + e] = key_cache[dev * per_block + e];",
        "host_key[dev * per_block + e] = key_cache[dev * per_block + e];",
    ),
    "tree_bit_off_by_one": (
        "return !tree || j < base || ((*tree >> (j - base)) & 1);",
        "return !tree || j < base || ((*tree >> (j - base + 1)) & 1);",
    ),
    "tree_hides_context": (
        "return !tree || j < base || ((*tree >> (j - base)) & 1);",
        "return !tree || ((*tree >> (j - base)) & 1);",
    ),
    "e4m3_bias": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "fp8_scale_constant": ("float sc = amax > 0.0f ? amax / 448.0f : 1.0f;",
                           "float sc = amax > 0.0f ? amax / 240.0f : 1.0f;"),
    "fp8_value_scale_from_keys": ("double w = s[j] / z, vs = value_scale[row];",
                                  "double w = s[j] / z, vs = key_scale[row];"),
    "fp8_value_untransposed": ("out_row[k] += w * (oracle_e4m3_to_f64(vt[k * ORACLE_BLOCK]) * vs);",
                               "out_row[k] += w * (oracle_e4m3_to_f64(vt[k]) * vs);"),
    "online_no_rescale": ("o[c] = alpha * o[c] + acc;", "o[c] = o[c] + acc;"),
    "merge_sign": ("double w = exp(lses[s] - m) / z;", "double w = exp(m - lses[s]) / z;"),
}


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, workdir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    path_c = os.path.join(workdir, f"{name}.c")
    path_so = os.path.join(workdir, f"{name}.so")
    with open(path_c, "w") as f:
        f.write(mutated)
    oracle.build(src=path_c, out=path_so)
    # a child process: a mutant that reads out of bounds may abort, which also counts as caught
    here = os.path.dirname(os.path.abspath(__file__))
    code = (
        "import json, sys; sys.path[:0] = [%r, %r]\n"
        "import oracle\nfrom oracle_pins import ALL_PINS\n"
        "L = oracle.load(%r)\nfailed = []\n"
        "for pin in ALL_PINS:\n"
        "    try:\n        pin(L)\n"
        "    except (AssertionError, ValueError):\n        failed.append(pin.__name__)\n        break\n"
        "print(json.dumps(failed))\n"
    ) % (here, os.path.dirname(here), path_so)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    if r.returncode != 0:
        return  # crashed on a pin: caught
    failed = json.loads(r.stdout.strip().splitlines()[-1])
    assert failed, f"no pin caught the planted mistake {name}"
