"""The oracle against its pins, and the pins against mutated oracles (CPU only)."""
import os
import subprocess
import sys

import pytest

import oracle
from tests import oracle_pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle.default())


# Plausible mistakes, each planted in a copy of the oracle source.  Every one
# must make at least one pin fail (or crash the child process).
MUTANTS = {
    "table_index_uses_modulo": ("int32_t block_id = table[j / block_size];\n        int offset = j % block_size;",
                                "int32_t block_id = table[j % block_size];\n        int offset = j / block_size;"),
    "gqa_head_modulo": ("int kvh = h / group;", "int kvh = h % Hkv;"),
    "scale_dropped": ("scores[j - j0] = scale * dot;", "scores[j - j0] = dot;"),
    "max_not_subtracted": ("scores[j - j0] = exp(scores[j - j0] - m);",
                           "scores[j - j0] = exp(scores[j - j0]);"),
    "normalisation_dropped": ("        o[d] /= l;\n", "\n"),
    "cache_axes_transposed": ("(((int64_t)block_id * block_size + offset) * Hkv + kvh) * D",
                              "(((int64_t)block_id * Hkv + kvh) * block_size + offset) * D"),
    "v_read_from_key_cache": ("const uint16_t *v = value_cache +", "const uint16_t *v = key_cache +"),
    "f16_exponent_bias": ("ldexp((double)(1024 + f), e - 25)", "ldexp((double)(1024 + f), e - 24)"),
    "bf16_exponent_bias": ("ldexp((double)(128 + f), e - 134)", "ldexp((double)(128 + f), e - 133)"),
    "f16_subnormal_scale": ("ldexp((double)f, -24)", "ldexp((double)f, -25)"),
    "write_offset_swapped": ("int64_t offset = slot % block_size;", "int64_t offset = slot / block_size;"),
    "write_skips_slot_zero": ("if (slot < 0)\n            continue;", "if (slot <= 0)\n            continue;"),
    "write_value_from_key": ("value_cache[dst + d] = value[src + d];", "value_cache[dst + d] = key[src + d];"),
    "merge_drops_partition_sum": ("double w = exp(mr[p] - M) * lr[p];", "double w = exp(mr[p] - M);"),
    "copy_uses_dst_index_for_src": ("const uint16_t *src = src_cache + (int64_t)mapping[2 * i] * block_elems;",
                                    "const uint16_t *src = src_cache + (int64_t)mapping[2 * i + 1] * block_elems;"),
    "prefill_not_causal": ("                     block_tables + (int64_t)b * max_blocks, h, 0, p + 1, Hq, Hkv, D,",
                           "                     block_tables + (int64_t)b * max_blocks, h, 0, context_lens[b], Hq, Hkv, D,"),
    "prefill_off_by_one": ("int p = context_lens[b] - C + i;", "int p = context_lens[b] - C + i - 1;"),
    "merge_sign_flipped": ("double w = exp(mr[p] - M) * lr[p];", "double w = exp(M - mr[p]) * lr[p];"),
}

_CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import oracle
from tests import oracle_pins
orc = oracle.Oracle({lib!r})
for pin in oracle_pins.ALL_PINS:
    try:
        pin(orc)
    except Exception as e:
        print("KILLED by", pin.__name__, type(e).__name__)
        sys.exit(0)
print("SURVIVED")
sys.exit(3)
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "pkv_oracle.c")).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    path = tmp_path / "mutant.c"
    path.write_text(mutated)
    lib = oracle.compile_source(str(path), str(tmp_path / "libmutant.so"))
    r = subprocess.run([sys.executable, "-c", _CHILD.format(root=ROOT, lib=lib)],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 3, f"mutant {name} survived every pin:\n{r.stdout}{r.stderr}"
