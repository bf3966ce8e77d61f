"""Plant plausible mistakes in copies of the oracle and check that the pins catch each one.

Each mutant is the oracle's C source with one textual change (a dropped term,
a wrong index, an off-by-one, a swapped operand), compiled into a temporary
library on the CPU.  The committed oracle is never modified.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    "drop_scale": ("x[j] = scale * dot;", "x[j] = dot;"),
    "group_head_mapping": ("int h = g * group + hh;\n                for (int d = 0; d < head_dim; ++d)\n"
                           "                    qv[d] = load_elem(query, (s *",
                           "int h = hh * num_kv_heads + g;\n                for (int d = 0; d < head_dim; ++d)\n"
                           "                    qv[d] = load_elem(query, (s *"),
    "offset_in_block": ("int64_t offset = j % block_size;", "int64_t offset = 0;"),
    "causal_off_by_one": ("c0 + i + 1,", "c0 + i,"),
    "chunk_start_zero": ("int64_t c0 = len - nq;", "int64_t c0 = 0;"),
    "unnormalised_weights": ("denom += x[j];", "denom += 1.0;"),
    "values_from_keys": ("o[d] += w * Vc[j * head_dim + d];", "o[d] += w * Kc[j * head_dim + d];"),
    "blocks_off_by_one": ("while (covered < num_tokens)", "while (covered <= num_tokens)"),
    "padding_slot_written": ("if (slot < 0) continue;", "if (slot < 0) slot = 0;"),
    "copy_direction": ("memmove((char*)key_caches[l] + dst * block_bytes, (char*)key_caches[l] + src * block_bytes,",
                       "memmove((char*)key_caches[l] + src * block_bytes, (char*)key_caches[l] + dst * block_bytes,"),
    "bf16_shift": ("((uint32_t)h) << 16;", "((uint32_t)h) << 15;"),
    "half_bias": ("expo - 25", "expo - 24"),
    "slot_ignores_table": ("return (int64_t)block_table_row[logical_block] * block_size + offset;",
                           "return logical_block * block_size + offset;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(before, after))
    mutant = oracle.Oracle(oracle.compile_source(str(path), str(tmp_path / f"lib{name}.so")))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin catches mutant {name}"
