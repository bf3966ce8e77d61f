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
    "group_head_mapping": ("int h = g * group + hh;\n            for (int d = 0; d < head_dim; ++d)\n"
                           "                qv[d] = load_elem(query, (s *",
                           "int h = hh * num_kv_heads + g;\n            for (int d = 0; d < head_dim; ++d)\n"
                           "                qv[d] = load_elem(query, (s *"),
    "offset_in_block": ("int64_t offset = j % block_size;", "int64_t offset = 0;"),
    "causal_off_by_one": ("c0 + i + 1,", "c0 + i,"),
    "chunk_start_zero": ("int64_t c0 = len - nq;", "int64_t c0 = 0;"),
    "unnormalised_weights": ("denom += x[j];", "denom += 1.0;"),
    "values_from_keys": ("o[d] += w * Vc[j * head_dim + d];", "o[d] += w * Kc[j * head_dim + d];"),
    "blocks_off_by_one": ("while (covered < num_tokens)", "while (covered <= num_tokens)"),
    "padding_slot_written": ("if (slot < 0) continue;", "if (slot < 0) slot = 0;", 0),
    "fp8_padding_slot_written": ("if (slot < 0) continue;", "if (slot < 0) slot = 0;", 1),
    "copy_direction": ("memmove((char*)key_caches[l] + dst * block_bytes, (char*)key_caches[l] + src * block_bytes,",
                       "memmove((char*)key_caches[l] + src * block_bytes, (char*)key_caches[l] + dst * block_bytes,"),
    "bf16_shift": ("((uint32_t)h) << 16;", "((uint32_t)h) << 15;"),
    "half_bias": ("expo - 25", "expo - 24"),
    "e4m3_bias": ("expo - 10);   /* 1.mant", "expo - 9);   /* 1.mant"),
    "e4m3_subnormal_scale": ("ldexp((double)mant, -9);", "ldexp((double)mant, -10);"),
    "e4m3_ties_to_odd": ("(err == best_err && (c & 1) == 0)", "(err == best_err && (c & 1) == 1)"),
    "e4m3_max_value_missed": ("for (int c = 0; c <= 0x7E; ++c)", "for (int c = 0; c < 0x7E; ++c)"),
    "fp8_k_scale_dropped": ("Kc[j * head_dim + d] = k_scale * load_elem(", "Kc[j * head_dim + d] = load_elem("),
    "fp8_quantise_multiplies": ("load_elem(key, src, src_dtype) / k_scale", "load_elem(key, src, src_dtype) * k_scale"),
    "fp8_v_scale_on_keys": ("Vc[j * head_dim + d] = v_scale *", "Vc[j * head_dim + d] = k_scale *"),
    "slot_ignores_table": ("return (int64_t)block_table_row[logical_block] * block_size + offset;",
                           "return logical_block * block_size + offset;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    before, after, *which = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    if which:  # the anchor occurs more than once: mutate occurrence number which[0]
        parts = src.split(before)
        k = which[0]
        assert len(parts) > k + 1, f"mutation anchor for {name} has no occurrence {k}"
        mutated = before.join(parts[:k + 1]) + after + before.join(parts[k + 1:])
    else:
        assert src.count(before) == 1, f"mutation anchor for {name} not unique"
        mutated = src.replace(before, after)
    path = tmp_path / f"{name}.c"
    path.write_text(mutated)
    mutant = oracle.Oracle(oracle.compile_source(str(path), str(tmp_path / f"lib{name}.so")))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin catches mutant {name}"
