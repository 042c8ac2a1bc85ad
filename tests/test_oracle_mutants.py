"""Plant one plausible mistake at a time in a copy of the oracle's C source and
check that the pins of ``test_oracle_pins.py`` catch every one of them.

The mistakes are planted in the oracle, on the CPU, in a temporary build; the
normal oracle library is restored after each case."""
from __future__ import annotations

import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.c")

# (name, exact text in the source, replacement)
MUTANTS = [
    ("ceil_always_rounds_up", "return (num_tokens % block_size == 0) ? whole : whole + 1;",
     "return whole + 1;"),
    ("pops_queue_back", "row[c] = free_queue[head++];",
     "row[c] = free_queue[queue_len - 1 - head++];"),
    ("prefix_not_shared", "for (int64_t c = 0; c < n_prefix; ++c) row[c] = free_queue[c];",
     "for (int64_t c = 0; c < n_prefix; ++c) row[c] = free_queue[head++];"),
    ("slot_offset_off_by_one", "slots[out++] = phys * block_size + offset;",
     "slots[out++] = phys * block_size + (offset + 1) % block_size;"),
    ("cache_write_wrong_head_stride",
     "int64_t dst = (((blk * num_kv_heads + h) * block_size + off) * head_dim + d) *",
     "int64_t dst = (((blk * num_kv_heads + 0) * block_size + off) * head_dim + d) *"),
    ("qsl_inclusive", "query_start_loc[s + 1] = query_start_loc[s] + query_lens[s];",
     "query_start_loc[s + 1] = query_start_loc[s] + query_lens[s] + (s == 0);"),
    ("no_scale", "x[t] = scale * dot;", "x[t] = dot;"),
    ("mask_top_left", "int64_t pos = seq_len - q_len + j;", "int64_t pos = j;"),
    ("mask_excludes_self", "int64_t nkeys = pos + 1;", "int64_t nkeys = pos > 0 ? pos : 1;"),
    ("gqa_interleaved", "int kvh = head / group;", "int kvh = head % num_kv_heads;"),
    ("no_normalisation", "for (int d = 0; d < head_dim; ++d) out_row[d] /= l;",
     "for (int d = 0; d < head_dim; ++d) out_row[d] /= 1.0;"),
    ("v_read_from_k_cache",
     "out_row[d] += x[t] * load_elem(v_cache,", "out_row[d] += x[t] * load_elem(k_cache,"),
    ("block_index_not_through_table",
     "int64_t b = table[t / block_size];\n    int o = (int)(t % block_size);\n    double dot",
     "int64_t b = t / block_size;\n    int o = (int)(t % block_size);\n    double dot"),
    ("bf16_ties_away", "if (frac > 0.5 || (frac == 0.5 && fmod(ip, 2.0) != 0.0)) ip += 1.0;",
     "if (frac >= 0.5) ip += 1.0;"),
    ("plan_overwrites_held_blocks",
     "for (int64_t c = have; c < need; ++c) row[c] = free_queue[next++];",
     "for (int64_t c = 0; c < need - have; ++c) row[c] = free_queue[next++];"),
    ("plan_slots_from_new_length",
     "if (oracle_slot_mapping(block_tables, max_blocks_per_seq, num_seqs, num_computed, "
     "query_lens,",
     "if (oracle_slot_mapping(block_tables, max_blocks_per_seq, num_seqs, seq_lens, "
     "query_lens,"),
    ("plan_head_not_advanced", "  *head = next;\n  return 0;", "  return 0;"),
    ("plan_pool_check_off_by_one", "if (wanted > queue_len - *head || tokens > max_tokens)",
     "if (wanted >= queue_len - *head || tokens > max_tokens)"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new, tmp_path, oracle_lib):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                    "-ffp-contract=off", str(path), "-o", str(lib), "-lm"], check=True)
    oracle.use_library(str(lib))
    try:
        failed = []
        for check in pins.CHECKS:
            try:
                check()
            except Exception:  # an assertion, or the oracle rejecting its own output
                failed.append(check.__name__)
        assert failed, f"no pin caught the planted mistake {name}"
    finally:
        oracle.use_library(None)
