"""The expected values of the GPU step planner (oracle_plan_step, a composition
of oracle functions) pinned on the CPU against allocate_slots walked by hand.

Page "LLM推論エンジンvLLMの内部構造を徹底解説", section "PagedAttentionの仕組み":
a request of n tokens holds one block per started group of 16 tokens;
allocate_slots gives a request the blocks it still lacks, taken one by one
from the front of free_block_queue, requests in order; the token at position
p sits at offset p % 16 of the request's block p // 16.  The walk below does
exactly that with a Python list, token by token, with no block arithmetic
shared with the oracle.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from paged_kv_cache_469_b200.inputs import planner_draws
from tests.oracle_side import oracle_plan_step

PAD = -3


def hand_walk(free_queue, steps):
    """Per step: (rows, seq_lens, query_start_loc, slots, head) from a plain walk."""
    queue = [int(b) for b in free_queue]
    taken = 0
    rows: dict = {}
    for num_computed, query_lens in steps:
        seq_lens, qsl, slots = [], [0], []
        for s in range(len(query_lens)):
            row = rows.setdefault(s, [])
            length = int(num_computed[s]) + int(query_lens[s])
            started = 0
            for t in range(length):  # one block per started group of 16 tokens
                if t % 16 == 0:
                    started += 1
            while len(row) < started:
                row.append(queue[taken])
                taken += 1
            seq_lens.append(length)
            qsl.append(qsl[-1] + int(query_lens[s]))
            for j in range(int(query_lens[s])):
                p = int(num_computed[s]) + j
                slots.append(row[p // 16] * 16 + p % 16)
        yield ({s: list(r) for s, r in rows.items()}, np.array(seq_lens), np.array(qsl),
               np.array(slots, dtype=np.int64), taken)


def _rows_match(tables, rows):
    for s, r in rows.items():
        assert tables[s, :len(r)].tolist() == r, f"row {s}"
        assert (tables[s, len(r):] == PAD).all(), f"row {s} written past its blocks"


@pytest.mark.parametrize("S", [1, 6, 57])
def test_fresh_step_is_the_whole_allocation(S, oracle_lib):
    fq, _, ql = planner_draws(100 + S, num_seqs=S, num_blocks=5000, max_ctx=0, max_chunk=300,
                              prefill_frac=0.6)
    tables = np.full((S, 32), PAD, np.int32)
    nc = np.zeros(S, np.int32)
    got = oracle_plan_step(fq, 0, tables, nc, ql, pad_value=PAD)
    whole, taken = oracle.allocate_block_tables(fq, ql, max_blocks_per_seq=32, pad_value=PAD)
    np.testing.assert_array_equal(got[0], whole)
    assert got[4] == taken
    (rows, sl, qsl, slots, head), = hand_walk(fq, [(nc, ql)])
    _rows_match(got[0], rows)
    np.testing.assert_array_equal(got[3], slots)
    np.testing.assert_array_equal(got[2], qsl)
    assert got[4] == head


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_chained_steps_follow_the_hand_walk(seed, oracle_lib):
    """A context allocation, then five steps of decodes, chunks and idle
    sequences, each starting where the previous one left the queue."""
    S = 23
    fq, nc0, ql = planner_draws(seed, num_seqs=S, num_blocks=4000, max_ctx=300, max_chunk=70,
                                prefill_frac=0.3, idle_frac=0.2)
    rng = np.random.default_rng(seed)
    steps = [(np.zeros(S, np.int32), nc0)]
    nc = nc0
    for _ in range(5):
        steps.append((nc, ql))
        nc = (nc + ql).astype(np.int32)
        ql = np.where(rng.random(S) < 0.3, rng.integers(0, 50, S), 1).astype(np.int32)
    tables = np.full((S, 64), PAD, np.int32)
    head = 0
    for (num_computed, query_lens), walk in zip(steps, hand_walk(fq, steps)):
        tables, sl, qsl, slots, head = oracle_plan_step(fq, head, tables, num_computed,
                                                        query_lens, pad_value=PAD)
        rows, w_sl, w_qsl, w_slots, w_head = walk
        _rows_match(tables, rows)
        np.testing.assert_array_equal(sl, w_sl)
        np.testing.assert_array_equal(qsl, w_qsl)
        np.testing.assert_array_equal(slots, w_slots)
        assert head == w_head


def test_step_invariants(oracle_lib):
    """Slots of one step are distinct; each lies in a block of its own
    sequence's row; the blocks a step appends are the queue entries it took."""
    S = 40
    fq, nc, ql = planner_draws(9, num_seqs=S, num_blocks=6000, max_ctx=500, max_chunk=100,
                               prefill_frac=0.4)
    tables0, head0 = oracle.allocate_block_tables(fq, nc, max_blocks_per_seq=64, pad_value=PAD)
    tables, _, qsl, slots, head = oracle_plan_step(fq, head0, tables0, nc, ql, pad_value=PAD)
    assert len(set(slots.tolist())) == len(slots)
    for s in range(S):
        own = set(tables[s][tables[s] != PAD].tolist())
        assert {int(x) // 16 for x in slots[qsl[s]:qsl[s + 1]]} <= own
    appended = sorted(set(tables[tables != PAD].tolist()) - set(tables0[tables0 != PAD].tolist()))
    assert appended == sorted(fq[head0:head].tolist())
