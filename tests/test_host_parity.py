"""Host steps of the path (block allocation, slot mapping, super-sequence
offsets) against the oracle: bit-exact on every workload and on random steps."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from paged_kv_cache_469_b200.block_pool import BlockPool, PoolExhausted, plan_step
from paged_kv_cache_469_b200.inputs import WORKLOADS, random_step, workload


def _compare(step):
    bs = step.block_size
    mb = oracle.blocks_needed(int(step.seq_lens.max()), bs)
    plan = plan_step(free_queue=step.free_queue, seq_lens=step.seq_lens,
                     query_lens=step.query_lens, ctx_first_pos=step.ctx_first_pos,
                     ctx_count=step.ctx_count, block_size=bs,
                     shared_prefix_tokens=step.shared_prefix_tokens, max_blocks_per_seq=mb)
    tables, taken = oracle.allocate_block_tables(
        step.free_queue, step.seq_lens, block_size=bs, max_blocks_per_seq=mb,
        shared_prefix_tokens=step.shared_prefix_tokens)
    np.testing.assert_array_equal(plan.block_tables, tables)
    assert plan.blocks_taken == taken
    np.testing.assert_array_equal(plan.query_start_loc, oracle.query_start_loc(step.query_lens))
    np.testing.assert_array_equal(
        plan.slot_mapping,
        oracle.slot_mapping(tables, step.seq_lens - step.query_lens, step.query_lens, bs))
    np.testing.assert_array_equal(
        plan.ctx_slot_mapping,
        oracle.slot_mapping(tables, step.ctx_first_pos, step.ctx_count, bs))
    return plan


@pytest.mark.parametrize("name", WORKLOADS)
def test_workload_host_plan_matches_oracle(name, oracle_lib):
    step = workload(name, with_values=False)
    plan = _compare(step)
    if name == "prefix_decode_llama3_8b":
        assert (plan.block_tables[:, :64] == plan.block_tables[0, :64]).all()


@pytest.mark.parametrize("seed", range(6))
def test_random_host_plan_matches_oracle(seed, oracle_lib):
    _compare(random_step(seed, num_seqs=7, max_ctx=90, max_q=40,
                         shared_prefix_tokens=32 if seed % 2 else 0))


def test_worked_example_and_pool_exhaustion():
    pool = BlockPool(range(3))
    assert pool.allocate_slots("a", 17) == [0, 1]  # 17 tokens -> 2 blocks, queue front
    assert pool.allocate_slots("a", 32) == []  # still fits in 2 blocks
    with pytest.raises(PoolExhausted):
        pool.allocate_slots("b", 33)


@pytest.mark.parametrize("seed", [3, 4])
def test_host_pool_across_steps_matches_oracle_plan_step(seed, oracle_lib):
    """A BlockPool kept across scheduler steps (each step: allocate_slots of
    every sequence's new length, then the table, slots and offsets) gives the
    oracle's plan_step step for step -- the same steps pa_plan_step runs on
    the GPU."""
    from paged_kv_cache_469_b200.block_pool import query_start_loc, slot_mapping
    from paged_kv_cache_469_b200.inputs import planner_draws
    S, mb = 30, 96
    fq, nc, ql = planner_draws(seed, num_seqs=S, num_blocks=5000, max_ctx=600, max_chunk=90,
                               prefill_frac=0.3, idle_frac=0.1)
    pool = BlockPool(fq)
    for s in range(S):
        pool.allocate_slots(s, int(nc[s]))
    tables = pool.block_table(range(S), mb)
    head = len(fq) - len(pool.free_block_queue)
    rng = np.random.default_rng(seed)
    for _ in range(5):
        want = oracle.plan_step(fq, head, tables, nc, ql)
        for s in range(S):
            pool.allocate_slots(s, int(nc[s] + ql[s]))
        tables = pool.block_table(range(S), mb)
        np.testing.assert_array_equal(tables, want[0])
        np.testing.assert_array_equal(slot_mapping(tables, nc, ql), want[3])
        np.testing.assert_array_equal(query_start_loc(ql), want[2])
        head = len(fq) - len(pool.free_block_queue)
        assert head == want[4]
        nc = want[1]
        ql = np.where(rng.random(S) < 0.2, rng.integers(0, 80, S), 1).astype(np.int32)
