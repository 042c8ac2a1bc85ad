"""Oracle-side view of a step: block tables, cache and outputs built ONLY with
``oracle`` functions from the seeded draws of ``paged_kv_cache_469_b200.inputs``.

Test infrastructure (imports the oracle; the product never imports this)."""
from __future__ import annotations

import numpy as np

import oracle
from paged_kv_cache_469_b200.inputs import StepInputs, bf16_bits_to_f32


def oracle_state(step: StepInputs, max_blocks_per_seq: int | None = None, pad_value: int = 0):
    bs = step.block_size
    if max_blocks_per_seq is None:
        max_blocks_per_seq = max(1, oracle.blocks_needed(int(step.seq_lens.max()), bs))
    tables, taken = oracle.allocate_block_tables(
        step.free_queue, step.seq_lens, block_size=bs, max_blocks_per_seq=max_blocks_per_seq,
        shared_prefix_tokens=step.shared_prefix_tokens, pad_value=pad_value)
    qsl = oracle.query_start_loc(step.query_lens)
    new_slots = oracle.slot_mapping(tables, step.seq_lens - step.query_lens, step.query_lens, bs)
    ctx_slots = oracle.slot_mapping(tables, step.ctx_first_pos, step.ctx_count, bs)
    shape = (step.num_blocks, step.num_kv_heads, bs, step.head_dim)
    kc = np.zeros(shape, dtype=step.k_new.dtype)
    vc = np.zeros(shape, dtype=step.k_new.dtype)
    oracle.reshape_and_cache(step.k_ctx, step.v_ctx, kc, vc, ctx_slots)
    oracle.reshape_and_cache(step.k_new, step.v_new, kc, vc, new_slots)
    return dict(block_tables=tables, blocks_taken=taken, query_start_loc=qsl,
                slot_mapping=new_slots, ctx_slot_mapping=ctx_slots, k_cache=kc, v_cache=vc)


def oracle_outputs(step: StepInputs, state=None, num_threads: int = 1) -> np.ndarray:
    st = state or oracle_state(step)
    return oracle.paged_attention(step.q, st["k_cache"], st["v_cache"], st["block_tables"],
                                  step.seq_lens, st["query_start_loc"],
                                  num_q_heads=step.num_q_heads, scale=step.scale,
                                  num_threads=num_threads)


def as_f64(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def contiguous_kv(step: StepInputs, s: int):
    """Sequence s's K and V for positions 0..L-1, [L, Hkv, D] in fp64, assembled from
    the drawn rows without any block table (context rows, then the new rows)."""
    ctx_off = np.concatenate([[0], np.cumsum(step.ctx_count)]).astype(np.int64)
    q_off = np.concatenate([[0], np.cumsum(step.query_lens)]).astype(np.int64)
    parts_k, parts_v = [], []
    if step.shared_prefix_tokens and s > 0:
        parts_k.append(step.k_ctx[0:step.shared_prefix_tokens])
        parts_v.append(step.v_ctx[0:step.shared_prefix_tokens])
    parts_k.append(step.k_ctx[ctx_off[s]:ctx_off[s + 1]])
    parts_v.append(step.v_ctx[ctx_off[s]:ctx_off[s + 1]])
    parts_k.append(step.k_new[q_off[s]:q_off[s + 1]])
    parts_v.append(step.v_new[q_off[s]:q_off[s + 1]])
    k = as_f64(np.concatenate(parts_k))
    v = as_f64(np.concatenate(parts_v))
    assert k.shape[0] == step.seq_lens[s]
    return k, v
