"""Host-side block bookkeeping: free_block_queue, allocate_slots, req_to_blocks.

Follows the page "LLM推論エンジンvLLMの内部構造を徹底解説" (techfeed.io),
section "PagedAttentionの仕組み": KV lives in fixed 16-token blocks; a request
of n tokens holds ceil(n / 16) blocks (17 tokens -> 2); ``allocate_slots``
(1) counts the blocks still needed, (3) takes that many from the front of
``free_block_queue`` and appends them to the request's list in
``req_to_blocks``.  Step (2), preempting low-priority requests when the pool
is empty, is scheduler policy and is not modelled: an empty pool raises
:class:`PoolExhausted`.  Prefix caching (section "高度な機能群") is modelled by
starting a request's list with another request's blocks.

From the block lists this module builds the per-step device inputs of the
attention kernels: the padded ``block_tables`` matrix, the ``slot_mapping`` of
the tokens whose K/V a step writes, and the super-sequence offsets
``query_start_loc`` (an exclusive prefix sum of the query lengths).
"""
from __future__ import annotations

from collections import deque
from dataclasses import dataclass

import numpy as np


class PoolExhausted(RuntimeError):
    """The free queue holds fewer blocks than a request needs."""


class BlockPool:
    def __init__(self, free_block_queue, block_size: int = 16):
        if block_size <= 0:
            raise ValueError("block_size must be positive")
        self.block_size = int(block_size)
        self.free_block_queue = deque(int(b) for b in free_block_queue)
        self.req_to_blocks: dict = {}

    def blocks_needed(self, num_tokens: int) -> int:
        """ceil(num_tokens / block_size)."""
        return -(-int(num_tokens) // self.block_size) if num_tokens > 0 else 0

    def allocate_slots(self, req_id, num_tokens: int) -> list:
        """Make req_id hold enough blocks for num_tokens tokens; return the new blocks."""
        have = self.req_to_blocks.setdefault(req_id, [])
        n = self.blocks_needed(num_tokens) - len(have)
        if n <= 0:
            return []
        if n > len(self.free_block_queue):
            raise PoolExhausted(f"request {req_id!r} needs {n} blocks, "
                                f"{len(self.free_block_queue)} free")
        new = [self.free_block_queue.popleft() for _ in range(n)]
        have.extend(new)
        return new

    def share_prefix(self, req_id, prefix_req_id) -> None:
        """Start req_id's block list with every block of prefix_req_id (prefix caching)."""
        if self.req_to_blocks.get(req_id):
            raise ValueError(f"request {req_id!r} already holds blocks")
        self.req_to_blocks[req_id] = list(self.req_to_blocks[prefix_req_id])

    def block_table(self, req_ids, max_blocks_per_seq: int | None = None,
                    pad_value: int = 0) -> np.ndarray:
        """int32 [len(req_ids), max_blocks_per_seq], row s = req_to_blocks of req_ids[s]."""
        rows = [self.req_to_blocks[r] for r in req_ids]
        width = max((len(r) for r in rows), default=0)
        if max_blocks_per_seq is None:
            max_blocks_per_seq = max(1, width)
        if width > max_blocks_per_seq:
            raise ValueError("a block list is longer than max_blocks_per_seq")
        table = np.full((len(rows), max_blocks_per_seq), pad_value, dtype=np.int32)
        for s, r in enumerate(rows):
            table[s, :len(r)] = r
        return table


def slot_mapping(block_tables: np.ndarray, first_pos, count, block_size: int = 16) -> np.ndarray:
    """int64 cache slot of positions first_pos[s] .. +count[s]-1 of each sequence s.

    Position p of sequence s sits in logical block p // block_size at offset
    p % block_size, i.e. slot block_tables[s, p // block_size] * block_size +
    p % block_size; the output concatenates the sequences in order."""
    first_pos = np.asarray(first_pos, dtype=np.int64)
    count = np.asarray(count, dtype=np.int64)
    total = int(count.sum())
    seq = np.repeat(np.arange(len(count)), count)
    starts = np.concatenate([[0], np.cumsum(count)[:-1]]).astype(np.int64)
    pos = first_pos[seq] + (np.arange(total, dtype=np.int64) - starts[seq])
    blk = pos // block_size
    if total and int(blk.max()) >= block_tables.shape[1]:
        raise ValueError("position beyond the block table")
    return block_tables[seq, blk].astype(np.int64) * block_size + pos % block_size


def query_start_loc(query_lens) -> np.ndarray:
    """int32 [S+1]: start of each sequence's query rows in the flattened super-sequence."""
    q = np.asarray(query_lens, dtype=np.int64)
    out = np.zeros(len(q) + 1, dtype=np.int64)
    np.cumsum(q, out=out[1:])
    return out.astype(np.int32)


@dataclass
class StepPlan:
    """Host arrays that describe one step to the kernels."""

    block_tables: np.ndarray  # int32 [S, max_blocks_per_seq]
    seq_lens: np.ndarray  # int32 [S]
    query_start_loc: np.ndarray  # int32 [S+1]
    slot_mapping: np.ndarray  # int64 [T]: cache slots of this step's new tokens
    ctx_slot_mapping: np.ndarray  # int64 [sum ctx]: slots of earlier tokens (cache pre-fill)
    max_query_len: int
    max_seq_len: int
    blocks_taken: int


def plan_step(*, free_queue, seq_lens, query_lens, ctx_first_pos, ctx_count,
              block_size: int = 16, shared_prefix_tokens: int = 0,
              max_blocks_per_seq: int | None = None) -> StepPlan:
    """Allocate every sequence's blocks (in order) and build the step's device inputs."""
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    query_lens = np.asarray(query_lens, dtype=np.int32)
    pool = BlockPool(free_queue, block_size)
    n_free = len(pool.free_block_queue)
    if shared_prefix_tokens:
        if shared_prefix_tokens % block_size:
            raise ValueError("only whole blocks can be shared")
        pool.allocate_slots("prefix", shared_prefix_tokens)
    for s, n in enumerate(seq_lens):
        if shared_prefix_tokens:
            pool.share_prefix(s, "prefix")
        pool.allocate_slots(s, int(n))
    tables = pool.block_table(range(len(seq_lens)), max_blocks_per_seq)
    new_first = (seq_lens - query_lens).astype(np.int64)
    return StepPlan(
        block_tables=tables, seq_lens=seq_lens, query_start_loc=query_start_loc(query_lens),
        slot_mapping=slot_mapping(tables, new_first, query_lens, block_size),
        ctx_slot_mapping=slot_mapping(tables, ctx_first_pos, ctx_count, block_size),
        max_query_len=int(query_lens.max(initial=0)), max_seq_len=int(seq_lens.max(initial=0)),
        blocks_taken=n_free - len(pool.free_block_queue))
