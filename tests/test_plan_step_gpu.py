"""The on-GPU step planner (pa_plan_step, through the C ABI) against the
oracle's allocation, prefix sums and slot mapping, bit-exact.

One planner call must equal the oracle's plan_step entry for entry: the
blocks each sequence appends (allocate_slots from the queue front at the
current head, sequences in order), seq_lens, query_start_loc, the slots of the
new positions, and the new queue head.  A call that cannot fit sets its status
bit and writes nothing else.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_469_b200 import lib
from paged_kv_cache_469_b200.inputs import planner_draws

pytestmark = pytest.mark.gpu

PAD = -7  # entries no call should touch


def expected_step(free_queue, head, tables, num_computed, query_lens):
    """(tables, seq_lens, query_start_loc, slots, new head) one call must give."""
    return oracle.plan_step(free_queue, head, tables, num_computed, query_lens)


class Planner:
    """Device buffers of one planner stream of steps."""

    def __init__(self, free_queue, tables, head, max_tokens):
        S = tables.shape[0]
        self.fq = torch.from_numpy(free_queue).cuda()
        self.state = lib.new_planner_state(head)
        self.tables = torch.from_numpy(tables).cuda()
        self.num_computed = torch.zeros(S, dtype=torch.int32, device="cuda")
        self.query_lens = torch.zeros(S, dtype=torch.int32, device="cuda")
        self.seq_lens = torch.full((S,), PAD, dtype=torch.int32, device="cuda")
        self.qsl = torch.full((S + 1,), PAD, dtype=torch.int32, device="cuda")
        self.slots = torch.full((max_tokens,), PAD, dtype=torch.int64, device="cuda")

    def run(self, num_computed=None, query_lens=None):
        if num_computed is not None:
            self.num_computed.copy_(torch.from_numpy(num_computed))
        if query_lens is not None:
            self.query_lens.copy_(torch.from_numpy(query_lens))
        lib.plan_step(self.fq, self.state, self.num_computed, self.query_lens, self.tables,
                      self.seq_lens, self.qsl, self.slots)

    def check(self, want, what=""):
        torch.cuda.synchronize()
        tables, seq_lens, qsl, slots, head = want
        st = self.state.cpu().numpy()
        assert st[1] == 0, f"{what}: status {st[1]}"
        assert st[0] == head and st[2] == 0, f"{what}: state {st}"
        np.testing.assert_array_equal(self.tables.cpu().numpy(), tables, err_msg=what)
        np.testing.assert_array_equal(self.seq_lens.cpu().numpy(), seq_lens, err_msg=what)
        np.testing.assert_array_equal(self.qsl.cpu().numpy(), qsl, err_msg=what)
        got = self.slots.cpu().numpy()
        np.testing.assert_array_equal(got[:len(slots)], slots, err_msg=what)
        assert (got[len(slots):] == PAD).all(), f"{what}: slots past the step written"


def _start(seed, S, num_blocks, mb, max_tokens, **kw):
    fq, nc, ql = planner_draws(seed, num_seqs=S, num_blocks=num_blocks, **kw)
    # the blocks of the tokens already computed, from the oracle's allocation
    tables, taken = oracle.allocate_block_tables(fq, nc, max_blocks_per_seq=mb, pad_value=PAD)
    return fq, nc, ql, tables, taken, Planner(fq, tables, taken, max_tokens)


@pytest.mark.parametrize("S", [1, 5, 300, 1024, 1025, 3000])
def test_fresh_allocation_equals_oracle(S):
    """Nothing computed yet: the tables are the oracle's allocate_slots of the
    whole lengths, and the slots cover every token."""
    fq, _, ql, _, _, _ = _start(11 + S, S, 40000, 64, 1, max_ctx=0, max_chunk=600,
                                prefill_frac=0.5)
    tables0 = np.full((S, 64), PAD, np.int32)
    p = Planner(fq, tables0, 0, int(ql.sum()) + 5)
    nc = np.zeros(S, np.int32)
    p.run(nc, ql)
    want = expected_step(fq, 0, tables0, nc, ql)
    direct, taken = oracle.allocate_block_tables(fq, ql, max_blocks_per_seq=64, pad_value=PAD)
    np.testing.assert_array_equal(want[0], direct)  # the composition is the plain allocation
    assert want[4] == taken
    p.check(want, f"fresh S={S}")


@pytest.mark.parametrize("seed,S", [(1, 7), (2, 64), (3, 700), (4, 2500)])
def test_incremental_steps(seed, S):
    """Six steps in a row; each step's num_computed is the previous seq_lens."""
    fq, nc, ql, tables, taken, p = _start(seed, S, 200000, 400, 160000,
                                          max_ctx=4096 if S <= 1000 else 2000)
    rng = np.random.default_rng(seed)
    want = (tables, None, None, None, taken)
    for step in range(6):
        want = expected_step(fq, want[4], want[0], nc, ql)
        p.run(nc, ql)
        p.check(want, f"step {step}")
        p.slots.fill_(PAD)
        nc = want[1]
        ql = np.where(rng.random(S) < 0.1, rng.integers(0, 300, S), 1).astype(np.int32)


def test_block_boundaries_and_idle_sequences():
    """Lengths at, just below and just past block boundaries; idle sequences
    (nothing scheduled) take no block and no slot."""
    nc = np.array([0, 15, 16, 17, 31, 32, 0, 48, 5, 16], np.int32)
    ql = np.array([16, 1, 1, 15, 2, 0, 0, 33, 11, 16], np.int32)
    fq = np.random.default_rng(3).permutation(500).astype(np.int32)
    tables, taken = oracle.allocate_block_tables(fq, nc, max_blocks_per_seq=8, pad_value=PAD)
    p = Planner(fq, tables, taken, 200)
    p.run(nc, ql)
    p.check(expected_step(fq, taken, tables, nc, ql), "boundaries")


def test_no_sequences():
    fq = np.arange(8, dtype=np.int32)
    p = Planner(fq, np.zeros((0, 4), np.int32), 3, 4)
    p.run(np.zeros(0, np.int32), np.zeros(0, np.int32))
    torch.cuda.synchronize()
    assert p.qsl.cpu().tolist() == [0]
    assert p.state.cpu().tolist() == [3, 0, 0, 0]


def test_largest_steps():
    """The most sequences one call plans (16384 decodes), and one long prefill
    (131072 tokens: the writes spread over many CTAs)."""
    S = 16384
    fq, nc, ql, tables, taken, p = _start(21, S, 600000, 64, S, max_ctx=900, prefill_frac=0.0,
                                          idle_frac=0.0)
    p.run(nc, ql)
    p.check(expected_step(fq, taken, tables, nc, ql), "16384 decodes")

    nc = np.array([100, 0, 7], np.int32)
    ql = np.array([131072, 1, 1], np.int32)
    fq = np.random.default_rng(5).permutation(20000).astype(np.int32)
    tables, taken = oracle.allocate_block_tables(fq, nc, max_blocks_per_seq=8300, pad_value=PAD)
    p = Planner(fq, tables, taken, 131074)
    p.run(nc, ql)
    p.check(expected_step(fq, taken, tables, nc, ql), "131072-token prefill")


def test_graph_replay_decode_loop():
    """A decode loop captured once (planner, then seq_lens becomes the next
    num_computed) and replayed: the head and the tables move on every replay."""
    S = 200
    fq, nc, _, tables, taken, p = _start(31, S, 60000, 300, S, max_ctx=2000)
    ql = np.ones(S, np.int32)
    p.run(nc, ql)  # warm: the first step runs eagerly
    want = expected_step(fq, taken, tables, nc, ql)
    p.check(want, "eager step")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        p.num_computed.copy_(p.seq_lens)
        with torch.cuda.graph(g, stream=side):
            lib.plan_step(p.fq, p.state, p.num_computed, p.query_lens, p.tables, p.seq_lens,
                          p.qsl, p.slots, stream=side)
            p.num_computed.copy_(p.seq_lens)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    # capture ran nothing: the state is still the eager step's
    p.check(want, "after capture")
    for r in range(5):
        g.replay()
        want = expected_step(fq, want[4], want[0], want[1], ql)
        p.check(want, f"replay {r}")


def _snapshot(p):
    torch.cuda.synchronize()
    return [t.cpu().clone() for t in (p.tables, p.seq_lens, p.qsl, p.slots)]


@pytest.mark.parametrize("case,bit", [("pool", lib.PLAN_POOL_EMPTY), ("row", lib.PLAN_ROW_FULL),
                                      ("slots", lib.PLAN_SLOTS_FULL),
                                      ("negative", lib.PLAN_BAD_LENGTH),
                                      ("head", lib.PLAN_BAD_HEAD)])
def test_refused_steps_write_nothing(case, bit):
    """A step that does not fit sets its bit, writes nothing and keeps the head;
    the next step that fits runs normally and the bit stays set."""
    S = 40
    # rows of 200 blocks, room for 20000 slots, a queue of 10000 blocks: each
    # case below breaks exactly one of the limits
    fq, nc, ql, tables, taken, p = _start(41, S, 10000, 200, 20000, max_ctx=1000)
    bad_nc, bad_ql = nc.copy(), ql.copy()
    if case == "pool":
        p.state[0] = len(fq) - 3  # three free blocks left
        bad_ql[:] = 40
    elif case == "row":
        bad_ql[3] = 200 * 16 - int(nc[3]) + 1  # one token past the row
    elif case == "slots":
        bad_ql[:] = 501  # 20040 tokens
    elif case == "negative":
        bad_ql[5] = -1
    else:
        p.state[0] = len(fq) + 1
    before = _snapshot(p)
    head_before = int(p.state[0].item())
    p.run(bad_nc, bad_ql)
    after = _snapshot(p)
    for a, b in zip(before, after):
        assert torch.equal(a, b), f"{case}: a refused step wrote output"
    st = p.state.cpu().tolist()
    assert st[1] == bit and st[0] == head_before and st[2] == 0, (case, st)
    if case in ("head", "pool"):
        p.state[0] = taken
    p.run(nc, ql)
    want = expected_step(fq, taken, tables, nc, ql)
    torch.cuda.synchronize()
    assert p.state[1].item() == bit  # sticky
    p.state[1] = 0
    p.check(want, f"{case}: the next step")
