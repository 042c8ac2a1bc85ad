"""Pins of the CPU oracle against what the pages and the mathematics fix.

Page "LLM推論エンジンvLLMの内部構造を徹底解説" (techfeed.io), section
"PagedAttentionの仕組み": 16-token blocks, 17 tokens -> ceil(17/16) = 2 blocks,
allocate_slots takes the front of free_block_queue into req_to_blocks, and the
flattened super-sequence masks every sequence to its own tokens; section
"高度な機能群": chunked prefill, prefix caching.

Each check is a plain function so that ``test_oracle_mutants.py`` can run the
same checks against deliberately broken copies of the oracle and show that
every planted mistake is caught.
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_469_b200.inputs import make_step, planner_draws, random_step, workload
from tests.oracle_side import as_f64, contiguous_kv, oracle_outputs, oracle_state

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- block bookkeeping

def check_worked_example():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "worked_example_blocks.txt"))
            if l.strip() and not l.startswith("#")]
    for n, bs, want in rows:
        assert oracle.blocks_needed(int(n), int(bs)) == int(want)


def check_blocks_needed_brute_force():
    for bs in (1, 2, 3, 16, 32):
        for n in range(0, 200):
            assert oracle.blocks_needed(n, bs) == math.ceil(n / bs), (n, bs)


def check_allocation_pops_queue_front():
    rng = np.random.default_rng(7)
    queue = rng.permutation(500).astype(np.int32)
    lens = np.array([17, 1, 16, 33, 48, 0, 5], dtype=np.int32)
    tables, taken = oracle.allocate_block_tables(queue, lens, max_blocks_per_seq=8,
                                                 pad_value=-7)
    # brute force: walk the queue from the front, request by request
    head = 0
    for s, n in enumerate(lens):
        need = math.ceil(n / 16)
        assert list(tables[s, :need]) == list(queue[head:head + need])
        assert (tables[s, need:] == -7).all()
        head += need
    assert taken == head
    used = tables[tables >= 0]
    assert len(set(used.tolist())) == len(used)  # no block handed out twice


def check_shared_prefix_allocation():
    queue = np.arange(100, 300, dtype=np.int32)[::-1].copy()
    lens = np.array([64 + 1, 64 + 20, 64 + 16], dtype=np.int32)
    tables, taken = oracle.allocate_block_tables(queue, lens, max_blocks_per_seq=6,
                                                 shared_prefix_tokens=64)
    for s in range(3):
        assert list(tables[s, :4]) == list(queue[:4])  # the prefix blocks, popped first
    assert list(tables[0, 4:5]) == list(queue[4:5])
    assert list(tables[1, 4:6]) == list(queue[5:7])
    assert list(tables[2, 4:5]) == list(queue[7:8])
    assert taken == 8


def check_slot_mapping_brute_force():
    rng = np.random.default_rng(3)
    queue = rng.permutation(40).astype(np.int32)
    lens = np.array([17, 33, 5], dtype=np.int32)
    tables, _ = oracle.allocate_block_tables(queue, lens, max_blocks_per_seq=3)
    slots = oracle.slot_mapping(tables, np.zeros(3, np.int32), lens)
    assert len(set(slots.tolist())) == len(slots)  # every token its own slot
    assert (slots >= 0).all() and (slots < 40 * 16).all()
    i = 0
    for s, n in enumerate(lens):
        for p in range(n):
            blk, off = divmod(int(slots[i]), 16)
            assert off == p % 16  # offsets fill a block in token order
            assert blk == tables[s, p // 16]  # block = the request's (p//16)-th block
            i += 1
    # a later window of positions maps to the same slots as before
    part = oracle.slot_mapping(tables, np.array([16, 30, 0], np.int32),
                               np.array([1, 3, 0], np.int32))
    assert list(part) == [slots[16], slots[17 + 30], slots[17 + 31], slots[17 + 32]]


def check_query_start_loc():
    ql = np.array([17, 1, 1, 0, 4], dtype=np.int32)
    assert list(oracle.query_start_loc(ql)) == [0, 17, 18, 19, 19, 23]


def check_reshape_and_cache():
    rng = np.random.default_rng(11)
    nb, hkv, bs, d, t = 6, 2, 16, 8, 9
    k = rng.standard_normal((t, hkv, d)).astype(np.float32)
    v = rng.standard_normal((t, hkv, d)).astype(np.float32)
    kc = np.full((nb, hkv, bs, d), 1234.5, np.float32)
    vc = np.full((nb, hkv, bs, d), -99.0, np.float32)
    slots = np.array([0, 17, 95, -1, 40, 41, 16, -5, 3], dtype=np.int64)
    oracle.reshape_and_cache(k, v, kc, vc, slots)
    wk = np.full_like(kc, 1234.5)
    wv = np.full_like(vc, -99.0)
    for i, sl in enumerate(slots):
        if sl < 0:
            continue
        wk[sl // bs, :, sl % bs, :] = k[i]
        wv[sl // bs, :, sl % bs, :] = v[i]
    assert wk.tobytes() == kc.tobytes() and wv.tobytes() == vc.tobytes()


# ---------------------------------------------------------------- attention

def _sdpa_rows(step, s):
    """torch's fp64 scaled_dot_product_attention on sequence s's contiguous K/V,
    with the mask of the flattened super-sequence (query j at position
    L - q_len + j sees keys 0..that position) and GQA by repeating KV heads."""
    k, v = contiguous_kv(step, s)
    L = int(step.seq_lens[s])
    ql = int(step.query_lens[s])
    q0 = int(np.sum(step.query_lens[:s]))
    q = torch.from_numpy(as_f64(step.q[q0:q0 + ql]))
    g = step.num_q_heads // step.num_kv_heads
    kt = torch.from_numpy(k).repeat_interleave(g, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(g, dim=1)
    pos = torch.arange(L - ql, L).unsqueeze(1)
    mask = torch.arange(L).unsqueeze(0) <= pos
    out = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1), kt.transpose(0, 1), vt.transpose(0, 1), attn_mask=mask,
        scale=step.scale)
    return out.transpose(0, 1).numpy()


def check_dense_agreement(seeds=(1, 2, 3, 4)):
    steps = [random_step(sd, dtype="f32", num_q_heads=8, num_kv_heads=2, head_dim=16,
                         num_seqs=5, max_ctx=40, max_q=20) for sd in seeds]
    steps.append(random_step(9, dtype="bf16", num_q_heads=4, num_kv_heads=4, head_dim=32,
                             num_seqs=3, max_ctx=70, max_q=3))
    steps.append(random_step(10, dtype="bf16", num_q_heads=6, num_kv_heads=2, head_dim=8,
                             num_seqs=4, max_ctx=20, max_q=9, shared_prefix_tokens=32))
    for step in steps:
        out = oracle_outputs(step)
        q0 = 0
        for s in range(step.num_seqs):
            ql = int(step.query_lens[s])
            ref = _sdpa_rows(step, s)
            np.testing.assert_allclose(out[q0:q0 + ql], ref, rtol=1e-12, atol=1e-12)
            q0 += ql


def check_block_permutation_invariance():
    step = random_step(21, dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=16,
                       num_seqs=4, max_ctx=60, max_q=12)
    base = oracle_outputs(step)
    rng = np.random.default_rng(5)
    for _ in range(3):
        step.free_queue = rng.permutation(step.num_blocks).astype(np.int32)
        again = oracle_outputs(step)
        assert again.tobytes() == base.tobytes()


def check_sequence_reorder_invariance():
    step = random_step(31, dtype="f32", num_q_heads=4, num_kv_heads=1, head_dim=16,
                       num_seqs=4, max_ctx=50, max_q=10)
    base = oracle_outputs(step)
    perm = np.array([2, 0, 3, 1])
    q_off = np.concatenate([[0], np.cumsum(step.query_lens)])
    c_off = np.concatenate([[0], np.cumsum(step.ctx_count)])
    rows = lambda a, off, s: a[off[s]:off[s + 1]]
    re = make_step(name="re", dtype="f32", num_q_heads=4, num_kv_heads=1, head_dim=16,
                   num_blocks=step.num_blocks, seq_lens=step.seq_lens[perm],
                   query_lens=step.query_lens[perm], seed=99)
    re.q = np.concatenate([rows(step.q, q_off, s) for s in perm])
    re.k_new = np.concatenate([rows(step.k_new, q_off, s) for s in perm])
    re.v_new = np.concatenate([rows(step.v_new, q_off, s) for s in perm])
    re.k_ctx = np.concatenate([rows(step.k_ctx, c_off, s) for s in perm])
    re.v_ctx = np.concatenate([rows(step.v_ctx, c_off, s) for s in perm])
    out = oracle_outputs(re)
    r_off = np.concatenate([[0], np.cumsum(re.query_lens)])
    for i, s in enumerate(perm):
        assert out[r_off[i]:r_off[i + 1]].tobytes() == base[q_off[s]:q_off[s + 1]].tobytes()


def _single(dtype, L, ql, hq=2, hkv=1, d=8, seed=0):
    return make_step(name="one", dtype=dtype, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                     num_blocks=64, seq_lens=[L], query_lens=[ql], seed=seed)


def check_special_cases():
    # one visible key: the output is that key's value row, exactly
    st = _single("f32", 1, 1)
    out = oracle_outputs(st)
    np.testing.assert_array_equal(out[0, 0], st.v_new[0, 0].astype(np.float64))
    # constant V rows: the output is that row whatever the weights
    st = _single("f32", 37, 5, seed=1)
    st.v_ctx[:] = st.v_new[0]
    st.v_new[:] = st.v_new[0]
    out = oracle_outputs(st)
    np.testing.assert_allclose(out, np.broadcast_to(st.v_new[0, 0], out.shape), rtol=0,
                               atol=1e-14)
    # zero query: uniform weights -> mean of the visible V rows (closed form)
    st = _single("f32", 29, 4, seed=2)
    st.q[:] = 0
    out = oracle_outputs(st)
    vall = np.concatenate([st.v_ctx, st.v_new]).astype(np.float64)[:, 0]  # [L, D]
    for j in range(4):
        pos = 29 - 4 + j
        np.testing.assert_allclose(out[j, 0], vall[:pos + 1].mean(axis=0), rtol=1e-13,
                                   atol=1e-14)
    # two keys with scores a, b: weights are the logistic function of (a - b)
    st = _single("f32", 2, 1, hq=1, d=4, seed=3)
    out = oracle_outputs(st)
    k0, k1 = st.k_ctx[0, 0].astype(np.float64), st.k_new[0, 0].astype(np.float64)
    q = st.q[0, 0].astype(np.float64)
    a, b = q @ k0 * st.scale, q @ k1 * st.scale
    w0 = 1.0 / (1.0 + math.exp(b - a))
    want = w0 * st.v_ctx[0, 0].astype(np.float64) + (1 - w0) * st.v_new[0, 0].astype(np.float64)
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-13, atol=1e-15)


def check_gqa_equals_repeated_mha():
    st = random_step(41, dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=16, num_seqs=3,
                     max_ctx=30, max_q=6)
    out = oracle_outputs(st)
    mha = make_step(name="mha", dtype="bf16", num_q_heads=8, num_kv_heads=8, head_dim=16,
                    num_blocks=st.num_blocks, seq_lens=st.seq_lens, query_lens=st.query_lens,
                    seed=st.seed)
    mha.q = st.q
    for name in ("k_new", "v_new", "k_ctx", "v_ctx"):
        setattr(mha, name, np.repeat(getattr(st, name), 4, axis=1))
    assert oracle_outputs(mha).tobytes() == out.tobytes()


def check_chunked_prefill_equals_one_shot():
    """Prefill 40 tokens at once, or as chunks of 16 + 13 + 11 with the cache
    written between chunks: the rows agree bit for bit; a decode at position p
    equals the last row of a prefill of p + 1 tokens."""
    one = _single("bf16", 40, 40, hq=4, hkv=2, d=16, seed=5)
    full = oracle_outputs(one)
    kall = np.concatenate([one.k_ctx, one.k_new])
    vall = np.concatenate([one.v_ctx, one.v_new])
    start = 0
    for n in (16, 13, 11):
        ch = make_step(name="chunk", dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=16,
                       num_blocks=64, seq_lens=[start + n], query_lens=[n], seed=5)
        ch.free_queue = one.free_queue
        ch.q = one.q[start:start + n]
        ch.k_ctx, ch.v_ctx = kall[:start], vall[:start]
        ch.k_new, ch.v_new = kall[start:start + n], vall[start:start + n]
        assert oracle_outputs(ch).tobytes() == full[start:start + n].tobytes()
        start += n
    dec = make_step(name="dec", dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=16,
                    num_blocks=64, seq_lens=[40], query_lens=[1], seed=5)
    dec.free_queue = one.free_queue
    dec.q = one.q[39:40]
    dec.k_ctx, dec.v_ctx, dec.k_new, dec.v_new = kall[:39], vall[:39], kall[39:], vall[39:]
    assert oracle_outputs(dec).tobytes() == full[39:40].tobytes()


def check_shared_prefix_equals_private_copies():
    st = random_step(51, dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=16, num_seqs=4,
                     max_ctx=20, max_q=3, shared_prefix_tokens=48)
    shared = oracle_outputs(st)
    st_state = oracle_state(st)
    # every table starts with the same 3 physical blocks
    assert (st_state["block_tables"][:, :3] == st_state["block_tables"][0, :3]).all()
    priv = make_step(name="priv", dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=16,
                     num_blocks=st.num_blocks + 16, seq_lens=st.seq_lens,
                     query_lens=st.query_lens, seed=st.seed)
    c_off = np.concatenate([[0], np.cumsum(st.ctx_count)])
    parts_k, parts_v = [], []
    for s in range(st.num_seqs):
        if s > 0:
            parts_k.append(st.k_ctx[:48])
            parts_v.append(st.v_ctx[:48])
        parts_k.append(st.k_ctx[c_off[s]:c_off[s + 1]])
        parts_v.append(st.v_ctx[c_off[s]:c_off[s + 1]])
    priv.k_ctx, priv.v_ctx = np.concatenate(parts_k), np.concatenate(parts_v)
    priv.q, priv.k_new, priv.v_new = st.q, st.k_new, st.v_new
    assert oracle_outputs(priv).tobytes() == shared.tobytes()


def check_bf16_rounding_exhaustive():
    """Every finite bf16 value b: b itself, the midpoint to the next value (ties
    go to the even pattern) and the doubles just either side of it."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32)  # finite, non-negative patterns
    lo = (bits << 16).view(np.float32).astype(np.float64)
    hi = ((bits + 1) << 16).view(np.float32).astype(np.float64)
    hi[-1] = 2.0 ** 128  # the value after the largest finite bf16
    mid = (lo + hi) / 2  # exact in fp64: 9 significant bits
    tie = np.where(bits % 2 == 0, bits, bits + 1)
    for sign in (1.0, -1.0):
        sb = 0x8000 if sign < 0 else 0
        for x, want in ((lo, bits), (mid, tie), (np.nextafter(mid, -np.inf), bits),
                        (np.nextafter(mid, np.inf), bits + 1)):
            got = oracle.round_to_bf16(sign * x).astype(np.uint32)
            np.testing.assert_array_equal(got, (want | sb).astype(np.uint32))


def check_workload_block_counts():
    """The tiny workload: the prefill of 17 tokens holds 2 blocks, the decodes at
    33 and 48 tokens hold 3 each, 8 of the 64 pool blocks in all."""
    st = workload("tiny_f32")
    state = oracle_state(st)
    assert state["blocks_taken"] == 8
    assert list(state["block_tables"][0, :2]) == list(st.free_queue[:2])


# ---------------------------------------------------------------- step planning
#
# oracle.plan_step against allocate_slots walked by hand: a Python list for the
# queue, one block per started group of 16 tokens counted token by token, the
# slot of position p read from the row at p // 16, offset p % 16 -- no block
# arithmetic shared with the oracle.

PLAN_PAD = -3


def _hand_walk(free_queue, steps):
    """Per step: (rows, seq_lens, query_start_loc, slots, head)."""
    queue = [int(b) for b in free_queue]
    taken = 0
    rows: dict = {}
    for num_computed, query_lens in steps:
        seq_lens, qsl, slots = [], [0], []
        for s in range(len(query_lens)):
            row = rows.setdefault(s, [])
            length = int(num_computed[s]) + int(query_lens[s])
            started = sum(1 for t in range(length) if t % 16 == 0)
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
        assert (tables[s, len(r):] == PLAN_PAD).all(), f"row {s} written past its blocks"


def check_plan_step_fresh_is_whole_allocation():
    for S in (1, 6, 57):
        fq, _, ql = planner_draws(100 + S, num_seqs=S, num_blocks=5000, max_ctx=0,
                                  max_chunk=300, prefill_frac=0.6)
        nc = np.zeros(S, np.int32)
        tables, sl, qsl, slots, head = oracle.plan_step(
            fq, 0, np.full((S, 32), PLAN_PAD, np.int32), nc, ql)
        whole, taken = oracle.allocate_block_tables(fq, ql, max_blocks_per_seq=32,
                                                    pad_value=PLAN_PAD)
        np.testing.assert_array_equal(tables, whole)
        assert head == taken
        (rows, w_sl, w_qsl, w_slots, w_head), = _hand_walk(fq, [(nc, ql)])
        _rows_match(tables, rows)
        np.testing.assert_array_equal(slots, w_slots)
        np.testing.assert_array_equal(qsl, w_qsl)
        np.testing.assert_array_equal(sl, w_sl)


def check_plan_step_chained_steps():
    """A context allocation, then five steps of decodes, chunks and idle
    sequences, each starting where the previous one left the queue."""
    for seed in (1, 2, 3):
        S = 23
        fq, nc0, ql = planner_draws(seed, num_seqs=S, num_blocks=4000, max_ctx=300,
                                    max_chunk=70, prefill_frac=0.3, idle_frac=0.2)
        rng = np.random.default_rng(seed)
        steps = [(np.zeros(S, np.int32), nc0)]
        nc = nc0
        for _ in range(5):
            steps.append((nc, ql))
            nc = (nc + ql).astype(np.int32)
            ql = np.where(rng.random(S) < 0.3, rng.integers(0, 50, S), 1).astype(np.int32)
        tables = np.full((S, 64), PLAN_PAD, np.int32)
        head = 0
        for (num_computed, query_lens), walk in zip(steps, _hand_walk(fq, steps)):
            tables, sl, qsl, slots, head = oracle.plan_step(fq, head, tables, num_computed,
                                                            query_lens)
            rows, w_sl, w_qsl, w_slots, w_head = walk
            _rows_match(tables, rows)
            np.testing.assert_array_equal(sl, w_sl)
            np.testing.assert_array_equal(qsl, w_qsl)
            np.testing.assert_array_equal(slots, w_slots)
            assert head == w_head


def check_plan_step_invariants():
    """One step's slots are distinct, each lies in a block of its own
    sequence's row, and the blocks appended are the queue entries taken."""
    S = 40
    fq, nc, ql = planner_draws(9, num_seqs=S, num_blocks=6000, max_ctx=500, max_chunk=100,
                               prefill_frac=0.4)
    tables0, head0 = oracle.allocate_block_tables(fq, nc, max_blocks_per_seq=64,
                                                  pad_value=PLAN_PAD)
    tables, _, qsl, slots, head = oracle.plan_step(fq, head0, tables0, nc, ql)
    assert len(set(slots.tolist())) == len(slots)
    for s in range(S):
        own = set(tables[s][tables[s] != PLAN_PAD].tolist())
        assert {int(x) // 16 for x in slots[qsl[s]:qsl[s + 1]]} <= own
    appended = sorted(set(tables[tables != PLAN_PAD].tolist()) -
                      set(tables0[tables0 != PLAN_PAD].tolist()))
    assert appended == sorted(fq[head0:head].tolist())


def check_plan_step_refusals():
    """A step that does not fit is refused as a whole; the limits themselves fit."""
    fq = np.arange(10, dtype=np.int32)
    t = np.full((2, 4), PLAN_PAD, np.int32)
    nc = np.array([16, 0], np.int32)
    ok = oracle.plan_step(fq, 1, t, nc, np.array([48, 64], np.int32))  # rows exactly full
    assert ok[4] == 1 + 3 + 4
    for head, ql, cap in ((3, [48, 64], None),   # 7 blocks wanted, 7 left: fits ...
                          (4, [48, 64], None),   # ... 6 left: pool runs dry
                          (0, [49, 0], None),    # row 0 would need a 5th block
                          (0, [1, -1], None),    # negative count
                          (11, [1, 1], None),    # head past the queue
                          (0, [3, 4], 6)):       # 7 tokens, room for 6
        try:
            oracle.plan_step(fq, head, t, nc, np.array(ql, np.int32), max_tokens=cap)
            refused = False
        except ValueError:
            refused = True
        assert refused == (head != 3), (head, ql, cap)


CHECKS = [check_worked_example, check_blocks_needed_brute_force,
          check_allocation_pops_queue_front, check_shared_prefix_allocation,
          check_slot_mapping_brute_force, check_query_start_loc, check_reshape_and_cache,
          check_dense_agreement, check_block_permutation_invariance,
          check_sequence_reorder_invariance, check_special_cases, check_gqa_equals_repeated_mha,
          check_chunked_prefill_equals_one_shot, check_shared_prefix_equals_private_copies,
          check_bf16_rounding_exhaustive, check_workload_block_counts,
          check_plan_step_fresh_is_whole_allocation, check_plan_step_chained_steps,
          check_plan_step_invariants, check_plan_step_refusals]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_oracle_pin(check, oracle_lib):
    check()
