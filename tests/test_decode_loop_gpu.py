"""A decode loop run the way a serving engine runs it on the GPU: every step
plans itself on the device (pa_plan_step, with the previous step's seq_lens
as num_computed and one new token per sequence), then one
pa_attention_varlen_write_cache call stores the new K/V and attends.  No
lengths or tables travel to or from the host between steps.

Every step's cache bytes (bit-exact) and outputs (bf16 tolerance against the
fp64 values) equal the oracle's plan_step, cache write and attention on the
same draws.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_469_b200 import lib
from paged_kv_cache_469_b200.inputs import normal_values, planner_draws
from tests.oracle_side import as_f64

pytestmark = pytest.mark.gpu


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(
        torch.bfloat16)


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


class OracleLoop:
    """The oracle's side of the loop: its own tables, queue head and cache."""

    def __init__(self, seed, S, hkv, d, num_blocks, max_blocks):
        self.fq, self.nc, _ = planner_draws(seed, num_seqs=S, num_blocks=num_blocks, max_ctx=700)
        self.tables, self.head = oracle.allocate_block_tables(
            self.fq, self.nc, max_blocks_per_seq=max_blocks, pad_value=0)
        shape = (num_blocks, hkv, 16, d)
        self.kc = np.zeros(shape, np.uint16)
        self.vc = np.zeros(shape, np.uint16)
        n = int(self.nc.sum())
        ctx_slots = oracle.slot_mapping(self.tables, np.zeros(S, np.int32), self.nc)
        k = normal_values(seed, 4, n * hkv * d, "bf16").reshape(n, hkv, d)
        v = normal_values(seed, 5, n * hkv * d, "bf16").reshape(n, hkv, d)
        oracle.reshape_and_cache(k, v, self.kc, self.vc, ctx_slots)

    def step(self, q, k_new, v_new, hq, scale):
        ql = np.ones(len(self.nc), np.int32)
        self.tables, sl, qsl, slots, self.head = oracle.plan_step(
            self.fq, self.head, self.tables, self.nc, ql)
        oracle.reshape_and_cache(k_new, v_new, self.kc, self.vc, slots)
        self.nc = sl
        return oracle.paged_attention(q, self.kc, self.vc, self.tables, sl, qsl, num_q_heads=hq,
                                      scale=scale)


def step_values(seed, step, S, hq, hkv, d):
    q = normal_values(seed + 100 + step, 1, S * hq * d, "bf16").reshape(S, hq, d)
    k = normal_values(seed + 100 + step, 2, S * hkv * d, "bf16").reshape(S, hkv, d)
    v = normal_values(seed + 100 + step, 3, S * hkv * d, "bf16").reshape(S, hkv, d)
    return q, k, v


@pytest.mark.parametrize("hq,hkv,d", [(32, 4, 64), (32, 8, 128)])
def test_decode_loop_planned_on_gpu(hq, hkv, d):
    seed, S, steps, num_blocks, max_blocks = 77, 12, 5, 2000, 64
    ref = OracleLoop(seed, S, hkv, d, num_blocks, max_blocks)
    scale = 1.0 / math.sqrt(d)
    max_seq_len = int(ref.nc.max()) + steps

    # device state, starting from the same context
    fq = torch.from_numpy(ref.fq).cuda()
    state = lib.new_planner_state(ref.head)
    tables = torch.from_numpy(ref.tables).cuda()
    num_computed = torch.from_numpy(ref.nc).cuda()
    query_lens = torch.ones(S, dtype=torch.int32, device="cuda")
    seq_lens = torch.empty(S, dtype=torch.int32, device="cuda")
    qsl = torch.empty(S + 1, dtype=torch.int32, device="cuda")
    slots = torch.empty(S, dtype=torch.int64, device="cuda")
    k_cache, v_cache = _bf16(ref.kc), _bf16(ref.vc)
    ws = lib.new_workspace(S, hq, hkv, d, max_seq_len)
    out = torch.empty((S, hq, d), dtype=torch.bfloat16, device="cuda")

    for step in range(steps):
        q, k_new, v_new = step_values(seed, step, S, hq, hkv, d)
        lib.plan_step(fq, state, num_computed, query_lens, tables, seq_lens, qsl, slots)
        lib.attention_varlen_write_cache(out, _bf16(q), _bf16(k_new), _bf16(v_new), k_cache,
                                         v_cache, slots, tables, seq_lens, qsl, max_query_len=1,
                                         max_seq_len=max_seq_len, scale=scale, workspace=ws)
        num_computed.copy_(seq_lens)  # the next step continues from this one
        want = ref.step(q, k_new, v_new, hq, scale)
        torch.cuda.synchronize()
        assert state.cpu().tolist()[:3] == [ref.head, 0, 0], f"step {step}"
        assert lib.workspace_status(ws) == 0
        np.testing.assert_array_equal(_bits(k_cache), ref.kc, err_msg=f"step {step} K cache")
        np.testing.assert_array_equal(_bits(v_cache), ref.vc, err_msg=f"step {step} V cache")
        got = as_f64(_bits(out))
        err = np.abs(got - want)
        bad = err > 2e-2 + 1e-2 * np.abs(want)
        assert not bad.any(), f"step {step}: {bad.sum()} elements out of tolerance"


@pytest.mark.parametrize("hq,hkv,d", [(32, 4, 64), (32, 8, 128)])
def test_decode_loop_graph_replayed_over_growing_steps(hq, hkv, d):
    """The serving loop's CUDA graph: one step (pa_plan_step, then
    pa_attention_varlen_write_cache without host copies, then the new
    lengths copied into num_computed) is captured once, after a first eager
    step, for this batch size and a bound on the lengths, and replayed for
    every later step while the sequences grow by one token per step.  Only
    the step's new q/k/v rows are copied in between replays.  Every step's
    caches are bit-exact and its outputs within the bf16 bar against the
    oracle's plan_step, cache write and attention."""
    seed, S, steps, num_blocks, max_blocks = 91, 12, 6, 2000, 64
    ref = OracleLoop(seed, S, hkv, d, num_blocks, max_blocks)
    scale = 1.0 / math.sqrt(d)
    max_seq_len = int(ref.nc.max()) + steps

    fq = torch.from_numpy(ref.fq).cuda()
    state = lib.new_planner_state(ref.head)
    tables = torch.from_numpy(ref.tables).cuda()
    num_computed = torch.from_numpy(ref.nc).cuda()
    query_lens = torch.ones(S, dtype=torch.int32, device="cuda")
    seq_lens = torch.empty(S, dtype=torch.int32, device="cuda")
    qsl = torch.empty(S + 1, dtype=torch.int32, device="cuda")
    slots = torch.empty(S, dtype=torch.int64, device="cuda")
    k_cache, v_cache = _bf16(ref.kc), _bf16(ref.vc)
    ws = lib.new_workspace(S, hq, hkv, d, max_seq_len)
    out = torch.empty((S, hq, d), dtype=torch.bfloat16, device="cuda")
    q_in = torch.empty((S, hq, d), dtype=torch.bfloat16, device="cuda")
    k_in = torch.empty((S, hkv, d), dtype=torch.bfloat16, device="cuda")
    v_in = torch.empty((S, hkv, d), dtype=torch.bfloat16, device="cuda")

    def one_step():
        lib.plan_step(fq, state, num_computed, query_lens, tables, seq_lens, qsl, slots)
        lib.attention_varlen_write_cache(out, q_in, k_in, v_in, k_cache, v_cache, slots, tables,
                                         seq_lens, qsl, max_query_len=1,
                                         max_seq_len=max_seq_len, scale=scale, workspace=ws)
        num_computed.copy_(seq_lens)

    graph = None
    for step in range(steps):
        q, k_new, v_new = step_values(seed, step, S, hq, hkv, d)
        q_in.copy_(_bf16(q))
        k_in.copy_(_bf16(k_new))
        v_in.copy_(_bf16(v_new))
        if step == 0:
            one_step()  # the first step runs eagerly (it also sets up every launch)
        else:
            if graph is None:
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    one_step()
            graph.replay()
        want = ref.step(q, k_new, v_new, hq, scale)
        torch.cuda.synchronize()
        assert state.cpu().tolist()[:3] == [ref.head, 0, 0], f"step {step}"
        assert lib.workspace_status(ws) == 0
        np.testing.assert_array_equal(_bits(k_cache), ref.kc, err_msg=f"step {step} K cache")
        np.testing.assert_array_equal(_bits(v_cache), ref.vc, err_msg=f"step {step} V cache")
        got = as_f64(_bits(out))
        err = np.abs(got - want)
        bad = err > 2e-2 + 1e-2 * np.abs(want)
        assert not bad.any(), f"step {step}: {bad.sum()} elements out of tolerance"
