"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Bars: the cache write is bit-exact over the whole pool; fp32 outputs within
1e-4 absolute; bf16 outputs within 2e-2 + 1e-2 * |ref| elementwise, ref being
the oracle's fp64 value before any rounding.
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_469_b200.inputs import make_step, random_step, workload
from tests.oracle_side import oracle_outputs, oracle_state

pytestmark = pytest.mark.gpu

NTHREADS = max(1, os.cpu_count() or 1)


def _bits(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if dtype == "f32":
        assert err.max(initial=0.0) <= 1e-4, f"{what}: max abs err {err.max()}"
    else:
        bound = 2e-2 + 1e-2 * np.abs(ref)
        bad = err > bound
        assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements out of tolerance, "
                               f"worst {err.max()}")


def assert_cache_equal(dev_cache: torch.Tensor, want: np.ndarray, what: str,
                       chunk_blocks: int = 16384):
    """The whole device pool equals the oracle's, byte for byte (compared in
    chunks of blocks, so that a multi-GB pool never needs a second host copy)."""
    n = want.shape[0]
    for b in range(0, n, chunk_blocks):
        e = min(n, b + chunk_blocks)
        assert _bits(dev_cache[b:e]).tobytes() == want[b:e].tobytes(), \
            f"{what}: blocks {b}..{e - 1} differ from the oracle"


def assert_header_clear(workspace: torch.Tensor):
    """After a call the workspace header holds no error bit, and the decode
    grid's claim counters (words 1 and 2) are back at zero for the next call."""
    head = workspace[:12].view(torch.int32).cpu().tolist()
    assert head == [0, 0, 0], f"workspace header {head}"


def run_and_check(step, *, full=True, rows=None, check_cache=True, host_hints=True,
                  cache_fill=0.0):
    from paged_kv_cache_469_b200 import lib
    from paged_kv_cache_469_b200.step import DeviceStep
    ds = DeviceStep(step, cache_fill=cache_fill)
    ds.run(host_hints=host_hints)
    torch.cuda.synchronize()
    if step.dtype == "bf16":
        assert lib.workspace_status(ds.workspace) == 0, "a kernel gave up waiting"
    st = oracle_state(step)
    if check_cache and cache_fill == 0.0:
        assert_cache_equal(ds.k_cache, st["k_cache"], "k_cache")
        assert_cache_equal(ds.v_cache, st["v_cache"], "v_cache")
    got = ds.out_f64()
    if full:
        ref = oracle_outputs(step, st, num_threads=NTHREADS)
        assert_close(got, ref, step.dtype, step.name)
    if rows is not None:
        tok, head = rows
        ref = oracle.paged_attention_rows(step.q, st["k_cache"], st["v_cache"],
                                          st["block_tables"], step.seq_lens,
                                          st["query_start_loc"], tok, head,
                                          num_q_heads=step.num_q_heads, scale=step.scale,
                                          num_threads=NTHREADS)
        assert_close(got[tok, head], ref, step.dtype, step.name + " (sampled rows)")
    assert_header_clear(ds.workspace)
    return ds, st


def test_tiny_fp32_workload():
    run_and_check(workload("tiny_f32"))


def test_tiny_fp32_without_host_hints():
    run_and_check(workload("tiny_f32"), host_hints=False)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("heads", [(8, 1), (8, 2), (4, 4), (32, 4), (16, 1)])
@pytest.mark.parametrize("seed", [0, 1])
def test_random_mixed_steps_bf16(d, heads, seed):
    hq, hkv = heads
    step = random_step(100 + seed, dtype="bf16", num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                       num_seqs=6, max_ctx=300, max_q=40)
    run_and_check(step)


@pytest.mark.parametrize("d", [64, 128])
def test_random_mixed_steps_fp32(d):
    step = random_step(7, dtype="f32", num_q_heads=8, num_kv_heads=2, head_dim=d, num_seqs=5,
                       max_ctx=200, max_q=30)
    run_and_check(step)


@pytest.mark.parametrize("hq,hkv,ql", [(32, 4, 2), (32, 8, 4), (16, 4, 3), (8, 8, 16),
                                       (16, 16, 1), (16, 1, 1)])
def test_multi_token_decode_rows(hq, hkv, ql):
    """Decode-class sequences whose q_len * group fills 9..16 MMA rows (speculative
    verification shapes), mixed with plain decodes."""
    lens = [1000, 37, 300, 16, 17]
    qls = [ql, 1, ql, 1, ql]
    step = make_step(name="mtd", dtype="bf16", num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
                     num_blocks=200, seq_lens=lens, query_lens=qls, seed=5)
    run_and_check(step)


def test_long_split_k_and_edge_lengths():
    """Many partitions (L up to 5000), one-key sequences, ragged last blocks,
    empty sequences (q_len 0) between non-empty ones."""
    lens = [5000, 1, 2, 15, 16, 17, 0, 4097, 33, 3]
    qls = [1, 1, 2, 1, 16, 17, 0, 1, 0, 3]
    step = make_step(name="edges", dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=64,
                     num_blocks=800, seq_lens=lens, query_lens=qls, seed=8)
    run_and_check(step)
    run_and_check(step, host_hints=False)


@pytest.mark.parametrize("d", [64, 128])
def test_uninitialised_pool_slots_are_never_used(d):
    """Every slot the step does not write holds NaN: partial last blocks,
    decodes and prefill chunks must still match the oracle."""
    step = random_step(300 + d, dtype="bf16", num_q_heads=16, num_kv_heads=4, head_dim=d,
                       num_seqs=8, max_ctx=500, max_q=150)
    run_and_check(step, cache_fill=float("nan"))


def test_pool_edge_blocks():
    """The first and last block of the pool are handed out."""
    step = make_step(name="pooledge", dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=128,
                     num_blocks=10, seq_lens=[40, 100], query_lens=[1, 30], seed=3)
    step.free_queue = np.array([9, 0, 5, 1, 8, 2, 7, 3, 6, 4], dtype=np.int32)
    run_and_check(step)


def test_decode_tinyllama_full():
    run_and_check(workload("decode_tinyllama"))


@pytest.mark.parametrize("name", ["mixed_llama3_8b", "prefix_decode_llama3_8b",
                                  "long_decode_llama3_8b"])
def test_full_size_workloads_every_row(name):
    """The three Llama-3-8B workloads at their full sizes, in the launch
    configuration the benchmark times (host copies of the lengths given), and
    again with the plan estimated on the device (no host copies): every output
    row of every sequence and q-head against the oracle, and the whole pool
    byte for byte.  Full-size prefill chunks run items of up to 23 key tiles
    and a host work list of 256 items; the long contexts split into many
    partitions per sequence."""
    from paged_kv_cache_469_b200 import lib
    from paged_kv_cache_469_b200.step import DeviceStep
    step = workload(name)
    ds = DeviceStep(step)
    st = oracle_state(step)
    ref = oracle_outputs(step, st, num_threads=NTHREADS)
    for hints in (True, False):
        ds.out.fill_(float("nan"))
        ds.run(host_hints=hints)
        torch.cuda.synchronize()
        assert lib.workspace_status(ds.workspace) == 0, "a kernel gave up waiting"
        assert_cache_equal(ds.k_cache, st["k_cache"], f"{name} k_cache")
        assert_cache_equal(ds.v_cache, st["v_cache"], f"{name} v_cache")
        assert_close(ds.out_f64(), ref, "bf16", f"{name} (host copies: {hints})")
        assert_header_clear(ds.workspace)
    del st, ref


# ---------------------------------------------------------------- invariances on the GPU

def _gpu_out(step, host_hints=True):
    from paged_kv_cache_469_b200.step import DeviceStep
    ds = DeviceStep(step)
    ds.run(host_hints=host_hints)
    torch.cuda.synchronize()
    return _bits(ds.out)


def test_block_permutation_bit_identical():
    step = random_step(61, dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                       num_seqs=6, max_ctx=600, max_q=40)
    base = _gpu_out(step)
    step.free_queue = np.random.default_rng(9).permutation(step.num_blocks).astype(np.int32)
    assert _gpu_out(step).tobytes() == base.tobytes()


def test_shared_prefix_equals_private_copies_gpu():
    st = random_step(71, dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                     num_seqs=5, max_ctx=200, max_q=1, shared_prefix_tokens=256)
    shared = _gpu_out(st)
    priv = make_step(name="priv", dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                     num_blocks=st.num_blocks + 5 * 16, seq_lens=st.seq_lens,
                     query_lens=st.query_lens, seed=st.seed)
    c_off = np.concatenate([[0], np.cumsum(st.ctx_count)])
    ks, vs = [], []
    for s in range(st.num_seqs):
        if s > 0:
            ks.append(st.k_ctx[:256])
            vs.append(st.v_ctx[:256])
        ks.append(st.k_ctx[c_off[s]:c_off[s + 1]])
        vs.append(st.v_ctx[c_off[s]:c_off[s + 1]])
    priv.k_ctx, priv.v_ctx = np.concatenate(ks), np.concatenate(vs)
    priv.q, priv.k_new, priv.v_new = st.q, st.k_new, st.v_new
    assert _gpu_out(priv).tobytes() == shared.tobytes()


def test_sequence_order_does_not_change_rows():
    step = random_step(81, dtype="bf16", num_q_heads=16, num_kv_heads=4, head_dim=64,
                       num_seqs=5, max_ctx=400, max_q=24)
    base = _gpu_out(step)
    perm = np.array([3, 1, 4, 0, 2])
    q_off = np.concatenate([[0], np.cumsum(step.query_lens)])
    c_off = np.concatenate([[0], np.cumsum(step.ctx_count)])
    re = make_step(name="re", dtype="bf16", num_q_heads=16, num_kv_heads=4, head_dim=64,
                   num_blocks=step.num_blocks, seq_lens=step.seq_lens[perm],
                   query_lens=step.query_lens[perm], seed=1)
    take = lambda a, off: np.concatenate([a[off[s]:off[s + 1]] for s in perm])
    re.q, re.k_new, re.v_new = take(step.q, q_off), take(step.k_new, q_off), take(step.v_new, q_off)
    re.k_ctx, re.v_ctx = take(step.k_ctx, c_off), take(step.v_ctx, c_off)
    out = _gpu_out(re)
    r_off = np.concatenate([[0], np.cumsum(re.query_lens)])
    for i, s in enumerate(perm):
        assert out[r_off[i]:r_off[i + 1]].tobytes() == base[q_off[s]:q_off[s + 1]].tobytes()


def test_chunked_prefill_matches_one_shot_gpu():
    """Prefill 700 tokens at once vs 3 chunks with cache writes in between."""
    from paged_kv_cache_469_b200.inputs import bf16_bits_to_f32
    one = make_step(name="one", dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                    num_blocks=64, seq_lens=[700], query_lens=[700], seed=12)
    full = _gpu_out(one)
    kall, vall = one.k_new, one.v_new
    start = 0
    for n in (256, 300, 144):
        ch = make_step(name="chunk", dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                       num_blocks=64, seq_lens=[start + n], query_lens=[n], seed=12)
        ch.free_queue = one.free_queue
        ch.q = one.q[start:start + n]
        ch.k_ctx, ch.v_ctx = kall[:start], vall[:start]
        ch.k_new, ch.v_new = kall[start:start + n], vall[start:start + n]
        got = bf16_bits_to_f32(_gpu_out(ch)).astype(np.float64)
        ref = bf16_bits_to_f32(full[start:start + n]).astype(np.float64)
        np.testing.assert_allclose(got, ref, atol=2e-2, rtol=1e-2)
        start += n


def test_zero_token_call_is_a_no_op():
    from paged_kv_cache_469_b200 import lib
    dev = "cuda"
    kc = torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16, device=dev)
    out = torch.empty(0, 8, 64, dtype=torch.bfloat16, device=dev)
    lib.attention_varlen(out, out, kc, kc, torch.zeros(1, 1, dtype=torch.int32, device=dev),
                         torch.zeros(1, dtype=torch.int32, device=dev),
                         torch.zeros(2, dtype=torch.int32, device=dev), max_query_len=0,
                         max_seq_len=0, scale=0.125, workspace=None)
    lib.reshape_and_cache(out[:, :2], out[:, :2], kc, kc,
                          torch.zeros(0, dtype=torch.int64, device=dev))
    torch.cuda.synchronize()


@pytest.mark.parametrize("d", [64, 128])
def test_graph_replay_matches_direct_calls(d):
    """A CUDA graph of the step (cache write + attention, the launches chained
    as programmatic dependents) replays to the same bytes as direct calls, and
    both match the oracle; so does a graph of the attention call alone."""
    from paged_kv_cache_469_b200 import lib
    from paged_kv_cache_469_b200.step import DeviceStep
    step = random_step(71 + d, dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=d,
                       num_seqs=8, max_ctx=900, max_q=300)
    ds = DeviceStep(step)
    ds.run()
    torch.cuda.synchronize()
    direct = _bits(ds.out).copy()
    g_step = ds.capture("step")
    g_attn = ds.capture("attention")
    for g in (g_step, g_attn, g_step):
        ds.out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert _bits(ds.out).tobytes() == direct.tobytes()
    assert lib.workspace_status(ds.workspace) == 0
    st = oracle_state(step)
    assert _bits(ds.k_cache).tobytes() == st["k_cache"].tobytes()
    assert_close(ds.out_f64(), oracle_outputs(step, st, num_threads=NTHREADS), "bf16",
                 "graph replay")


def _fused_check(step, host_hints=True, d_dtype="bf16"):
    from paged_kv_cache_469_b200 import lib
    from paged_kv_cache_469_b200.step import DeviceStep
    ds = DeviceStep(step)
    ds.run_fused(host_hints=host_hints)
    torch.cuda.synchronize()
    if step.dtype == "bf16":
        assert lib.workspace_status(ds.workspace) == 0
    st = oracle_state(step)
    assert _bits(ds.k_cache).tobytes() == st["k_cache"].tobytes(), "k_cache differs"
    assert _bits(ds.v_cache).tobytes() == st["v_cache"].tobytes(), "v_cache differs"
    assert_close(ds.out_f64(), oracle_outputs(step, st, num_threads=NTHREADS), step.dtype,
                 step.name + " (one call)")
    assert_header_clear(ds.workspace)
    return ds


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv,ql", [(32, 4, 1), (32, 8, 2), (8, 8, 16), (16, 1, 1)])
@pytest.mark.parametrize("hints", [True, False])
def test_write_cache_call_decode_steps(d, hq, hkv, ql, hints):
    """Decode-class steps: the decode kernel writes the new rows itself (new
    tokens crossing block and partition boundaries included); cache bytes and
    outputs equal the two-call path's and the oracle's."""
    rng = np.random.default_rng(1000 + d + hq + ql)
    lens = rng.integers(ql, 3000, size=12)
    lens[0], lens[1] = 17, ql  # a token at a block's start; a sequence of only new tokens
    step = make_step(name="fused_decode", dtype="bf16", num_q_heads=hq, num_kv_heads=hkv,
                     head_dim=d, num_blocks=int(np.sum((lens + 15) // 16)) + 40,
                     seq_lens=lens, query_lens=np.full(12, ql), seed=77)
    ds = _fused_check(step, host_hints=hints)
    if hints:  # the same partitioning as the two-call path: the same bytes
        two = DeviceStepTwoCall(step)
        assert _bits(two.out).tobytes() == _bits(ds.out).tobytes()


def DeviceStepTwoCall(step):
    from paged_kv_cache_469_b200.step import DeviceStep
    ds = DeviceStep(step)
    ds.run()
    torch.cuda.synchronize()
    return ds


@pytest.mark.parametrize("d", [64, 128])
def test_write_cache_call_mixed_and_fp32_steps(d):
    """Steps with prefill chunks (and fp32 steps) take the write-then-attend
    order inside the one call."""
    _fused_check(random_step(91 + d, dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=d,
                             num_seqs=5, max_ctx=400, max_q=200))
    _fused_check(random_step(93 + d, dtype="f32", num_q_heads=4, num_kv_heads=4, head_dim=d,
                             num_seqs=3, max_ctx=60, max_q=20))


def test_write_cache_call_graph_replay():
    from paged_kv_cache_469_b200.step import DeviceStep
    step = workload("decode_tinyllama")
    ds = DeviceStep(step)
    g = ds.capture("fused")
    ds.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    got = _bits(ds.out).copy()
    ref = DeviceStepTwoCall(step)
    assert got.tobytes() == _bits(ref.out).tobytes()


@pytest.mark.parametrize("case", ["one_long_unit", "many_tiny_units", "mixed_with_prefill"])
@pytest.mark.parametrize("hints", [True, False])
def test_decode_partition_edge_steps(case, hints):
    """Split-K decode on edge-shaped steps, with the partition length taken
    from the host copies or estimated without them: one long unit split into
    several partitions, hundreds of one- and two-block units, and decode units
    mixed with a prefill chunk."""
    if case == "one_long_unit":
        step = make_step(name=case, dtype="bf16", num_q_heads=8, num_kv_heads=1, head_dim=128,
                         num_blocks=260, seq_lens=[3000], query_lens=[1], seed=5)
    elif case == "many_tiny_units":
        lens = np.random.default_rng(3).integers(1, 40, size=300)
        step = make_step(name=case, dtype="bf16", num_q_heads=32, num_kv_heads=4, head_dim=64,
                         num_blocks=int(np.sum((lens + 15) // 16)) + 10, seq_lens=lens,
                         query_lens=np.ones(300, np.int32), seed=6)
    else:
        step = random_step(97, dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                           num_seqs=10, max_ctx=1500, max_q=3)
        step = make_step(name=case, dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                         num_blocks=step.num_blocks + 64,
                         seq_lens=np.concatenate([step.seq_lens, [700]]),
                         query_lens=np.concatenate([step.query_lens, [300]]), seed=7)
    run_and_check(step, host_hints=hints)


def test_packed_inputs_one_host_copy():
    """A step's inputs are one device buffer: one H2D copy of host_inputs()
    restores all of them, and the step then gives the same bytes."""
    from paged_kv_cache_469_b200.step import DeviceStep
    step = random_step(101, dtype="bf16", num_q_heads=32, num_kv_heads=4, head_dim=64,
                       num_seqs=6, max_ctx=500, max_q=2)
    ds = DeviceStep(step)
    ds.run_fused()
    torch.cuda.synchronize()
    ref = _bits(ds.out).copy()
    host = ds.host_inputs()
    ds.inputs.zero_()
    ds.inputs.copy_(host, non_blocking=True)
    ds.out.zero_()
    ds.run_fused()
    torch.cuda.synchronize()
    assert _bits(ds.out).tobytes() == ref.tobytes()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv,ql", [(32, 4, 3), (32, 4, 8), (32, 8, 5), (32, 8, 16),
                                       (16, 1, 3), (8, 8, 40), (32, 8, 17)])
@pytest.mark.parametrize("hints", [True, False])
def test_multi_token_decode_row_groups(d, hq, hkv, ql, hints):
    """Queries of 17..64 rows per kv-head (q_len * group) stay on the split-K
    decode kernel as up to four 16-row groups (one CTA each, each with its own
    partials and merge), mixed with one-token decodes and, for (32, 8, 17),
    with a prefill-class neighbour (68 rows)."""
    lens = [5000, 37, 300, 16, ql, 1200]
    qls = [ql, 1, ql, 1, ql, min(ql, 1200)]
    step = make_step(name="mtd_rg", dtype="bf16", num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                     num_blocks=int(np.sum((np.array(lens) + 15) // 16)) + 30, seq_lens=lens,
                     query_lens=qls, seed=11 + ql)
    run_and_check(step, host_hints=hints)


@pytest.mark.parametrize("ql", [3, 8])
def test_write_cache_call_row_groups(ql):
    """The one-call path on multi-token decodes: every row group of a partition
    writes the same new rows and reads them back."""
    lens = np.array([2100, 700, 33, ql])
    step = make_step(name="fused_rg", dtype="bf16", num_q_heads=32, num_kv_heads=4, head_dim=64,
                     num_blocks=int(np.sum((lens + 15) // 16)) + 20, seq_lens=lens,
                     query_lens=np.full(4, ql), seed=23 + ql)
    _fused_check(step)


@pytest.mark.parametrize("d", [64, 128])
def test_mixed_step_classes_side_by_side_join_the_stream(d):
    """A step with prefill chunks and decodes, host copies given, runs its two
    classes of work side by side (the prefill kernel on a side stream, on a
    share of the SMs).  Work queued on the caller's stream right after the
    call, with no host synchronisation in between, must see every output row
    of both classes: here a copy of the output, compared with the oracle."""
    from paged_kv_cache_469_b200.step import DeviceStep
    lens = [3000, 2600, 1800, 1200, 900, 700, 64, 33, 2000, 5000]
    qls = [1024, 768, 1, 1, 1, 1, 1, 1, 300, 2]
    step = make_step(name="side_by_side", dtype="bf16", num_q_heads=32, num_kv_heads=8,
                     head_dim=d, num_blocks=int(np.sum((np.array(lens) + 15) // 16)) + 16,
                     seq_lens=lens, query_lens=qls, seed=41 + d)
    ds = DeviceStep(step)
    st = oracle_state(step)
    ref = oracle_outputs(step, st, num_threads=NTHREADS)
    for rep in range(3):
        ds.out.fill_(float("nan"))
        ds.run()
        snap = ds.out.clone()  # same stream, queued right behind the call
        torch.cuda.synchronize()
        assert_close(snap.float().cpu().numpy().astype(np.float64), ref, "bf16",
                     f"side-by-side step, rep {rep}")
