"""pa_attention_varlen_static_scratch: the attention call for callers that
cannot allocate device memory (allocator callbacks, plugins that are handed
only their inputs and outputs, paths where a cudaMalloc is not allowed).  It
keeps its scratch in a fixed array inside the library instead of a workspace
from the caller.

Its result must match pa_attention_varlen's on the same step, on two calls in
a row (the second call finds the first call's leftovers in the shared array).
This file is collected last so that a run stopping at the first failure has
already run every other test."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_469_b200 import lib
from paged_kv_cache_469_b200.inputs import make_step, random_step
from tests.oracle_side import oracle_outputs, oracle_state
from tests.test_gpu_parity import assert_close

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 16 << 20  # PA_STATIC_SCRATCH_BYTES in include/pa.h


def _entry():
    f = lib.library().pa_attention_varlen_static_scratch
    c_int, c_p, c_f = ctypes.c_int, ctypes.c_void_p, ctypes.c_float
    f.restype = c_int
    f.argtypes = [c_p, c_p, c_p, c_p, c_p, c_int, c_p, c_p, c_int, c_int, c_int, c_int, c_int,
                  c_int, c_int, c_int, c_int, c_f, c_int, c_p, c_p, c_p]
    return f


def _call(f, ds, out, hints=True, max_seq_len=None):
    p = ds.plan
    sl = np.ascontiguousarray(p.seq_lens, np.int32)
    qs = np.ascontiguousarray(p.query_start_loc, np.int32)
    q = ds.q
    dt = lib.PA_DTYPE_F32 if q.dtype == torch.float32 else lib.PA_DTYPE_BF16
    return f(out.data_ptr(), q.data_ptr(), ds.k_cache.data_ptr(), ds.v_cache.data_ptr(),
             ds.block_tables.data_ptr(), ds.block_tables.shape[1], ds.seq_lens.data_ptr(),
             ds.query_start_loc.data_ptr(), len(sl), q.shape[0], p.max_query_len,
             max_seq_len or p.max_seq_len, q.shape[1], ds.k_cache.shape[1], q.shape[2],
             ds.k_cache.shape[2], ds.k_cache.shape[0], float(ds.step.scale), dt,
             sl.ctypes.data if hints else None, qs.ctypes.data if hints else None,
             torch.cuda.current_stream().cuda_stream)


def test_static_scratch_matches_workspace_call_twice():
    from paged_kv_cache_469_b200.step import DeviceStep
    f = _entry()
    # two different steps (decode-class and prefill-class sequences, both head
    # sizes), so the second call sees a different layout's leftovers
    steps = [random_step(901, dtype="bf16", num_q_heads=16, num_kv_heads=4, head_dim=128,
                         num_seqs=8, max_ctx=1500, max_q=150),
             random_step(902, dtype="bf16", num_q_heads=32, num_kv_heads=4, head_dim=64,
                         num_seqs=12, max_ctx=2500, max_q=3)]
    for step in steps:
        ds = DeviceStep(step)
        need = lib.attention_workspace_size(step.num_seqs, step.num_q_heads, step.num_kv_heads,
                                            step.head_dim, ds.plan.max_seq_len)
        assert 0 < need <= STATIC_SCRATCH_BYTES
        ds.run()  # the workspace path: cache write + pa_attention_varlen
        torch.cuda.synchronize()
        ref = ds.out.float().cpu().numpy().astype(np.float64)
        for _ in range(2):
            out = torch.full_like(ds.out, float("nan"))
            assert _call(f, ds, out) == lib.PA_OK
            torch.cuda.synchronize()
            assert_close(out.float().cpu().numpy().astype(np.float64), ref, "bf16",
                         "static-scratch call vs workspace call")


def test_static_scratch_rejects_a_step_beyond_its_size():
    f = _entry()
    dev = "cuda"
    kc = torch.zeros(4, 8, 16, 128, dtype=torch.bfloat16, device=dev)
    q = torch.zeros(1, 32, 128, dtype=torch.bfloat16, device=dev)
    bt = torch.zeros(1, 8192, dtype=torch.int32, device=dev)
    sl = torch.ones(1, dtype=torch.int32, device=dev)
    qs = torch.tensor([0, 1], dtype=torch.int32, device=dev)
    big_seqs, big_len = 4096, 131072  # far more scratch than the fixed array holds
    assert lib.attention_workspace_size(big_seqs, 32, 8, 128, big_len) > STATIC_SCRATCH_BYTES
    rc = f(q.data_ptr(), q.data_ptr(), kc.data_ptr(), kc.data_ptr(), bt.data_ptr(), 8192,
           sl.data_ptr(), qs.data_ptr(), big_seqs, 1, 1, big_len, 32, 8, 128, 16, 4, 0.1,
           lib.PA_DTYPE_BF16, None, None, torch.cuda.current_stream().cuda_stream)
    assert rc == lib.PA_ERR_INVALID


def test_static_scratch_against_the_oracle():
    """One static-scratch call checked straight against the fp64 oracle, not
    only against the workspace path."""
    from paged_kv_cache_469_b200.step import DeviceStep
    f = _entry()
    step = random_step(903, dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                       num_seqs=7, max_ctx=2000, max_q=200)
    ds = DeviceStep(step)
    ds.write_new_tokens()
    out = torch.full_like(ds.out, float("nan"))
    assert _call(f, ds, out) == lib.PA_OK
    torch.cuda.synchronize()
    ref = oracle_outputs(step, oracle_state(step), num_threads=8)
    assert_close(out.float().cpu().numpy().astype(np.float64), ref, "bf16",
                 "static-scratch call vs oracle")


def test_static_scratch_smaller_layout_after_larger_split_k():
    """A step whose sequences are cut into many pieces fills the array's
    partials and decode work list under a large layout; a smaller step with
    pieces of its own follows, without host copies (so its work list is built
    on the device), and must still be right: its header words and lists lie
    where the larger layout kept other data."""
    from paged_kv_cache_469_b200.step import DeviceStep
    f = _entry()
    big = make_step(name="big", dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                    num_blocks=2200, seq_lens=[9000, 7000, 8000, 5000], query_lens=[1, 1, 1, 1],
                    seed=31)
    small = make_step(name="small", dtype="bf16", num_q_heads=16, num_kv_heads=4, head_dim=64,
                      num_blocks=700, seq_lens=[4000, 3000, 2500, 1], query_lens=[1, 2, 1, 1],
                      seed=32)
    for step, hints in ((big, True), (small, False), (big, False), (small, True)):
        ds = DeviceStep(step)
        ds.write_new_tokens()
        out = torch.full_like(ds.out, float("nan"))
        assert _call(f, ds, out, hints=hints) == lib.PA_OK
        torch.cuda.synchronize()
        ref = oracle_outputs(step, oracle_state(step), num_threads=8)
        assert_close(out.float().cpu().numpy().astype(np.float64), ref, "bf16",
                     f"static-scratch {step.name} (host copies: {hints})")


def test_static_scratch_fp32_steps_use_no_scratch():
    """fp32 steps run the CUDA-core kernel, which needs no scratch: a bound far
    beyond the array's size is not refused, and the result is the oracle's."""
    from paged_kv_cache_469_b200.step import DeviceStep
    f = _entry()
    step = random_step(904, dtype="f32", num_q_heads=8, num_kv_heads=2, head_dim=64,
                       num_seqs=64, max_ctx=200, max_q=20)
    bound = 1 << 20
    ds = DeviceStep(step, max_blocks_per_seq=bound // 16)
    assert lib.attention_workspace_size(64, 8, 2, 64, bound) > STATIC_SCRATCH_BYTES
    ds.write_new_tokens()
    out = torch.full_like(ds.out, float("nan"))
    assert _call(f, ds, out, max_seq_len=bound) == lib.PA_OK
    torch.cuda.synchronize()
    ref = oracle_outputs(step, oracle_state(step), num_threads=8)
    assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 1e-4
