"""One paged-attention step on the GPU, end to end, through the C ABI.

``DeviceStep`` takes a step description (``inputs.StepInputs``), plans it on
the host (block allocation, slot mapping, super-sequence offsets), puts the
cache and the step's tensors in device memory, writes the earlier tokens' K/V
into the cache with ``pa_reshape_and_cache``, and then runs the step itself:
``pa_reshape_and_cache`` for the new tokens followed by
``pa_attention_varlen``.  ``capture`` records those launches in a CUDA graph,
the way a serving loop replays a steady decode step without paying the host
cost of each call again.
"""
from __future__ import annotations

import numpy as np
import torch

from . import lib
from .block_pool import plan_step
from .inputs import StepInputs


def to_torch(a: np.ndarray, device) -> torch.Tensor:
    """numpy array (float32, or uint16 holding bf16 bits, or ints) -> torch tensor."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.to(device, non_blocking=False)


class DeviceStep:
    def __init__(self, step: StepInputs, device: str = "cuda", *, max_blocks_per_seq=None,
                 ctx_chunk_rows: int = 1 << 18, cache_fill: float = 0.0):
        self.step = step
        self.device = device
        plan = plan_step(free_queue=step.free_queue, seq_lens=step.seq_lens,
                         query_lens=step.query_lens, ctx_first_pos=step.ctx_first_pos,
                         ctx_count=step.ctx_count, block_size=step.block_size,
                         shared_prefix_tokens=step.shared_prefix_tokens,
                         max_blocks_per_seq=max_blocks_per_seq)
        self.plan = plan
        dt = torch.float32 if step.dtype == "f32" else torch.bfloat16
        shape = (step.num_blocks, step.num_kv_heads, step.block_size, step.head_dim)
        # cache_fill: what the never-written slots hold (a pool fresh from the
        # allocator may hold anything; NaN is the worst case)
        self.k_cache = torch.full(shape, cache_fill, dtype=dt, device=device)
        self.v_cache = torch.full(shape, cache_fill, dtype=dt, device=device)
        # earlier tokens' K/V: written through the library, in chunks of rows
        n = step.k_ctx.shape[0]
        for s in range(0, n, ctx_chunk_rows):
            e = min(n, s + ctx_chunk_rows)
            lib.reshape_and_cache(to_torch(step.k_ctx[s:e], device),
                                  to_torch(step.v_ctx[s:e], device), self.k_cache, self.v_cache,
                                  to_torch(plan.ctx_slot_mapping[s:e], device))
        self.q = to_torch(step.q, device)
        self.k_new = to_torch(step.k_new, device)
        self.v_new = to_torch(step.v_new, device)
        self.block_tables = to_torch(plan.block_tables, device)
        self.seq_lens = to_torch(plan.seq_lens, device)
        self.query_start_loc = to_torch(plan.query_start_loc, device)
        self.slot_mapping = to_torch(plan.slot_mapping, device)
        self.out = torch.empty_like(self.q)
        self.workspace = lib.new_workspace(step.num_seqs, step.num_q_heads, step.num_kv_heads,
                                           step.head_dim, max(1, plan.max_seq_len), device)
        torch.cuda.synchronize()

    def write_new_tokens(self, stream=None) -> None:
        lib.reshape_and_cache(self.k_new, self.v_new, self.k_cache, self.v_cache,
                              self.slot_mapping, stream=stream)

    def attention(self, stream=None, host_hints: bool = True) -> torch.Tensor:
        p = self.plan
        return lib.attention_varlen(
            self.out, self.q, self.k_cache, self.v_cache, self.block_tables, self.seq_lens,
            self.query_start_loc, max_query_len=p.max_query_len, max_seq_len=p.max_seq_len,
            scale=self.step.scale, workspace=self.workspace,
            seq_lens_host=p.seq_lens if host_hints else None,
            query_start_loc_host=p.query_start_loc if host_hints else None, stream=stream)

    def run(self, stream=None, host_hints: bool = True) -> torch.Tensor:
        """One step: cache write of the new tokens, then attention (two calls)."""
        self.write_new_tokens(stream)
        return self.attention(stream, host_hints)

    def run_fused(self, stream=None, host_hints: bool = True) -> torch.Tensor:
        """One step as a single pa_attention_varlen_write_cache call."""
        p = self.plan
        return lib.attention_varlen_write_cache(
            self.out, self.q, self.k_new, self.v_new, self.k_cache, self.v_cache,
            self.slot_mapping, self.block_tables, self.seq_lens, self.query_start_loc,
            max_query_len=p.max_query_len, max_seq_len=p.max_seq_len, scale=self.step.scale,
            workspace=self.workspace, seq_lens_host=p.seq_lens if host_hints else None,
            query_start_loc_host=p.query_start_loc if host_hints else None, stream=stream)

    def capture(self, what: str = "step", prologue=None, epilogue=None) -> torch.cuda.CUDAGraph:
        """A CUDA graph of this step's launches: "step" (cache write of the new
        tokens, then attention), "fused" (the same as one
        pa_attention_varlen_write_cache call) or "attention" (the attention
        call alone).
        ``prologue`` / ``epilogue`` are captured before / after them (for
        example host-device copies).  Replaying the graph repeats the step on
        whatever the step's device tensors hold at that time."""
        fn = {"step": self.run, "fused": self.run_fused, "attention": self.attention}[what]

        def body():
            if prologue is not None:
                prologue()
            fn()
            if epilogue is not None:
                epilogue()

        # one call outside the capture first (one-time attribute set-up)
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            body()
        torch.cuda.current_stream(self.device).wait_stream(side)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            body()
        return g

    def out_f64(self) -> np.ndarray:
        return self.out.float().cpu().numpy().astype(np.float64)
