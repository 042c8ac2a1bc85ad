"""One paged-attention step on the GPU, end to end, through the C ABI.

``DeviceStep`` takes a step description (``inputs.StepInputs``), plans it on
the host (block allocation, slot mapping, super-sequence offsets), puts the
cache and the step's tensors in device memory, writes the earlier tokens' K/V
into the cache with ``pa_reshape_and_cache``, and then runs the step itself:
``run`` makes two calls (``pa_reshape_and_cache`` for the new tokens, then
``pa_attention_varlen``), ``run_fused`` makes one
(``pa_attention_varlen_write_cache``).  The step's inputs sit in one device
buffer, so one copy from ``host_inputs()`` refills them.  ``capture`` records
a step in a CUDA graph, the way a serving loop replays a steady decode step
without paying the host cost of each call again.
"""
from __future__ import annotations

import numpy as np
import torch

from . import lib
from .block_pool import plan_step
from .inputs import StepInputs


_TORCH_DTYPE = {np.dtype(np.uint16): torch.bfloat16, np.dtype(np.float32): torch.float32,
                np.dtype(np.int32): torch.int32, np.dtype(np.int64): torch.int64}


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
        # the step's inputs live in one contiguous device buffer (each 256-byte
        # aligned), so that a caller bringing them from the host needs one copy
        self._input_arrays = [("q", step.q), ("k_new", step.k_new), ("v_new", step.v_new),
                              ("slot_mapping", plan.slot_mapping),
                              ("block_tables", plan.block_tables),
                              ("seq_lens", plan.seq_lens),
                              ("query_start_loc", plan.query_start_loc)]
        self._layout, total = [], 0
        for name, a in self._input_arrays:
            a = np.ascontiguousarray(a)
            self._layout.append((name, total, a.nbytes, a.dtype, a.shape))
            total += (a.nbytes + 255) // 256 * 256
        self.inputs = torch.empty(total, dtype=torch.uint8, device=device)
        for (name, off, nbytes, dt, shape), (_, a) in zip(self._layout, self._input_arrays):
            view = self.inputs[off:off + nbytes].view(_TORCH_DTYPE[np.dtype(dt)]).view(shape)
            view.copy_(to_torch(np.ascontiguousarray(a), "cpu"))
            setattr(self, name, view)
        self.out = torch.empty_like(self.q)
        self.workspace = lib.new_workspace(step.num_seqs, step.num_q_heads, step.num_kv_heads,
                                           step.head_dim, max(1, plan.max_seq_len), device)
        torch.cuda.synchronize()

    def host_inputs(self) -> torch.Tensor:
        """A pinned host copy of ``inputs`` (same layout): one H2D copy of it
        into ``inputs`` gives the step all of its inputs."""
        host = torch.zeros(self.inputs.numel(), dtype=torch.uint8).pin_memory()
        for (name, off, nbytes, dt, shape), (_, a) in zip(self._layout, self._input_arrays):
            host[off:off + nbytes].copy_(
                torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)))
        return host

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
