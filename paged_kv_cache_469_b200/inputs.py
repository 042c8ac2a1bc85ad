"""Seeded synthetic inputs for one paged-attention step.

This module draws random numbers and nothing else: sequence lengths, the
shuffled ``free_block_queue`` and the q/k/v values.  It holds none of the
method's arithmetic (no block counting, slot mapping, prefix sums or
attention); the CUDA path and the CPU oracle each do that on their own, from
the same draws.

The workloads mirror the shapes the pages talk about (page
"LLM推論エンジンvLLMの内部構造を徹底解説", sections "PagedAttentionの仕組み",
"高度な機能群" and "エンジンの中核"): 16-token blocks, a pool of up to a few
hundred thousand blocks handed out from a shuffled free queue, decode steps of
one query token per sequence, chunked prefill over already cached context,
prefix-shared block lists, and steps that mix prefill chunks with decodes.

Values: every q/k/v element is an independent N(0, 1) draw in fp32 (numpy
``standard_normal``), rounded to bf16 (round to nearest even) for bf16
workloads.  Large arrays are drawn in fixed chunks of 2**22 values, chunk c
from ``default_rng([seed, stream, c])``, so the values do not depend on how
many threads draw them.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass, field

import numpy as np

_CHUNK = 1 << 22

# stream tags of the independent value streams of one step
_S_Q, _S_KNEW, _S_VNEW, _S_KCTX, _S_VCTX = 1, 2, 3, 4, 5


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of finite fp32 values, round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >>
            np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


def normal_values(seed: int, stream: int, n: int, dtype: str) -> np.ndarray:
    """n independent N(0,1) values: float32 for "f32", bf16 bits (uint16) for "bf16"."""
    out = np.empty(n, dtype=np.float32 if dtype == "f32" else np.uint16)
    nchunks = (n + _CHUNK - 1) // _CHUNK

    def fill(c: int) -> None:
        s = c * _CHUNK
        e = min(n, s + _CHUNK)
        g = np.random.default_rng([seed, stream, c])
        vals = g.standard_normal(e - s, dtype=np.float32)
        out[s:e] = vals if dtype == "f32" else f32_to_bf16_bits(vals)

    if nchunks <= 1:
        for c in range(nchunks):
            fill(c)
    else:
        with _cf.ThreadPoolExecutor(min(_threads(), nchunks)) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


@dataclass
class StepInputs:
    """Everything a scheduler would hand the attention layer for one step.

    Sequence s has ``seq_lens[s]`` KV tokens in total after this step, the last
    ``query_lens[s]`` of which are this step's new tokens.  Sequences appear in
    super-sequence order.  The K/V of earlier tokens ("context") must already
    be in the cache before the step: ``k_ctx``/``v_ctx`` hold them, sequence s
    owning rows for positions ``ctx_first_pos[s]`` .. ``+ctx_count[s]-1``.
    With a shared prefix of ``shared_prefix_tokens`` tokens, sequence 0 owns
    the prefix rows and every other sequence's context starts after it.
    """

    name: str
    dtype: str  # "f32" or "bf16" (bf16 arrays are uint16 bit patterns)
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    seed: int
    seq_lens: np.ndarray  # int32 [S]
    query_lens: np.ndarray  # int32 [S]
    shared_prefix_tokens: int
    free_queue: np.ndarray  # int32 [num_blocks]: free_block_queue, front first
    q: np.ndarray  # [T, Hq, D]
    k_new: np.ndarray  # [T, Hkv, D]
    v_new: np.ndarray  # [T, Hkv, D]
    ctx_first_pos: np.ndarray  # int32 [S]
    ctx_count: np.ndarray  # int32 [S]
    k_ctx: np.ndarray  # [sum(ctx_count), Hkv, D]
    v_ctx: np.ndarray
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(len(self.seq_lens))

    @property
    def num_tokens(self) -> int:
        return int(self.q.shape[0])

    @property
    def scale(self) -> float:
        return float(1.0 / np.sqrt(self.head_dim))


def make_step(*, name: str, dtype: str, num_q_heads: int, num_kv_heads: int, head_dim: int,
              num_blocks: int, seq_lens, query_lens, seed: int, block_size: int = 16,
              shared_prefix_tokens: int = 0, rng: np.random.Generator | None = None,
              with_values: bool = True) -> StepInputs:
    """Draw the free queue and the values of a step whose lengths are given."""
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    query_lens = np.asarray(query_lens, dtype=np.int32)
    if rng is None:
        rng = np.random.default_rng(seed)
    free_queue = rng.permutation(num_blocks).astype(np.int32)

    ctx_count = (seq_lens - query_lens).astype(np.int64)
    ctx_first = np.zeros(len(seq_lens), dtype=np.int64)
    if shared_prefix_tokens:
        ctx_first[1:] = shared_prefix_tokens
        ctx_count[1:] -= shared_prefix_tokens
    t = int(query_lens.sum())
    nctx = int(ctx_count.sum())
    hq, hkv, d = num_q_heads, num_kv_heads, head_dim

    def draw(stream, rows, heads):
        if not with_values:
            return np.zeros((rows, heads, d), dtype=np.float32 if dtype == "f32" else np.uint16)
        return normal_values(seed, stream, rows * heads * d, dtype).reshape(rows, heads, d)

    return StepInputs(
        name=name, dtype=dtype, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
        block_size=block_size, num_blocks=num_blocks, seed=seed, seq_lens=seq_lens,
        query_lens=query_lens, shared_prefix_tokens=shared_prefix_tokens,
        free_queue=free_queue, q=draw(_S_Q, t, hq), k_new=draw(_S_KNEW, t, hkv),
        v_new=draw(_S_VNEW, t, hkv), ctx_first_pos=ctx_first.astype(np.int32),
        ctx_count=ctx_count.astype(np.int32), k_ctx=draw(_S_KCTX, nctx, hkv),
        v_ctx=draw(_S_VCTX, nctx, hkv))


# --------------------------------------------------------------------------
# the five workloads (lengths drawn from default_rng(seed) before anything else)
# --------------------------------------------------------------------------

WORKLOADS = ("tiny_f32", "decode_tinyllama", "mixed_llama3_8b", "prefix_decode_llama3_8b",
             "long_decode_llama3_8b")


def workload(name: str, *, with_values: bool = True) -> StepInputs:
    """One of the five named workloads (seed 1001..1005 in the order above).

    - tiny_f32: fp32, 4 q / 4 kv heads, D=64, 64-block pool; a 17-token prefill
      and decodes at context 33 and 48.
    - decode_tinyllama: bf16, TinyLlama-1.1B attention shape (32 q / 4 kv heads,
      D=64); 64 decodes with context U[128, 2048]; 100k-block pool.
    - mixed_llama3_8b: bf16, Llama-3-8B attention shape (32 q / 8 kv heads,
      D=128); 4 prefill chunks of 512 tokens over prior context U[0, 4096],
      then 192 decodes with context U[256, 8192]; 100k-block pool.
    - prefix_decode_llama3_8b: 128 decodes sharing a 1024-token (64-block)
      prefix, then a private suffix U[0, 2048] and the decode token;
      200k-block pool.
    - long_decode_llama3_8b: 16 decodes with context U[32768, 131072];
      131072-block pool (8.59 GB of K+V).
    """
    idx = WORKLOADS.index(name)
    seed = 1001 + idx
    rng = np.random.default_rng(seed)
    common = dict(name=name, seed=seed, rng=rng, with_values=with_values)
    if name == "tiny_f32":
        return make_step(dtype="f32", num_q_heads=4, num_kv_heads=4, head_dim=64,
                         num_blocks=64, seq_lens=[17, 33, 48], query_lens=[17, 1, 1], **common)
    if name == "decode_tinyllama":
        lens = rng.integers(128, 2048, size=64, endpoint=True)
        return make_step(dtype="bf16", num_q_heads=32, num_kv_heads=4, head_dim=64,
                         num_blocks=100_000, seq_lens=lens, query_lens=np.ones(64, np.int32),
                         **common)
    if name == "mixed_llama3_8b":
        prior = rng.integers(0, 4096, size=4, endpoint=True)
        dec = rng.integers(256, 8192, size=192, endpoint=True)
        lens = np.concatenate([prior + 512, dec])
        qls = np.concatenate([np.full(4, 512), np.ones(192)])
        return make_step(dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                         num_blocks=100_000, seq_lens=lens, query_lens=qls, **common)
    if name == "prefix_decode_llama3_8b":
        suffix = rng.integers(0, 2048, size=128, endpoint=True)
        lens = 1024 + suffix + 1
        return make_step(dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                         num_blocks=200_000, seq_lens=lens, query_lens=np.ones(128, np.int32),
                         shared_prefix_tokens=1024, **common)
    if name == "long_decode_llama3_8b":
        lens = rng.integers(32768, 131072, size=16, endpoint=True)
        return make_step(dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                         num_blocks=131_072, seq_lens=lens, query_lens=np.ones(16, np.int32),
                         **common)
    raise KeyError(name)


def prefill_part(step: StepInputs, decode_rows: int = 64) -> StepInputs:
    """A step of the same shape holding only ``step``'s prefill-class sequences
    (q_len * group > ``decode_rows``), with the same lengths, fresh draws from
    the same seed and a pool just large enough for them."""
    g = step.num_q_heads // step.num_kv_heads
    idx = [i for i, q in enumerate(step.query_lens.tolist()) if q * g > decode_rows]
    lens, qls = step.seq_lens[idx], step.query_lens[idx]
    return make_step(name=f"{step.name}_prefill_only", dtype=step.dtype,
                     num_q_heads=step.num_q_heads, num_kv_heads=step.num_kv_heads,
                     head_dim=step.head_dim, num_blocks=int(np.sum((lens + 15) // 16)) + 64,
                     seq_lens=lens, query_lens=qls, seed=step.seed)


def random_step(seed: int, *, dtype: str = "bf16", num_q_heads: int = 8, num_kv_heads: int = 2,
                head_dim: int = 64, num_seqs: int = 4, max_ctx: int = 100, max_q: int = 20,
                num_blocks: int | None = None, shared_prefix_tokens: int = 0) -> StepInputs:
    """A small random step mixing decodes and prefill chunks (for parity tests)."""
    rng = np.random.default_rng(seed)
    qls = rng.integers(1, max_q, size=num_seqs, endpoint=True)
    ctx = rng.integers(0, max_ctx, size=num_seqs, endpoint=True)
    lens = qls + ctx + shared_prefix_tokens
    if num_blocks is None:
        num_blocks = int(lens.sum()) // 16 + 2 * num_seqs + 8  # ample: an upper bound
    return make_step(name=f"random{seed}", dtype=dtype, num_q_heads=num_q_heads,
                     num_kv_heads=num_kv_heads, head_dim=head_dim, num_blocks=num_blocks,
                     seq_lens=lens, query_lens=qls, seed=seed, rng=rng,
                     shared_prefix_tokens=shared_prefix_tokens)


def planner_draws(seed: int, *, num_seqs: int, num_blocks: int, max_ctx: int = 4096,
                  max_chunk: int = 512, prefill_frac: float = 0.1, idle_frac: float = 0.05):
    """Draws for one scheduler step of the block planner: a shuffled
    free_block_queue, the tokens each sequence already holds blocks for, and
    the tokens it schedules now (mostly one-token decodes, some prefill chunks
    of 2..max_chunk tokens, a few sequences with nothing scheduled)."""
    rng = np.random.default_rng([seed, 7])
    free_queue = rng.permutation(num_blocks).astype(np.int32)
    num_computed = rng.integers(0, max_ctx, size=num_seqs, endpoint=True).astype(np.int32)
    kind = rng.random(num_seqs)
    chunk = rng.integers(2, max(2, max_chunk), size=num_seqs, endpoint=True)
    query_lens = np.where(kind < idle_frac, 0,
                          np.where(kind < idle_frac + prefill_frac, chunk, 1)).astype(np.int32)
    return free_queue, num_computed, query_lens
