"""CPU oracle for paged attention (fp64) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (``paged_kv_cache_469_b200``)
never does, and the two share no code: they meet only through the seeded
synthetic inputs of ``paged_kv_cache_469_b200.inputs``.

The arithmetic lives in ``pa_oracle.c`` (plain C, fp64); this module loads it
with ctypes and passes numpy arrays.  bf16 tensors travel as ``np.uint16`` bit
patterns, fp32 tensors as ``np.float32``.

Every function follows the page "LLM推論エンジンvLLMの内部構造を徹底解説"
(techfeed.io), section "PagedAttentionの仕組み" (16-token blocks, ceil block
count, allocate_slots popping the front of free_block_queue into
req_to_blocks, the flattened super-sequence with a per-sequence mask) and
section "高度な機能群" (chunked prefill over cached context, shared prefix
blocks).  Pins: ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, library_path

F32 = 0
BF16 = 1

_lib = None
_lib_path_override = None


def use_library(path: str | None) -> None:
    """Load the oracle from another build of it (tests that plant a mistake in a
    modified copy of the C source use this to check that the pins catch it);
    None goes back to the normal build."""
    global _lib, _lib_path_override
    _lib = None
    _lib_path_override = path


def _load():
    global _lib
    if _lib is None:
        path = _lib_path_override or library_path()
        if _lib_path_override is None and not os.path.exists(path):
            build_oracle()
        lib = ctypes.CDLL(path)
        c_i64, c_i32, c_int, c_p, c_d = (ctypes.c_int64, ctypes.c_int32, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_double)
        lib.oracle_blocks_needed.restype = c_i64
        lib.oracle_blocks_needed.argtypes = [c_i64, c_i64]
        lib.oracle_allocate_block_tables.restype = c_int
        lib.oracle_allocate_block_tables.argtypes = [c_p, c_i64, c_int, c_p, c_int, c_int,
                                                     c_int, c_i32, c_p, c_p]
        lib.oracle_query_start_loc.restype = None
        lib.oracle_query_start_loc.argtypes = [c_p, c_int, c_p]
        lib.oracle_slot_mapping.restype = c_int
        lib.oracle_slot_mapping.argtypes = [c_p, c_int, c_int, c_p, c_p, c_int, c_p]
        lib.oracle_plan_step.restype = c_int
        lib.oracle_plan_step.argtypes = [c_p, c_i64, c_p, c_p, c_p, c_int, c_p, c_int, c_int,
                                         c_p, c_p, c_p, c_i64]
        lib.oracle_reshape_and_cache.restype = None
        lib.oracle_reshape_and_cache.argtypes = [c_p, c_p, c_p, c_p, c_p, c_i64, c_int, c_int,
                                                 c_int, c_int]
        lib.oracle_paged_attention.restype = c_int
        lib.oracle_paged_attention.argtypes = [c_p, c_p, c_p, c_p, c_int, c_p, c_p, c_int,
                                               c_int, c_int, c_int, c_int, c_d, c_int, c_p,
                                               c_int]
        lib.oracle_paged_attention_rows.restype = c_int
        lib.oracle_paged_attention_rows.argtypes = [c_p, c_p, c_p, c_p, c_int, c_p, c_p, c_int,
                                                    c_int, c_int, c_int, c_int, c_d, c_int,
                                                    c_i64, c_p, c_p, c_p, c_int]
        lib.oracle_round_to_bf16.restype = None
        lib.oracle_round_to_bf16.argtypes = [c_p, c_i64, c_p]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _dtype_code(arr: np.ndarray) -> int:
    if arr.dtype == np.float32:
        return F32
    if arr.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or bf16-as-uint16 arrays, got {arr.dtype}")


def blocks_needed(num_tokens: int, block_size: int = 16) -> int:
    """ceil(num_tokens / block_size): blocks a request of num_tokens occupies."""
    return int(_load().oracle_blocks_needed(num_tokens, block_size))


def allocate_block_tables(free_queue: np.ndarray, seq_lens: np.ndarray, *,
                          block_size: int = 16, max_blocks_per_seq: int,
                          shared_prefix_tokens: int = 0, pad_value: int = 0):
    """allocate_slots steps 1 and 3 for each request in order -> (block_tables, taken)."""
    fq = np.ascontiguousarray(free_queue, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    tables = np.empty((len(sl), max_blocks_per_seq), dtype=np.int32)
    taken = ctypes.c_int64(0)
    rc = _load().oracle_allocate_block_tables(_ptr(fq), len(fq), len(sl), _ptr(sl),
                                              shared_prefix_tokens, block_size,
                                              max_blocks_per_seq, pad_value, _ptr(tables),
                                              ctypes.addressof(taken))
    if rc != 0:
        raise ValueError("oracle allocation failed (pool exhausted or bad sizes)")
    return tables, int(taken.value)


def query_start_loc(query_lens: np.ndarray) -> np.ndarray:
    """Offsets of each sequence's query rows in the flattened super-sequence, [S+1]."""
    ql = np.ascontiguousarray(query_lens, dtype=np.int32)
    out = np.empty(len(ql) + 1, dtype=np.int32)
    _load().oracle_query_start_loc(_ptr(ql), len(ql), _ptr(out))
    return out


def slot_mapping(block_tables: np.ndarray, first_pos: np.ndarray, count: np.ndarray,
                 block_size: int = 16) -> np.ndarray:
    """Slots of positions first_pos[s] .. first_pos[s]+count[s]-1 of each sequence."""
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    fp = np.ascontiguousarray(first_pos, dtype=np.int32)
    ct = np.ascontiguousarray(count, dtype=np.int32)
    out = np.empty(int(ct.sum()), dtype=np.int64)
    rc = _load().oracle_slot_mapping(_ptr(bt), bt.shape[1], bt.shape[0], _ptr(fp), _ptr(ct),
                                     block_size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle slot mapping: position beyond the block table")
    return out


def plan_step(free_queue: np.ndarray, head: int, block_tables: np.ndarray,
              num_computed: np.ndarray, query_lens: np.ndarray, *, block_size: int = 16,
              max_tokens: int | None = None):
    """One scheduler step of block planning (allocate_slots for a running batch)
    -> (block_tables, seq_lens, query_start_loc, slots, new head); the input
    table is not modified.  Raises ValueError when the step does not fit."""
    fq = np.ascontiguousarray(free_queue, dtype=np.int32)
    nc = np.ascontiguousarray(num_computed, dtype=np.int32)
    ql = np.ascontiguousarray(query_lens, dtype=np.int32)
    tables = np.array(block_tables, dtype=np.int32, copy=True, order="C")
    s = len(ql)
    seq_lens = np.empty(s, dtype=np.int32)
    qsl = np.empty(s + 1, dtype=np.int32)
    total = int(np.maximum(ql, 0).sum())
    cap = total if max_tokens is None else int(max_tokens)
    slots = np.empty(max(total, 1), dtype=np.int64)
    h = ctypes.c_int64(int(head))
    rc = _load().oracle_plan_step(_ptr(fq), len(fq), ctypes.addressof(h), _ptr(nc), _ptr(ql), s,
                                  _ptr(tables), tables.shape[1], block_size, _ptr(seq_lens),
                                  _ptr(qsl), _ptr(slots), cap)
    if rc != 0:
        raise ValueError("oracle plan_step: the step does not fit (pool, row, slots or counts)")
    return tables, seq_lens, qsl, slots[:total], int(h.value)


def reshape_and_cache(k: np.ndarray, v: np.ndarray, k_cache: np.ndarray,
                      v_cache: np.ndarray, slots: np.ndarray) -> None:
    """Write rows k[i], v[i] ([Hkv, D]) into cache slot slots[i] (in place)."""
    assert k.dtype == v.dtype == k_cache.dtype == v_cache.dtype
    num_blocks, hkv, bs, d = k_cache.shape
    sm = np.ascontiguousarray(slots, dtype=np.int64)
    _load().oracle_reshape_and_cache(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(sm),
                                     len(sm), hkv, d, bs, k.dtype.itemsize)


def paged_attention(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc, *,
                    num_q_heads: int, scale: float, num_threads: int = 1) -> np.ndarray:
    """All output rows of the step, fp64, before any rounding: [T, Hq, D]."""
    num_blocks, hkv, bs, d = k_cache.shape
    dt = _dtype_code(q)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
    t = int(qsl[-1])
    out = np.zeros((t, num_q_heads, d), dtype=np.float64)
    rc = _load().oracle_paged_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(bt),
                                        bt.shape[1], _ptr(sl), _ptr(qsl), len(sl),
                                        num_q_heads, hkv, d, bs, float(scale), dt, _ptr(out),
                                        num_threads)
    if rc != 0:
        raise ValueError("oracle attention: malformed step description")
    return out


def paged_attention_rows(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc,
                         row_token, row_head, *, num_q_heads: int, scale: float,
                         num_threads: int = 1) -> np.ndarray:
    """Selected output rows (token row_token[r], head row_head[r]) -> [R, D] fp64."""
    num_blocks, hkv, bs, d = k_cache.shape
    dt = _dtype_code(q)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
    rt = np.ascontiguousarray(row_token, dtype=np.int64)
    rh = np.ascontiguousarray(row_head, dtype=np.int32)
    out = np.zeros((len(rt), d), dtype=np.float64)
    rc = _load().oracle_paged_attention_rows(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(bt),
                                             bt.shape[1], _ptr(sl), _ptr(qsl), len(sl),
                                             num_q_heads, hkv, d, bs, float(scale), dt,
                                             len(rt), _ptr(rt), _ptr(rh), _ptr(out),
                                             num_threads)
    if rc != 0:
        raise ValueError("oracle attention: malformed step description")
    return out


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest bf16 (ties to even) of each fp64 value, as uint16 bit patterns."""
    xs = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(xs.shape, dtype=np.uint16)
    _load().oracle_round_to_bf16(_ptr(xs), xs.size, _ptr(out))
    return out
