"""Python binding of libpa.so: argument marshalling only.

Every call forwards torch tensors' device pointers and the current CUDA
stream to the C ABI declared in ``include/pa.h``; every step of the
computation runs in the library's CUDA kernels.  There is no fallback: if
the library is missing or a call fails, an exception says so.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpa.so")

PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_CUDA = 0, -1, -2, -3
PA_DTYPE_F32, PA_DTYPE_BF16 = 0, 1

# every symbol include/pa.h declares
EXPORTS = ("pa_status_string", "pa_reshape_and_cache", "pa_attention_workspace_size",
           "pa_workspace_init", "pa_workspace_status", "pa_attention_varlen",
           "pa_attention_varlen_write_cache", "pa_attention_varlen_static_scratch",
           "pa_plan_step")

_lib = None


class PAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {library().pa_status_string(status).decode()} ({status})")
        self.status = status


def library() -> ctypes.CDLL:
    """Load libpa.so (built in-tree by ``paged_kv_cache_469_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m paged_kv_cache_469_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        c_int, c_p, c_sz, c_f = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
        lib.pa_status_string.restype = ctypes.c_char_p
        lib.pa_status_string.argtypes = [c_int]
        lib.pa_reshape_and_cache.restype = c_int
        lib.pa_reshape_and_cache.argtypes = [c_p, c_p, c_p, c_p, c_p, c_int, c_int, c_int, c_int,
                                             c_int, c_int, c_p]
        lib.pa_attention_workspace_size.restype = c_sz
        lib.pa_attention_workspace_size.argtypes = [c_int, c_int, c_int, c_int, c_int]
        lib.pa_workspace_status.restype = c_int
        lib.pa_workspace_status.argtypes = [c_p, c_sz, c_p, c_p]
        lib.pa_workspace_init.restype = c_int
        lib.pa_workspace_init.argtypes = [c_p, c_sz, c_p]
        lib.pa_attention_varlen.restype = c_int
        lib.pa_attention_varlen.argtypes = [c_p, c_p, c_p, c_p, c_p, c_int, c_p, c_p, c_int,
                                            c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                            c_int, c_f, c_int, c_p, c_sz, c_p, c_p, c_p]
        lib.pa_attention_varlen_write_cache.restype = c_int
        lib.pa_attention_varlen_write_cache.argtypes = [
            c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_int, c_p, c_p, c_int, c_int, c_int, c_int,
            c_int, c_int, c_int, c_int, c_int, c_f, c_int, c_p, c_sz, c_p, c_p, c_p]
        lib.pa_plan_step.restype = c_int
        lib.pa_plan_step.argtypes = [c_p, c_int, c_p, c_p, c_p, c_int, c_p, c_int, c_int, c_p,
                                     c_p, c_p, c_int, c_p]
        _lib = lib
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return PA_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return PA_DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return t.data_ptr()


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _host_i32(a):
    """(pointer, keep-alive) of an optional host int32 array."""
    if a is None:
        return None, None
    if isinstance(a, torch.Tensor):
        a = a.cpu().numpy()
    import numpy as np
    arr = np.ascontiguousarray(a, dtype=np.int32)
    return arr.ctypes.data, arr


def reshape_and_cache(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, slot_mapping: torch.Tensor, stream=None) -> None:
    """k, v: [T, Hkv, D]; caches: [num_blocks, Hkv, 16, D]; slot_mapping: int64 [T]."""
    num_blocks, hkv, bs, d = k_cache.shape
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    rc = library().pa_reshape_and_cache(
        _dev(k, "k"), _dev(v, "v"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(slot_mapping, "slot_mapping"), k.shape[0], hkv, d, bs, num_blocks, _dtype_code(k),
        _stream(stream))
    if rc != PA_OK:
        raise PAError(rc, "pa_reshape_and_cache")


def attention_workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                             max_seq_len: int) -> int:
    return int(library().pa_attention_workspace_size(num_seqs, num_q_heads, num_kv_heads,
                                                     head_dim, max_seq_len))


def new_workspace(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                  max_seq_len: int, device="cuda", stream=None) -> torch.Tensor:
    """A zeroed workspace (uint8 CUDA tensor) sized for steps up to these bounds."""
    n = attention_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len)
    if n == 0:
        raise ValueError("invalid workspace bounds")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    rc = library().pa_workspace_init(ws.data_ptr(), n, _stream(stream))
    if rc != PA_OK:
        raise PAError(rc, "pa_workspace_init")
    return ws


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Status word of a workspace (0 = every kernel so far ran to completion)."""
    out = ctypes.c_int(0)
    rc = library().pa_workspace_status(_dev(workspace, "workspace"), workspace.numel(),
                                       ctypes.addressof(out), _stream(stream))
    if rc != PA_OK:
        raise PAError(rc, "pa_workspace_status")
    return int(out.value)


def attention_varlen(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                     v_cache: torch.Tensor, block_tables: torch.Tensor, seq_lens: torch.Tensor,
                     query_start_loc: torch.Tensor, *, max_query_len: int, max_seq_len: int,
                     scale: float, workspace: torch.Tensor | None, seq_lens_host=None,
                     query_start_loc_host=None, stream=None) -> torch.Tensor:
    """Paged attention over one flattened step (see pa_attention_varlen in pa.h)."""
    num_blocks, hkv, bs, d = k_cache.shape
    t, hq, _ = q.shape
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32 or \
            query_start_loc.dtype != torch.int32:
        raise TypeError("block_tables, seq_lens and query_start_loc must be int32")
    sl_ptr, sl_keep = _host_i32(seq_lens_host)
    qs_ptr, qs_keep = _host_i32(query_start_loc_host)
    ws_ptr, ws_n = (0, 0) if workspace is None else (_dev(workspace, "workspace"),
                                                     workspace.numel() * workspace.element_size())
    rc = library().pa_attention_varlen(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(seq_lens, "seq_lens"),
        _dev(query_start_loc, "query_start_loc"), seq_lens.shape[0], t, max_query_len,
        max_seq_len, hq, hkv, d, bs, num_blocks, float(scale), _dtype_code(q), ws_ptr, ws_n,
        sl_ptr, qs_ptr, _stream(stream))
    del sl_keep, qs_keep
    if rc != PA_OK:
        raise PAError(rc, "pa_attention_varlen")
    return out


def attention_varlen_write_cache(out: torch.Tensor, q: torch.Tensor, k_new: torch.Tensor,
                                 v_new: torch.Tensor, k_cache: torch.Tensor,
                                 v_cache: torch.Tensor, slot_mapping: torch.Tensor,
                                 block_tables: torch.Tensor, seq_lens: torch.Tensor,
                                 query_start_loc: torch.Tensor, *, max_query_len: int,
                                 max_seq_len: int, scale: float, workspace: torch.Tensor | None,
                                 seq_lens_host=None, query_start_loc_host=None,
                                 stream=None) -> torch.Tensor:
    """The step's cache write and attention in one call (see
    pa_attention_varlen_write_cache in pa.h)."""
    num_blocks, hkv, bs, d = k_cache.shape
    t, hq, _ = q.shape
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32 or \
            query_start_loc.dtype != torch.int32:
        raise TypeError("block_tables, seq_lens and query_start_loc must be int32")
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    sl_ptr, sl_keep = _host_i32(seq_lens_host)
    qs_ptr, qs_keep = _host_i32(query_start_loc_host)
    ws_ptr, ws_n = (0, 0) if workspace is None else (_dev(workspace, "workspace"),
                                                     workspace.numel() * workspace.element_size())
    rc = library().pa_attention_varlen_write_cache(
        _dev(out, "out"), _dev(q, "q"), _dev(k_new, "k_new"), _dev(v_new, "v_new"),
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(slot_mapping, "slot_mapping"),
        _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(seq_lens, "seq_lens"),
        _dev(query_start_loc, "query_start_loc"), seq_lens.shape[0], t, max_query_len,
        max_seq_len, hq, hkv, d, bs, num_blocks, float(scale), _dtype_code(q), ws_ptr, ws_n,
        sl_ptr, qs_ptr, _stream(stream))
    del sl_keep, qs_keep
    if rc != PA_OK:
        raise PAError(rc, "pa_attention_varlen_write_cache")
    return out


# bits of planner_state[1] (see pa_plan_step in pa.h)
PLAN_POOL_EMPTY, PLAN_ROW_FULL, PLAN_SLOTS_FULL, PLAN_BAD_LENGTH, PLAN_BAD_HEAD = 1, 2, 4, 8, 16


def new_planner_state(queue_head: int = 0, device="cuda") -> torch.Tensor:
    """int32[4] planner state: queue head, status bits, two words the call uses."""
    st = torch.zeros(4, dtype=torch.int32, device=device)
    st[0] = queue_head
    return st


def plan_step(free_queue: torch.Tensor, planner_state: torch.Tensor,
              num_computed: torch.Tensor, query_lens: torch.Tensor, block_tables: torch.Tensor,
              seq_lens: torch.Tensor, query_start_loc: torch.Tensor,
              slot_mapping: torch.Tensor, block_size: int = 16, stream=None) -> None:
    """Block allocation, seq_lens, query_start_loc and slot mapping of one step on
    the GPU (see pa_plan_step in pa.h); errors land in planner_state[1]."""
    for name, t in (("free_queue", free_queue), ("planner_state", planner_state),
                    ("num_computed", num_computed), ("query_lens", query_lens),
                    ("block_tables", block_tables), ("seq_lens", seq_lens),
                    ("query_start_loc", query_start_loc)):
        if t.dtype != torch.int32:
            raise TypeError(f"{name} must be int32")
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    num_seqs = query_lens.shape[0]
    if num_computed.shape[0] != num_seqs or seq_lens.shape[0] != num_seqs or \
            query_start_loc.shape[0] != num_seqs + 1 or block_tables.shape[0] != num_seqs or \
            planner_state.numel() != 4:
        raise ValueError("plan_step: inconsistent sizes")
    rc = library().pa_plan_step(
        _dev(free_queue, "free_queue"), free_queue.numel(), _dev(planner_state, "planner_state"),
        _dev(num_computed, "num_computed"), _dev(query_lens, "query_lens"), num_seqs,
        _dev(block_tables, "block_tables"), block_tables.shape[1], block_size,
        _dev(seq_lens, "seq_lens"), _dev(query_start_loc, "query_start_loc"),
        _dev(slot_mapping, "slot_mapping"), slot_mapping.numel(), _stream(stream))
    if rc != PA_OK:
        raise PAError(rc, "pa_plan_step")
