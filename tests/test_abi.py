"""The C-ABI library loads without a GPU, exports every symbol include/pa.h
declares, and its host-side argument checks reject bad calls before any launch."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from paged_kv_cache_469_b200 import lib as palib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(pa_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    from paged_kv_cache_469_b200.build import build
    build()
    return palib.library()


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert len(names) >= 5
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert set(names) == set(palib.EXPORTS)


def test_status_strings(L):
    for code in (0, -1, -2, -3):
        assert L.pa_status_string(code).startswith(b"PA_")


def test_workspace_size_host_only(L):
    n = L.pa_attention_workspace_size(64, 32, 4, 64, 2048)
    assert n > 0 and n % 256 == 0
    assert L.pa_attention_workspace_size(64, 32, 5, 64, 2048) == 0  # 32 % 5 != 0
    assert L.pa_attention_workspace_size(64, 32, 4, 96, 2048) == 0  # head_dim 96
    assert L.pa_attention_workspace_size(0, 32, 4, 64, 0) > 0


def _varlen(L, **kw):
    args = dict(out=16, q=16, kc=16, vc=16, bt=16, mb=8, sl=16, qsl=16, S=1, T=1, mq=1, ms=16,
                hq=8, hkv=2, d=64, bs=16, nb=4, scale=0.125, dt=1, ws=0, wsb=0, slh=None,
                qslh=None, stream=None)
    args.update(kw)
    return L.pa_attention_varlen(*args.values())


def test_attention_argument_checks(L):
    assert _varlen(L, d=96) == palib.PA_ERR_UNSUPPORTED
    assert _varlen(L, bs=32) == palib.PA_ERR_UNSUPPORTED
    assert _varlen(L, dt=7) == palib.PA_ERR_UNSUPPORTED
    assert _varlen(L, hkv=3) == palib.PA_ERR_INVALID
    assert _varlen(L, hq=64, hkv=2) == palib.PA_ERR_UNSUPPORTED  # 32 q-heads per kv-head
    assert _varlen(L, scale=0.0) == palib.PA_ERR_INVALID
    assert _varlen(L, scale=float("nan")) == palib.PA_ERR_INVALID
    assert _varlen(L, mq=20, ms=16) == palib.PA_ERR_INVALID
    assert _varlen(L, mb=0) == palib.PA_ERR_INVALID  # table narrower than max_seq_len
    assert _varlen(L, q=8) == palib.PA_ERR_INVALID  # misaligned pointer
    assert _varlen(L, out=0) == palib.PA_ERR_INVALID
    assert _varlen(L, S=-1) == palib.PA_ERR_INVALID
    assert _varlen(L, T=0) == palib.PA_OK  # nothing to do, nothing launched
    # any number of sequences: a large call is refused only for its missing
    # workspace (the persistent decode grid does not depend on the count)
    assert _varlen(L, S=65536, T=65536) == palib.PA_ERR_INVALID
    # a bound past the split-K partial slots one (sequence, kv-head) may hold
    # (8 + ceil(blocks / 256) > 1536)
    big = 391_169 * 16
    assert _varlen(L, ms=big, mb=big // 16) == palib.PA_ERR_UNSUPPORTED
    assert _varlen(L, ms=big - 16, mb=big // 16) == palib.PA_ERR_INVALID  # fits, no workspace
    # host copies that contradict the scalars are rejected
    import numpy as np
    sl = np.array([4], np.int32)
    bad_qsl = np.array([0, 5], np.int32)  # q_len 5 > seq_len 4
    assert _varlen(L, T=5, mq=5, slh=sl.ctypes.data, qslh=bad_qsl.ctypes.data) == \
        palib.PA_ERR_INVALID
    # decode work needs a big enough workspace
    ok_qsl = np.array([0, 1], np.int32)
    assert _varlen(L, slh=sl.ctypes.data, qslh=ok_qsl.ctypes.data, ws=0, wsb=0) == \
        palib.PA_ERR_INVALID


def _varlen_wc(L, **kw):
    args = dict(out=16, q=16, kn=16, vn=16, kc=16, vc=16, slots=16, bt=16, mb=8, sl=16, qsl=16,
                S=1, T=1, mq=1, ms=16, hq=8, hkv=2, d=64, bs=16, nb=4, scale=0.125, dt=1, ws=0,
                wsb=0, slh=None, qslh=None, stream=None)
    args.update(kw)
    return L.pa_attention_varlen_write_cache(*args.values())


def test_write_cache_call_argument_checks(L):
    """pa_attention_varlen_write_cache checks what pa_attention_varlen checks,
    plus its new-row arguments, on the host, before any launch (and so before
    any cache write)."""
    assert _varlen_wc(L, d=96) == palib.PA_ERR_UNSUPPORTED
    assert _varlen_wc(L, hkv=3) == palib.PA_ERR_INVALID
    assert _varlen_wc(L, slots=0) == palib.PA_ERR_INVALID   # no slot mapping
    assert _varlen_wc(L, kn=0) == palib.PA_ERR_INVALID      # no new K rows
    assert _varlen_wc(L, vn=8) == palib.PA_ERR_INVALID      # misaligned new V rows
    assert _varlen_wc(L, q=8) == palib.PA_ERR_INVALID
    assert _varlen_wc(L, T=0) == palib.PA_OK                # nothing to do
    import numpy as np
    sl = np.array([4], np.int32)
    ok_qsl = np.array([0, 1], np.int32)
    # a decode step without a big enough workspace fails before the cache write
    assert _varlen_wc(L, slh=sl.ctypes.data, qslh=ok_qsl.ctypes.data, ws=0, wsb=0) == \
        palib.PA_ERR_INVALID


def test_reshape_argument_checks(L):
    f = L.pa_reshape_and_cache
    assert f(16, 16, 16, 16, 16, 4, 2, 96, 16, 8, 1, None) == palib.PA_ERR_UNSUPPORTED
    assert f(16, 16, 16, 16, 16, 4, 2, 64, 8, 8, 1, None) == palib.PA_ERR_UNSUPPORTED
    assert f(16, 16, 16, 16, 16, -1, 2, 64, 16, 8, 1, None) == palib.PA_ERR_INVALID
    assert f(16, 16, 16, 24, 16, 4, 2, 64, 16, 8, 1, None) == palib.PA_ERR_INVALID
    assert f(0, 16, 16, 16, 16, 4, 2, 64, 16, 8, 1, None) == palib.PA_ERR_INVALID
    assert f(0, 0, 0, 0, 0, 0, 2, 64, 16, 8, 1, None) == palib.PA_OK


def _plan(L, **kw):
    args = dict(fq=16, qlen=64, state=16, nc=16, ql=16, S=2, bt=16, mb=8, bs=16, sl=16,
                qsl=16, slots=16, cap=8, stream=None)
    args.update(kw)
    return L.pa_plan_step(*args.values())


def test_plan_step_argument_checks(L):
    """pa_plan_step rejects bad sizes, pointers and alignments on the host."""
    assert _plan(L, bs=32) == palib.PA_ERR_UNSUPPORTED
    assert _plan(L, S=16385) == palib.PA_ERR_UNSUPPORTED  # more sequences than one call plans
    assert _plan(L, S=-1) == palib.PA_ERR_INVALID
    assert _plan(L, qlen=-1) == palib.PA_ERR_INVALID
    assert _plan(L, mb=-1) == palib.PA_ERR_INVALID
    assert _plan(L, cap=-1) == palib.PA_ERR_INVALID
    assert _plan(L, state=0) == palib.PA_ERR_INVALID
    assert _plan(L, state=8) == palib.PA_ERR_INVALID     # state not 16-byte aligned
    assert _plan(L, qsl=0) == palib.PA_ERR_INVALID
    assert _plan(L, nc=0) == palib.PA_ERR_INVALID
    assert _plan(L, bt=0) == palib.PA_ERR_INVALID
    assert _plan(L, fq=0) == palib.PA_ERR_INVALID        # a queue of 64 entries at NULL
    assert _plan(L, slots=0) == palib.PA_ERR_INVALID     # room for 8 slots at NULL
    assert _plan(L, slots=20) == palib.PA_ERR_INVALID    # int64 slots misaligned
    assert _plan(L, ql=18) == palib.PA_ERR_INVALID       # int32 array misaligned


def test_plan_step_rejects_outputs_aliasing_inputs(L):
    """num_computed and query_lens are read in full by every CTA while other
    CTAs write seq_lens, query_start_loc and the slots: a call whose outputs
    share memory with those inputs is refused on the host."""
    base = 1 << 20
    ok = dict(nc=base, ql=base + 64, sl=base + 128, qsl=base + 192, slots=base + 256)
    # the same pointers, but pa_plan_step never runs: a bad block size is
    # reported first, so an otherwise valid set of separate buffers passes the
    # alias check and fails only on the block size
    assert _plan(L, bs=32, **ok) == palib.PA_ERR_UNSUPPORTED
    assert _plan(L, **dict(ok, sl=ok["nc"])) == palib.PA_ERR_INVALID   # seq_lens = num_computed
    assert _plan(L, **dict(ok, sl=ok["ql"] + 4)) == palib.PA_ERR_INVALID  # partly overlapping
    assert _plan(L, **dict(ok, qsl=ok["nc"])) == palib.PA_ERR_INVALID
    assert _plan(L, **dict(ok, slots=ok["ql"] - 8)) == palib.PA_ERR_INVALID


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(palib, "_lib", None)
    monkeypatch.setattr(palib, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="missing"):
        palib.library()
