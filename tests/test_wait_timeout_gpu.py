"""The kernels' time-bounded waits, made to run out on purpose.

Every wait of the prefill and decode kernels on another warp of their CTA (an
mbarrier phase, a shared-memory flag) gives up after a time limit, records
the timeout in the workspace status word and raises the CTA's abort flag, so
that the other waiting roles give up too and the kernel returns instead of
hanging.  No input of the library reaches that path, so this test drives the
same wait functions (``csrc/pa_wait.cuh``) from a probe kernel, with a 1 ms
limit, on a barrier and a flag that nothing completes, and checks what they
return, the status bit, the abort flag, and that the GPU context is still
usable afterwards.  Every wait in the probe is bounded (1 ms, or 200 ms for
the role that must give up early), so nothing can hang.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

torch = pytest.importorskip("torch")

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kernels", "wait_timeout_probe.cu")
OUT = os.path.join(HERE, "_build", "libwait_timeout_probe.so")

LIMIT_NS = 1_000_000      # the wait that must run out
OTHER_NS = 200_000_000    # the wait that must give up on the abort flag well before this
STATUS_WAIT_TIMEOUT = 1   # kStatusWaitTimeout


def _probe():
    from paged_kv_cache_469_b200.build import ARCH, CSRC, INCLUDE, NVCC
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    deps = [SRC, os.path.join(CSRC, "pa_wait.cuh"), os.path.join(CSRC, "pa_internal.cuh")]
    if not os.path.exists(OUT) or os.path.getmtime(OUT) < max(map(os.path.getmtime, deps)):
        tmp = OUT + f".tmp{os.getpid()}"
        subprocess.run([NVCC, *ARCH, "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
                        "-I", CSRC, "-I", INCLUDE, SRC, "-o", tmp, "-lcudart"], check=True,
                       capture_output=True)
        os.replace(tmp, OUT)
    lib = ctypes.CDLL(OUT)
    lib.wait_timeout_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_ulonglong,
                                       ctypes.c_ulonglong, ctypes.c_int]
    lib.wait_timeout_probe.restype = ctypes.c_int
    return lib


def _run(mode):
    lib = _probe()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    result = torch.full((5,), -1, dtype=torch.int32, device="cuda")
    assert lib.wait_timeout_probe(status.data_ptr(), result.data_ptr(), LIMIT_NS, OTHER_NS,
                                  mode) == 0
    torch.cuda.synchronize()
    return int(status.item()), result.cpu().numpy()


def test_probe_builds():
    """The probe compiles against the library's wait header (no GPU needed)."""
    _probe()


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [0, 1])
def test_a_wait_that_runs_out_winds_the_cta_down(mode):
    status, res = _run(mode)
    barrier_ok, flag_ok, aborted, us0, us1 = res.tolist()
    assert status & STATUS_WAIT_TIMEOUT, "the timeout was not recorded"
    assert aborted == 1, "the abort flag was not raised"
    assert barrier_ok == 0 and flag_ok == 0, "a wait claimed success on nothing"
    timed_out, gave_up = (us0, us1) if mode == 0 else (us1, us0)
    assert timed_out >= LIMIT_NS // 1000, "the wait gave up before its limit"
    # the other role left on the abort flag, long before its own limit
    assert gave_up < OTHER_NS // 1000 // 4
    # the context is still usable: a kernel and a copy afterwards
    x = torch.arange(1 << 20, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == float(np.arange(1 << 20, dtype=np.float64).sum())


@pytest.mark.gpu
def test_waits_that_complete_report_nothing():
    status, res = _run(2)
    barrier_ok, flag_ok, aborted, _, _ = res.tolist()
    assert (status, barrier_ok, flag_ok, aborted) == (0, 1, 1, 0)
