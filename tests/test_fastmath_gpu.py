"""The prefill softmax's polynomial exp2 (``exp2_poly2`` in
``csrc/pa_fastmath.cuh``) against CUDA's exp2, on the GPU.

The polynomial's stated bound: relative error at most 7.5e-5 from the fit plus
a few fp32 roundings, for inputs in [-125, 8]; in [-126, -125) a result whose
polynomial factor is just below 1 takes a subnormal encoding (relative error up
to 1.5e-4); below -126 (and -inf, a masked score) it returns a value in
[0, 2^-126 * 1.5] instead of the exact result.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

torch = pytest.importorskip("torch")

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "kernels", "exp2_poly_probe.cu")
OUT = os.path.join(HERE, "_build", "libexp2_poly_probe.so")


def _probe_lib():
    from paged_kv_cache_469_b200.build import ARCH, CSRC, NVCC
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    if not os.path.exists(OUT) or os.path.getmtime(OUT) < max(
            os.path.getmtime(SRC), os.path.getmtime(os.path.join(CSRC, "pa_fastmath.cuh"))):
        tmp = OUT + f".tmp{os.getpid()}"
        subprocess.run([NVCC, *ARCH, "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
                        "-I", CSRC, SRC, "-o", tmp, "-lcudart"], check=True,
                       capture_output=True)
        os.replace(tmp, OUT)
    lib = ctypes.CDLL(OUT)
    lib.exp2_poly_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_long]
    lib.exp2_poly_probe.restype = ctypes.c_int
    return lib


def _run(x: np.ndarray) -> np.ndarray:
    lib = _probe_lib()
    assert x.size % 2 == 0
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    yd = torch.empty_like(xd)
    assert lib.exp2_poly_probe(xd.data_ptr(), yd.data_ptr(), x.size // 2) == 0
    torch.cuda.synchronize()
    return yd.cpu().numpy()


@pytest.mark.gpu
def test_exp2_poly_relative_error_in_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-126.0, 8.0, 1 << 21, dtype=np.float32),
        rng.uniform(-126.0, 8.0, 1 << 20).astype(np.float32),
        # both sides of every rounding boundary n + 1/2 and of every integer
        (np.arange(-126, 8, dtype=np.float32)[:, None]
         + np.array([-0.5, -0.4999999, 0.0, 1e-7, 0.4999999, 0.5], np.float32)).ravel(),
    ]).astype(np.float32)
    x = x[(x >= -125.0) & (x <= 8.0)]
    x = x[: x.size - (x.size % 2)]
    y = _run(x).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    # CUDA's own exp2 on the same inputs, for reference
    cuda_exp2 = torch.exp2(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    rel = np.abs(y / exact - 1.0)
    rel_cuda = np.abs(cuda_exp2 / exact - 1.0)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert rel.max() <= 8.0e-5, rel.max()
    # far below the bf16 half-ulp (2^-9) that P is rounded to afterwards
    assert rel.max() < 2.0 ** -9 / 20
    assert rel_cuda.max() < 1e-5  # sanity of the comparison itself


@pytest.mark.gpu
def test_exp2_poly_floor_and_masked_inputs():
    x = np.array([-np.inf, -1e30, -1000.0, -200.0, -127.0, -126.5, -126.0, 0.0,
                  0.5, -0.5, 1.0, 8.0], np.float32)
    y = _run(x).astype(np.float64)
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
    low = x <= -126.0
    assert np.all(y[low] <= 1.5 * 2.0 ** -126)
    hi = ~low
    assert np.allclose(y[hi], np.exp2(x[hi].astype(np.float64)), rtol=8e-5, atol=0)
    assert y[7] == pytest.approx(1.0, rel=8e-5)
    # just above the clamp: subnormal encodings, still within 1.5e-4
    x = np.linspace(-126.0, -125.0, 1 << 16, dtype=np.float32)
    y = _run(x).astype(np.float64)
    assert np.all(np.abs(y / np.exp2(x.astype(np.float64)) - 1.0) <= 1.5e-4)
