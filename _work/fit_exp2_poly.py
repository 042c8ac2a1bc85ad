"""Fit the degree-3 polynomial for 2^f on [-1/2, 1/2] used by the prefill
softmax (``csrc/pa_fastmath.cuh``, ``exp2_poly2``).

Remez exchange on the relative error: solve for coefficients c and error E
with p(x_i) - 2^x_i = (-1)^i E 2^x_i at deg + 2 reference points, move the
references to the extrema of the error, repeat.  Prints the fp32
coefficients, their bit patterns and the largest relative error of the
polynomial evaluated in fp32 (Horner with fused multiply-adds).

    python -m paged_kv_cache_469_b200.fit_exp2_poly
"""
from __future__ import annotations

import struct

import numpy as np


def remez_exp2(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    n = deg + 2
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        a = np.zeros((n, n))
        for i in range(n):
            a[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            a[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        coef = np.linalg.solve(a, 2.0 ** x)[:deg + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # one extremum per run of equal sign
        sign = np.sign(err)
        ext = [0]
        for k in range(1, len(grid)):
            if sign[k] != sign[ext[-1]]:
                ext.append(k)
            elif abs(err[k]) > abs(err[ext[-1]]):
                ext[-1] = k
        if len(ext) > n:
            ext = sorted(sorted(ext, key=lambda k: -abs(err[k]))[:n])
        if len(ext) == n:
            x = grid[ext]
    return coef


def fp32_relative_error(coef32: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        p = (p.astype(np.float64) * f + np.float64(c)).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0).max())


def main() -> None:
    coef = remez_exp2(3).astype(np.float32)
    for i, c in enumerate(coef):
        bits = struct.unpack("<I", struct.pack("<f", c))[0]
        print(f"c{i} = {float(c):.8f}  0x{bits:08X}")
    print(f"max relative error (fp32 Horner): {fp32_relative_error(coef):.3e}")


if __name__ == "__main__":
    main()
