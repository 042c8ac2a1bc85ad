"""Compile the CPU oracle (plain C, fp64) into ``oracle/_build/liboracle.so``.

Test infrastructure: building the checker is not using it; ``__graft_entry__``
calls :func:`build_oracle` so that the test suite finds it ready.
"""
from __future__ import annotations

import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "_build", "liboracle.so")


def build_oracle(force: bool = False) -> str:
    out = library_path()
    src = os.path.join(_HERE, "pa_oracle.c")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    # -ffp-contract=off: every product and sum is rounded on its own, in the
    # order the C source states (no fused multiply-add).
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(force=True))
