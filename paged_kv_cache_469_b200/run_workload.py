"""Run a named workload's step a few times through the C ABI (for profilers).

    python -m paged_kv_cache_469_b200.run_workload decode_tinyllama --steps 5
    python -m paged_kv_cache_469_b200.run_workload mixed_llama3_8b --prefill-only

Each step is the cache write of the new tokens followed by the attention
call, as in ``DeviceStep.run``.  The process exits 0 once the device has
finished every step, and raises if a launch fails or the workspace status
word reports an error.  No timing is printed: run it under a profiler.
"""
from __future__ import annotations

import argparse

import torch

from . import lib
from .inputs import WORKLOADS, prefill_part, workload
from .step import DeviceStep


def main(argv=None) -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("workload", choices=WORKLOADS)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--prefill-only", action="store_true",
                    help="keep only the prefill-class sequences (same lengths and shape)")
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("a CUDA device is required")
    lib.library()
    step = workload(args.workload)
    if args.prefill_only:
        step = prefill_part(step)
    ds = DeviceStep(step, device="cuda:0")
    for _ in range(args.steps):
        ds.run()
    torch.cuda.synchronize()
    status = lib.workspace_status(ds.workspace)
    if status != lib.PA_OK:
        raise SystemExit(f"workspace status {status} after {args.steps} steps")
    print(f"{step.name}: {args.steps} steps, {step.num_seqs} sequences, "
          f"{step.num_tokens} query tokens")


if __name__ == "__main__":
    main()
