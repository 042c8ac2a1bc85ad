"""Benchmark: one paged-attention step (cache write of the new tokens + attention)
on the decode workload, TinyLlama-1.1B attention shape (32 q / 4 kv heads,
head_dim 64, 64 sequences of context U[128, 2048], 16-token blocks, 100k-block
pool), bf16, synthetic N(0,1) data.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints ONE JSON line (rank 0).  `value` is decode KV GB/s: the K/V bytes the
step's attention must read (sum over sequences of seq_len * 2 * Hkv * D * 2 B,
summed over ranks) divided by the device time of a step (max over ranks).
Steps run back to back, as in a serving loop, each one a single
pa_attention_varlen_write_cache call (cache write fused into the decode
kernel).  Every timed figure is one replay of one CUDA graph holding exactly
--steps back-to-back calls (each launch a programmatic dependent of the one
before), timed with CUDA events on the launching stream, so the number is the
GPU's time and does not depend on how fast the host issues calls.  No step
finds its inputs in L2: when one step reads less than twice the L2 size, the
steps rotate over that many identical copies of the workload (own pool, own
tensors) that consecutive reads of one copy are separated by more than twice
the L2 size of other traffic.

The line also carries the mixed prefill + decode step (query tokens/s, and its
prefill chunks alone against the bf16 peak), the prefix-cached decode step
(unique and logical KV GB/s), the long-context decode step, the on-GPU step
planner, and the end-to-end figure from pinned host buffers.
`--impl reference` times the CPU oracle on a bounded sample of the decode
workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode paged-attn KV GB/s (% of HBM peak); mixed-step query tokens/s"
WORKLOAD = "decode_tinyllama"
MIXED_WORKLOAD = "mixed_llama3_8b"
L2_BYTES = 126 * 1000 * 1000  # B200 L2, for sizing the rotation of workload copies
MAX_COPIES = 8
REFERENCE_BUDGET_S = 120.0  # host seconds the --impl reference steps may take in all
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of DECODE_KERNEL
# on this workload, from an ncu capture of that launch; None whenever that
# kernel has changed since it was last captured
DECODE_TRAFFIC_BYTES = 70_217_472  # ncu --set full, third launch of run_workload decode_tinyllama
DECODE_KERNEL = "decode_persistent_kernel<64,8,false,false>"
KERNELS_PER_DECODE_STEP = 1  # the decode step is one launch (cache write inside the kernel)


def kv_bytes(step, seqs=None) -> int:
    """Algorithmic K+V bytes one step's attention reads: every key of every
    sequence once per kv-head."""
    import numpy as np
    lens = step.seq_lens if seqs is None else step.seq_lens[seqs]
    elem = 4 if step.dtype == "f32" else 2
    return int(np.sum(lens.astype(np.int64))) * 2 * step.num_kv_heads * step.head_dim * elem


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled in the background; only
    samples taken inside the marked timed windows are reported."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 20):
        self.proc = None
        self.windows = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)  # let it start sampling
        except (OSError, ValueError):
            self.proc = None

    def window(self):
        """Context manager marking a timed region (host wall clock)."""
        sampler = self

        class _W:
            def __enter__(self_w):
                self_w.t0 = time.time()

            def __exit__(self_w, *exc):
                sampler.windows.append((self_w.t0, time.time()))
                return False
        return _W()

    def stop(self) -> dict:
        import datetime
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons, total = [], [], set(), 0
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            total += 1
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                mhz, mx = float(f[2]), float(f[3])
            except ValueError:
                continue
            if not any(a - 0.02 <= ts <= b + 0.02 for a, b in self.windows):
                continue
            sm.append(mhz)
            smax.append(mx)
            for n, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples_in_timed_regions": len(sm), "samples_total": total}


def _nullctx():
    import contextlib
    return contextlib.nullcontext()


def dist_setup(n_gpus: int):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank scalar over all ranks (identity on one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- CPU oracle legs

def oracle_sample(step, target_s: float, threads: int):
    """Time the oracle on the first n sequences (all their query rows), n grown
    until one pass takes about target_s seconds.  Returns (GB/s, n, seconds)."""
    import numpy as np
    import oracle
    from tests.oracle_side import oracle_state
    st = oracle_state(step)
    qsl = st["query_start_loc"]

    def run(n):
        tok = np.repeat(np.arange(int(qsl[n]), dtype=np.int64), step.num_q_heads)
        head = np.tile(np.arange(step.num_q_heads, dtype=np.int32), int(qsl[n]))
        t0 = time.perf_counter()
        oracle.paged_attention_rows(step.q, st["k_cache"], st["v_cache"], st["block_tables"],
                                    step.seq_lens, qsl, tok, head,
                                    num_q_heads=step.num_q_heads, scale=step.scale,
                                    num_threads=threads)
        return time.perf_counter() - t0

    n = 1
    dt = run(n)
    while dt < target_s and n < step.num_seqs:
        n = min(step.num_seqs, max(n + 1, int(n * target_s / max(dt, 1e-3))))
        dt = run(n)
    # a whole step shorter than the target: repeat it until the target is reached
    passes, total = 1, dt
    while total < target_s:
        total += run(n)
        passes += 1
    return kv_bytes(step, np.arange(n)) * passes / total / 1e9, n, total, run, passes


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def bench_reference(args) -> None:
    """The CPU oracle as the reference arm: each step is one pass over a bounded
    sample of the workload, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from paged_kv_cache_469_b200.inputs import workload
    step = workload(WORKLOAD)
    threads = os.cpu_count() or 1
    # each step a bounded sample: about 1 s, less when there are many steps, so
    # that the whole run stays near two minutes of host time
    per_step = min(1.0, REFERENCE_BUDGET_S / (args.steps + args.warmup))
    gbs, n, dt, run, _ = oracle_sample(step, target_s=per_step, threads=threads)
    import numpy as np
    for _ in range(args.warmup):
        run(n)
    times = [run(n) for _ in range(args.steps)]
    ms = 1e3 * sum(times) / len(times)
    value = kv_bytes(step, np.arange(n)) / (ms / 1e3) / 1e9
    sample = (f"first {n} of {step.num_seqs} sequences, all {step.num_q_heads} q-heads, "
              f"fp64 oracle, {threads} threads")
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "num_seqs": step.num_seqs,
                       "context": "U[128,2048]", "num_q_heads": 32, "num_kv_heads": 4,
                       "head_dim": 64, "block_size": 16, "num_blocks": step.num_blocks},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm

def step_bytes(step) -> int:
    """Bytes one step touches in HBM at least: the K/V it reads plus q and out."""
    elem = 4 if step.dtype == "f32" else 2
    return kv_bytes(step) + 2 * int(step.q.size) * elem


def unique_kv_bytes(step) -> int:
    """K+V bytes of the distinct cache tokens a step reads: a shared prefix counts once."""
    import numpy as np
    p = int(step.shared_prefix_tokens)
    lens = step.seq_lens.astype(np.int64)
    tokens = int(lens.sum()) - p * max(0, step.num_seqs - 1)
    elem = 4 if step.dtype == "f32" else 2
    return tokens * 2 * step.num_kv_heads * step.head_dim * elem


def copies_for(step) -> int:
    """Copies of the workload to rotate over so that no step finds its inputs in
    L2: enough that the other copies' traffic between two reads of one copy
    exceeds twice the L2 size."""
    b = max(1, step_bytes(step))
    return int(min(MAX_COPIES, max(1, -(-2 * L2_BYTES // b) + 1))) if b < 2 * L2_BYTES else 1


def _upload(g) -> None:
    """Upload an instantiated graph to the device before it is timed, so that
    the first timed replay does not include the upload."""
    import ctypes
    import torch
    try:
        cu = ctypes.CDLL("libcuda.so.1")
        cu.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        cu.cuGraphUpload.restype = ctypes.c_int
        rc = cu.cuGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        torch.cuda.synchronize()
        if rc != 0:
            raise RuntimeError(f"cuGraphUpload returned {rc}")
    except (OSError, AttributeError):
        pass


def capture_steps(calls, k: int):
    """One CUDA graph of k back-to-back calls, calls[i % len(calls)]() for i < k.
    Each call is made once outside the capture first (one-time set-up)."""
    import torch
    for c in calls:
        c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(k):
            calls[i % len(calls)]()
    _upload(g)
    return g


def time_graph(g, stream) -> float:
    """Device ms of one replay of g (CUDA events on the launching stream,
    synchronised on both sides)."""
    import torch
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def timed_steps(calls, args, stream, world, clocks) -> float:
    """Mean device ms per call: args.warmup untimed calls (one graph), then one
    replay of a graph of exactly args.steps back-to-back calls, timed; the max
    over ranks."""
    import torch
    warm = capture_steps(calls, args.warmup)
    warm.replay()
    g = capture_steps(calls, args.steps)
    torch.cuda.synchronize()
    barrier(world)
    with clocks.window() if clocks else _nullctx():
        ms = time_graph(g, stream)
    barrier(world)
    del g, warm
    return max_over_ranks(ms / args.steps, world)


def prefill_flops(step) -> int:
    """Flops of the unmasked (query, key) pairs of the prefill-class sequences
    (q_len * group > 64): 4 * D * Hq per pair (Q.K^T and P.V)."""
    g = step.num_q_heads // step.num_kv_heads
    pairs = 0
    for ql, L in zip(step.query_lens.tolist(), step.seq_lens.tolist()):
        if ql * g > 64:
            pairs += ql * (L - ql) + ql * (ql + 1) // 2
    return 4 * step.head_dim * step.num_q_heads * pairs


def _free(*objs):
    import torch
    del objs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def bench_mixed(args, dev, stream, world, clocks):
    """Mixed prefill + decode step (Llama-3-8B attention shape): query tokens/s,
    plus the prefill chunks alone against the bf16 tensor peak."""
    from paged_kv_cache_469_b200.inputs import prefill_part, workload
    from paged_kv_cache_469_b200.step import DeviceStep
    step = workload(MIXED_WORKLOAD)
    dss = [DeviceStep(step, device=str(dev)) for _ in range(copies_for(step))]
    copies = len(dss)
    step_ms = timed_steps([d.run_fused for d in dss], args, stream, world, clocks)
    tokens = sum_over_ranks(step.num_tokens, world)
    g = step.num_q_heads // step.num_kv_heads
    kv_dec = int(sum(L for L, q in zip(step.seq_lens.tolist(), step.query_lens.tolist())
                     if q * g <= 64)) * 2 * step.num_kv_heads * step.head_dim * 2
    _free(*dss)
    del dss
    # the same step's prefill chunks alone (same lengths, same shape)
    pre = prefill_part(step)
    dps = [DeviceStep(pre, device=str(dev)) for _ in range(copies_for(pre))]
    pre_ms = timed_steps([d.attention for d in dps], args, stream, world, clocks)
    flops = prefill_flops(pre)
    peaks = load_peaks()
    tflops = flops / (pre_ms / 1e3) / 1e12
    pre_copies = len(dps)
    _free(*dps)
    del dps
    return {"workload": MIXED_WORKLOAD, "value": round(tokens / (step_ms / 1e3), 1),
            "unit": "query tokens/s", "ms_per_step": round(step_ms, 4), "steps": args.steps,
            "query_tokens_per_step_per_gpu": step.num_tokens,
            "decode_kv_bytes_per_step_per_gpu": kv_dec, "copies_rotated": copies,
            "launch": "one CUDA graph of --steps back-to-back pa_attention_varlen_write_cache calls",
            "prefill_only": {"ms": round(pre_ms, 4), "gflop": round(flops / 1e9, 3),
                             "tflops": round(tflops, 1),
                             "frac_of_bf16_peak": round(tflops / peaks["bf16_tflops"], 4),
                             "frac_of_bf16_sustained": round(
                                 tflops / peaks["bf16_tflops_sustained"], 4),
                             "peak_source": peaks["source"], "copies_rotated": pre_copies,
                             "kernels": ("prefill_tcgen05_kernel<128> (work list from the "
                                         "host copies of the step's lengths)")}}


def bench_decode_workload(name, args, dev, stream, world, clocks):
    """A decode-class workload's step (cache write of the new tokens + attention,
    one pa_attention_varlen_write_cache call): KV GB/s against the HBM peak."""
    from paged_kv_cache_469_b200.inputs import workload
    from paged_kv_cache_469_b200.step import DeviceStep
    step = workload(name)
    dss = [DeviceStep(step, device=str(dev)) for _ in range(copies_for(step))]
    copies = len(dss)
    ms = timed_steps([d.run_fused for d in dss], args, stream, world, clocks)
    _free(*dss)
    del dss
    peaks = load_peaks()
    logical = sum_over_ranks(kv_bytes(step), world)
    unique = sum_over_ranks(unique_kv_bytes(step), world)
    gbs = unique / (ms / 1e3) / 1e9
    rec = {"workload": name, "unit": "GB/s", "ms_per_step": round(ms, 4), "steps": args.steps,
           "num_seqs": step.num_seqs, "context_tokens": int(step.seq_lens.sum()),
           "value": round(gbs, 1), "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4),
           "peak_source": f"{peaks['source']} HBM copy bandwidth",
           "kv_bytes_per_step_per_gpu": unique_kv_bytes(step), "copies_rotated": copies,
           "launch": "one CUDA graph of --steps back-to-back pa_attention_varlen_write_cache calls"}
    if step.shared_prefix_tokens:
        rec["bytes"] = ("unique: the shared prefix's blocks counted once (the roofline "
                        "figure); logical: every sequence's keys")
        rec["logical_kv_bytes_per_step_per_gpu"] = kv_bytes(step)
        rec["logical_gbs"] = round(logical / (ms / 1e3) / 1e9, 1)
    return rec


def bench_planner(args, dev, stream) -> dict:
    """The on-GPU step planner (pa_plan_step) on the decode workload's step:
    device time per call, against the host path it replaces (BlockPool,
    numpy slot mapping and prefix sum, pinned copies to the device)."""
    import numpy as np
    import torch
    from paged_kv_cache_469_b200 import block_pool, lib
    from paged_kv_cache_469_b200.inputs import workload
    step = workload(WORKLOAD, with_values=False)
    S = step.num_seqs
    ql = step.query_lens.astype(np.int32)
    nc = (step.seq_lens - step.query_lens).astype(np.int32)
    mb = max(1, -(-int(step.seq_lens.max()) // 16))

    def host_pool():
        pool = block_pool.BlockPool(step.free_queue)
        for s in range(S):
            pool.allocate_slots(s, int(nc[s]))
        return pool

    pool = host_pool()
    head0 = len(step.free_queue) - len(pool.free_block_queue)
    tables0 = pool.block_table(range(S), mb)
    for s in range(S):
        pool.allocate_slots(s, int(nc[s] + ql[s]))
    tables1 = pool.block_table(range(S), mb)
    slots1 = block_pool.slot_mapping(tables1, nc, ql)
    qsl1 = block_pool.query_start_loc(ql)
    per_call = len(step.free_queue) - len(pool.free_block_queue) - head0

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    fq, tables, nc_t, ql_t = (to_dev(step.free_queue), to_dev(tables0), to_dev(nc),
                              to_dev(ql))
    state = lib.new_planner_state(head0, device=dev)
    seq_lens = torch.empty(S, dtype=torch.int32, device=dev)
    qsl = torch.empty(S + 1, dtype=torch.int32, device=dev)
    slots = torch.empty(int(ql.sum()), dtype=torch.int64, device=dev)

    def call():
        lib.plan_step(fq, state, nc_t, ql_t, tables, seq_lens, qsl, slots)

    call()
    torch.cuda.synchronize(dev)
    # both product paths must agree before anything is timed
    if not (np.array_equal(tables.cpu().numpy(), tables1) and
            np.array_equal(slots.cpu().numpy(), slots1) and
            np.array_equal(qsl.cpu().numpy(), qsl1) and
            np.array_equal(seq_lens.cpu().numpy(), nc + ql) and
            state.cpu().tolist()[:3] == [head0 + per_call, 0, 0]):
        raise RuntimeError("pa_plan_step and the host planner disagree")
    # every call repeats the step (same counts, the next blocks of the queue);
    # the queue must hold the blocks of every call, warm-up included
    left = len(step.free_queue) - head0 - per_call
    n = int(max(1, min(args.steps, left // max(1, per_call) - 2 * args.warmup - 2)))
    warm = capture_steps([call], args.warmup)
    warm.replay()
    g = capture_steps([call], n)
    dev_us = time_graph(g, stream) * 1e3 / n
    if state[1].item() != 0:
        raise RuntimeError("pa_plan_step refused a timed call")
    del g, warm

    def pinned_like(a):
        return torch.from_numpy(np.empty_like(a)).pin_memory()

    h_tab, h_slots, h_qsl, h_sl = (pinned_like(tables1), pinned_like(slots1), pinned_like(qsl1),
                                   pinned_like(nc))
    host_us = []
    for _ in range(20):
        pool = host_pool()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for s in range(S):
            pool.allocate_slots(s, int(nc[s] + ql[s]))
        tab = pool.block_table(range(S), mb)
        sm = block_pool.slot_mapping(tab, nc, ql)
        qs = block_pool.query_start_loc(ql)
        h_tab.numpy()[...] = tab
        h_slots.numpy()[...] = sm
        h_qsl.numpy()[...] = qs
        h_sl.numpy()[...] = nc + ql
        tables.copy_(h_tab, non_blocking=True)
        slots.copy_(h_slots, non_blocking=True)
        qsl.copy_(h_qsl, non_blocking=True)
        seq_lens.copy_(h_sl, non_blocking=True)
        stream.synchronize()
        host_us.append((time.perf_counter() - t0) * 1e6)
    return {"workload": WORKLOAD, "num_seqs": S, "new_tokens": int(ql.sum()),
            "blocks_taken_per_call": per_call,
            "device_us_per_call": round(dev_us, 3), "calls": n,
            "device_timing": "one CUDA graph of back-to-back pa_plan_step calls, CUDA events",
            "host_us_per_step": round(statistics.median(host_us), 1),
            "host_path": ("BlockPool.allocate_slots per sequence, block_table, slot_mapping, "
                          "query_start_loc, four pinned copies to the device, stream sync "
                          "(median of 20)"),
            "equal_outputs": True}


def bench_device_loop(args, dev, stream, world, clocks) -> dict:
    """The serving loop planned on the GPU: every step is pa_plan_step (one
    token more per sequence) and pa_attention_varlen_write_cache without host
    copies (its decode work listed on the device), for the decode workload's 64
    sequences, starting from its contexts.  The lengths alternate between two
    buffers: a step's new lengths are the next step's num_computed (the two
    never alias, as pa_plan_step requires).  --steps such steps are captured as one CUDA graph, rotating
    over the same copies of the workload as the main leg, and timed as one
    replay.  Query tokens/s (one per sequence and step), and KV GB/s on the
    keys the steps actually read (the sequences grow by one token per step)."""
    import numpy as np
    import torch
    from paged_kv_cache_469_b200 import lib
    from paged_kv_cache_469_b200.inputs import workload
    from paged_kv_cache_469_b200.step import DeviceStep
    step = workload(WORKLOAD)
    n = copies_for(step)
    per_copy = -(-(args.steps + args.warmup) // n) + 4  # steps each copy takes at most
    bound = int(step.seq_lens.max()) + per_copy
    loops = []
    for _ in range(n):
        d = DeviceStep(step, device=str(dev), max_blocks_per_seq=-(-bound // 16))
        S = step.num_seqs
        st = {"d": d,
              "fq": torch.from_numpy(step.free_queue).to(dev),
              "state": lib.new_planner_state(d.plan.blocks_taken, device=dev),
              "lens": [d.seq_lens.clone(), torch.empty(S, dtype=torch.int32, device=dev)],
              "flip": 0,  # lens[flip] holds the lengths computed so far
              "query_lens": torch.ones(S, dtype=torch.int32, device=dev),
              "qsl": torch.empty(S + 1, dtype=torch.int32, device=dev),
              "slots": torch.empty(S, dtype=torch.int64, device=dev),
              "ws": lib.new_workspace(S, step.num_q_heads, step.num_kv_heads, step.head_dim,
                                      bound, device=dev)}
        loops.append(st)

    def call_for(st):
        d = st["d"]

        def call():
            # (the buffers alternate call by call in the order the calls run:
            # eagerly, or as recorded in a graph that is replayed once)
            done, new = st["lens"][st["flip"]], st["lens"][1 - st["flip"]]
            lib.plan_step(st["fq"], st["state"], done, st["query_lens"], d.block_tables, new,
                          st["qsl"], st["slots"])
            lib.attention_varlen_write_cache(
                d.out, d.q, d.k_new, d.v_new, d.k_cache, d.v_cache, st["slots"], d.block_tables,
                new, st["qsl"], max_query_len=1, max_seq_len=bound, scale=step.scale,
                workspace=st["ws"])
            st["flip"] ^= 1
        return call

    calls = [call_for(st) for st in loops]
    # every call (the set-up call of capture_steps and the warm-up included)
    # advances its copy by one token per sequence
    ms = timed_steps(calls, args, stream, world, clocks)
    if any(int(st["state"][1].item()) != 0 for st in loops):
        raise RuntimeError("pa_plan_step refused a step of the device-planned loop")
    # keys read by the timed steps: copy c's k-th step reads the contexts + k + 1
    lens0 = step.seq_lens.astype(np.int64)
    done = [0] * n
    for c in range(n):  # set-up calls: one per copy per captured graph, plus the warm-up
        done[c] = 2
    for i in range(args.warmup):
        done[i % n] += 1
    keys = 0
    for i in range(args.steps):
        c = i % n
        keys += int((lens0 + done[c] + 1).sum())
        done[c] += 1
    kv = keys * 2 * step.num_kv_heads * step.head_dim * 2
    tokens = sum_over_ranks(step.num_seqs, world)
    del loops, calls
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return {"workload": WORKLOAD, "num_seqs": step.num_seqs, "steps": args.steps,
            "copies_rotated": n, "ms_per_step": round(ms, 5),
            "value": round(tokens / (ms / 1e3), 1), "unit": "query tokens/s",
            "kv_gbs": round(sum_over_ranks(kv, world) / args.steps / (ms / 1e3) / 1e9, 1),
            "launch": ("one CUDA graph of --steps steps, each pa_plan_step + "
                       "pa_attention_varlen_write_cache (no host copies), the lengths in two "
                       "alternating buffers; no host work between steps")}


def capture_e2e(dss, host_ins, host_out, k: int):
    """One CUDA graph of k steps end to end: step i copies its packed inputs in
    from pinned host memory (copy stream), runs pa_attention_varlen_write_cache
    (launching stream) and copies its output back (second copy stream).  At
    most two steps are in flight: step i's input copy waits for step i-2's
    kernel, and step i's kernel for step i-2's output copy, so that step i+1's
    copy in and step i-1's copy out overlap step i's kernel while no buffer is
    overwritten before it has been read."""
    import torch
    c = len(dss)
    depth = min(2, c)
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    for d, h in zip(dss, host_ins):  # one eager step per copy (one-time set-up)
        d.inputs.copy_(h, non_blocking=True)
        d.run_fused()
        host_out.copy_(d.out.view(torch.int16), non_blocking=True)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cap = torch.cuda.current_stream()
        start = torch.cuda.Event()
        start.record(cap)
        k_done, o_done = [], []
        for i in range(k):
            d = dss[i % c]
            cin.wait_event(k_done[i - depth] if i >= depth else start)
            with torch.cuda.stream(cin):
                d.inputs.copy_(host_ins[i % c], non_blocking=True)
            e_in = torch.cuda.Event()
            e_in.record(cin)
            cap.wait_event(e_in)
            if i >= depth:
                cap.wait_event(o_done[i - depth])
            d.run_fused()
            e_k = torch.cuda.Event()
            e_k.record(cap)
            k_done.append(e_k)
            cout.wait_event(e_k)
            with torch.cuda.stream(cout):
                host_out.copy_(d.out.view(torch.int16), non_blocking=True)
            e_o = torch.cuda.Event()
            e_o.record(cout)
            o_done.append(e_o)
        cap.wait_stream(cin)
        cap.wait_stream(cout)
    _upload(g)
    return g


def bench_ours(args) -> None:
    import torch

    from paged_kv_cache_469_b200 import lib
    from paged_kv_cache_469_b200.inputs import workload
    from paged_kv_cache_469_b200.step import DeviceStep

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    lib.library()
    step = workload(WORKLOAD)
    stream = torch.cuda.current_stream(dev)
    dss = [DeviceStep(step, device=str(dev)) for _ in range(copies_for(step))]
    copies = len(dss)
    clocks = ClockSampler(local) if rank == 0 or world > 1 else None

    # ---- device-resident steps: one CUDA graph of --steps back-to-back
    # pa_attention_varlen_write_cache calls over the rotating copies, timed
    # as one replay (each launch a programmatic dependent of the previous one)
    step_ms = timed_steps([d.run_fused for d in dss], args, stream, world, clocks)
    # the attention call alone (the roofline's kernel), the same way
    attn_ms = timed_steps([d.attention for d in dss], args, stream, world, clocks)
    bytes_rank = kv_bytes(step)
    bytes_all = sum_over_ranks(bytes_rank, world)
    value = bytes_all / (step_ms / 1e3) / 1e9

    # ---- end to end through the public API from pinned host buffers: every step
    # copies its inputs in (one copy: the step's inputs are packed into one
    # buffer on both sides), runs, and copies its output back
    host_ins = [d.host_inputs() for d in dss]
    host_out = torch.empty(dss[0].out.shape, dtype=torch.int16).pin_memory()
    h2d = host_ins[0].numel()
    d2h = host_out.numel() * host_out.element_size()
    warm = capture_e2e(dss, host_ins, host_out, args.warmup)
    warm.replay()
    g = capture_e2e(dss, host_ins, host_out, args.steps)
    barrier(world)
    with clocks.window() if clocks else _nullctx():
        e2e_ms = time_graph(g, stream) / args.steps
    barrier(world)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_value = bytes_all / (e2e_ms / 1e3) / 1e9
    del g, warm, host_ins
    _free(*dss)
    del dss
    mixed = None if args.no_mixed else bench_mixed(args, dev, stream, world, clocks)
    prefix = (None if args.no_decode_configs else
              bench_decode_workload("prefix_decode_llama3_8b", args, dev, stream, world, clocks))
    long_ = (None if args.no_decode_configs else
             bench_decode_workload("long_decode_llama3_8b", args, dev, stream, world, clocks))
    planner = None if args.no_planner or rank != 0 else bench_planner(args, dev, stream)
    device_loop = (None if args.no_planner else
                   bench_device_loop(args, dev, stream, world, clocks))
    clk = clocks.stop() if clocks else None

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    peaks = load_peaks()
    achieved = bytes_rank / (attn_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": DECODE_TRAFFIC_BYTES,
                "traffic_unit": "dram bytes read + written per launch (ncu)",
                "kernel": DECODE_KERNEL + " (attention call without the fused cache write)",
                "timing": ("one CUDA graph of --steps back-to-back attention calls over the "
                           "rotating copies, CUDA events around one replay"),
                "peak_source": f"{peaks['source']} HBM copy bandwidth (burst)",
                "frac_of_nominal_8TBs": round(achieved / 8000.0, 4)}
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        gbs, n, dt, _, passes = oracle_sample(step, target_s=10.0, threads=threads)
        gbs1, n1, dt1, _, passes1 = oracle_sample(step, target_s=4.0, threads=1)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"first {n} of {step.num_seqs} sequences (all q-heads), {passes} "
                         f"passes, {dt:.1f} s",
               "single_thread": {"value": round(gbs1, 4), "unit": "GB/s",
                                 "sample": f"first {n1} sequences, {passes1} passes, "
                                           f"{dt1:.1f} s"},
               "cpu_model": cpu_model()}
    launches = args.steps * KERNELS_PER_DECODE_STEP
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "num_seqs": step.num_seqs,
                       "context": "U[128,2048]", "num_q_heads": 32, "num_kv_heads": 4,
                       "head_dim": 64, "block_size": 16, "num_blocks": step.num_blocks,
                       "kv_bytes_per_step_per_gpu": bytes_rank,
                       "l2": f"not flushed: inputs larger than L2 (steps rotate over {copies} "
                             f"copies of the workload, {copies * step_bytes(step) / 1e6:.0f} MB "
                             f"touched per rotation)",
                       "parallelism": f"{world} independent replicas"},
            "attention_ms": round(attn_ms, 5),
            "launch": ("one CUDA graph of --steps back-to-back pa_attention_varlen_write_cache "
                       "calls (cache write fused into the decode kernel; each launch a "
                       "programmatic dependent of the previous step's), timed as one replay"),
            "gpu_launches": launches,
            "mixed_step": mixed,
            "prefix_decode": prefix,
            "long_decode": long_,
            "plan_step": planner,
            "device_planned_loop": device_loop,
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "ms_per_step": round(e2e_ms, 5),
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "overlap": ("copy in, kernel and copy out on three streams, at most two "
                                "steps in flight")},
            "roofline": roofline, "cpu_baseline": cpu, "clocks": clk}
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main(argv=None) -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-mixed", action="store_true",
                    help="skip the mixed prefill+decode leg (Llama-3-8B shape)")
    ap.add_argument("--no-planner", action="store_true",
                    help="skip the on-GPU step planner measurement")
    ap.add_argument("--no-decode-configs", action="store_true",
                    help="skip the prefix-cached and long-context decode legs")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_ours(args)


if __name__ == "__main__":
    main()
