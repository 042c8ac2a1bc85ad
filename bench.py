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
kernel): timed both as one CUDA graph replay per step and as plain calls
(each launch a programmatic dependent of the previous one); `value` uses the
faster and `launch` says which.  No step finds its inputs in L2:
when one step reads less than twice the L2 size, the timed loop rotates over
that many identical copies of the workload (own pool, own tensors) that
consecutive reads of one copy are separated by more than twice the L2 size of
other traffic.  `--impl reference` times the CPU oracle on a bounded sample of
the same workload instead.
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
# dram__bytes_read.sum + dram__bytes_write.sum of one decode_splitk_kernel<64,false,4,4,false>
# launch on this workload, from an ncu --set full capture of that launch; set
# to None whenever that kernel changes, until it is captured again
DECODE_TRAFFIC_BYTES = 68_948_736 + 1_102_080


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


def copies_for(step) -> int:
    """Copies of the workload to rotate over so that no step finds its inputs in
    L2: enough that the other copies' traffic between two reads of one copy
    exceeds twice the L2 size."""
    b = max(1, step_bytes(step))
    return int(min(MAX_COPIES, max(1, -(-2 * L2_BYTES // b) + 1))) if b < 2 * L2_BYTES else 1


def timed_loop(fns, stream, steps: int) -> float:
    """Mean device ms per call over `steps` back-to-back calls of fns[i % len(fns)]
    (CUDA events on the launching stream around the whole loop)."""
    import torch
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        fns[i % len(fns)]()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def prefill_flops(step) -> int:
    """Flops of the unmasked (query, key) pairs of the prefill-class sequences
    (q_len * group > 64): 4 * D * Hq per pair (Q.K^T and P.V)."""
    g = step.num_q_heads // step.num_kv_heads
    pairs = 0
    for ql, L in zip(step.query_lens.tolist(), step.seq_lens.tolist()):
        if ql * g > 64:
            pairs += ql * (L - ql) + ql * (ql + 1) // 2
    return 4 * step.head_dim * step.num_q_heads * pairs


def bench_mixed(args, dev, stream, world, clocks):
    """Mixed prefill + decode step (Llama-3-8B attention shape): query tokens/s,
    plus the prefill chunks alone against the bf16 tensor peak."""
    import torch
    from paged_kv_cache_469_b200.inputs import prefill_part, workload
    from paged_kv_cache_469_b200.step import DeviceStep
    step = workload(MIXED_WORKLOAD)
    n = min(args.steps, 200)
    dss = [DeviceStep(step, device=str(dev)) for _ in range(copies_for(step))]
    graphs = [d.capture("fused") for d in dss]
    for i in range(args.warmup):
        graphs[i % len(dss)].replay()
    torch.cuda.synchronize(dev)
    barrier(world)
    with clocks.window() if clocks else _nullctx():
        step_ms = timed_loop([g.replay for g in graphs], stream, n)
    barrier(world)
    step_ms = max_over_ranks(step_ms, world)
    tokens = sum_over_ranks(step.num_tokens, world)
    g = step.num_q_heads // step.num_kv_heads
    kv_dec = int(sum(L for L, q in zip(step.seq_lens.tolist(), step.query_lens.tolist())
                     if q * g <= 64)) * 2 * step.num_kv_heads * step.head_dim * 2
    copies = len(dss)
    del dss, graphs
    torch.cuda.empty_cache()
    # the same step's prefill chunks alone (same lengths, same shape)
    pre = prefill_part(step)
    dps = [DeviceStep(pre, device=str(dev)) for _ in range(copies_for(pre))]
    pgraphs = [d.capture("attention") for d in dps]
    for i in range(args.warmup):
        pgraphs[i % len(dps)].replay()
    torch.cuda.synchronize(dev)
    barrier(world)
    with clocks.window() if clocks else _nullctx():
        pre_ms = timed_loop([g.replay for g in pgraphs], stream, n)
    barrier(world)
    pre_ms = max_over_ranks(pre_ms, world)
    flops = prefill_flops(pre)
    peaks = load_peaks()
    tflops = flops / (pre_ms / 1e3) / 1e12
    pre_copies = len(dps)
    del dps, pgraphs
    torch.cuda.empty_cache()
    return {"workload": MIXED_WORKLOAD, "value": round(tokens / (step_ms / 1e3), 1),
            "unit": "query tokens/s", "ms_per_step": round(step_ms, 4), "steps": n,
            "query_tokens_per_step_per_gpu": step.num_tokens,
            "decode_kv_bytes_per_step_per_gpu": kv_dec, "copies_rotated": copies,
            "prefill_only": {"ms": round(pre_ms, 4), "gflop": round(flops / 1e9, 3),
                             "tflops": round(tflops, 1),
                             "frac_of_bf16_peak": round(tflops / peaks["bf16_tflops"], 4),
                             "frac_of_bf16_sustained": round(
                                 tflops / peaks["bf16_tflops_sustained"], 4),
                             "peak_source": peaks["source"], "copies_rotated": pre_copies,
                             "kernels": ("prefill_tcgen05_kernel<128> (work list from the "
                                         "host copies of the step's lengths)")}}


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
        lib.plan_step(fq, state, nc_t, ql_t, tables, seq_lens, qsl, slots, stream=stream)

    call()
    torch.cuda.synchronize(dev)
    # both product paths must agree before anything is timed
    if not (np.array_equal(tables.cpu().numpy(), tables1) and
            np.array_equal(slots.cpu().numpy(), slots1) and
            np.array_equal(qsl.cpu().numpy(), qsl1) and
            np.array_equal(seq_lens.cpu().numpy(), nc + ql) and
            state.cpu().tolist()[:3] == [head0 + per_call, 0, 0]):
        raise RuntimeError("pa_plan_step and the host planner disagree")
    # every call repeats the step (same counts, the next blocks of the queue)
    left = len(step.free_queue) - head0 - per_call
    n = int(max(1, min(args.steps, left // max(1, per_call) - args.warmup)))
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    dev_us = timed_loop([call], stream, n) * 1e3
    if state[1].item() != 0:
        raise RuntimeError("pa_plan_step refused a timed call")

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
            "device_timing": "back-to-back pa_plan_step calls, CUDA events around the loop",
            "host_us_per_step": round(statistics.median(host_us), 1),
            "host_path": ("BlockPool.allocate_slots per sequence, block_table, slot_mapping, "
                          "query_start_loc, four pinned copies to the device, stream sync "
                          "(median of 20)"),
            "equal_outputs": True}


def bench_ours(args) -> None:
    import numpy as np
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

    # ---- device-resident steps, back to back over the rotating copies: one
    # CUDA graph replay per step (and, for reference, plain stream launches)
    step_graphs = [d.capture("fused") for d in dss]
    attn_graphs = [d.capture("attention") for d in dss]
    for i in range(args.warmup):
        step_graphs[i % copies].replay()
        dss[i % copies].run_fused()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local) if rank == 0 or world > 1 else None
    barrier(world)
    torch.cuda.synchronize(dev)
    with clocks.window() if clocks else _nullctx():
        step_ms = timed_loop([g.replay for g in step_graphs], stream, args.steps)
    barrier(world)
    torch.cuda.synchronize(dev)
    # the attention call alone (the roofline's kernel): back-to-back stream
    # launches, each a programmatic dependent of the one before, so that the
    # interval is the kernel's own time (a one-kernel graph per call would add
    # its launch gap)
    with clocks.window() if clocks else _nullctx():
        attn_ms = timed_loop([d.attention for d in dss], stream, args.steps)
    barrier(world)
    torch.cuda.synchronize(dev)
    with clocks.window() if clocks else _nullctx():
        attn_graph_ms = timed_loop([g.replay for g in attn_graphs], stream, args.steps)
    barrier(world)
    attn_graph_ms = max_over_ranks(attn_graph_ms, world)
    torch.cuda.synchronize(dev)
    with clocks.window() if clocks else _nullctx():
        stream_step_ms = timed_loop([d.run_fused for d in dss], stream, args.steps)
    barrier(world)
    stream_step_ms = max_over_ranks(stream_step_ms, world)
    step_ms_max = max_over_ranks(step_ms, world)
    graph_step_ms = step_ms_max
    # the headline is the faster of the two ways to run the step: graph replays
    # (one per step) or plain back-to-back calls (each launch a programmatic
    # dependent of the previous one, which graph replays cannot be)
    launch = ("one CUDA graph replay per step of pa_attention_varlen_write_cache "
              "(cache write fused into the decode kernel)")
    if stream_step_ms < step_ms_max:
        step_ms_max = stream_step_ms
        launch = ("back-to-back pa_attention_varlen_write_cache calls, one per step "
                  "(cache write fused into the decode kernel; each launch a programmatic "
                  "dependent of the previous step's)")
    attn_ms_max = max_over_ranks(attn_ms, world)
    bytes_rank = kv_bytes(step)
    bytes_all = sum_over_ranks(bytes_rank, world)
    value = bytes_all / (step_ms_max / 1e3) / 1e9

    # ---- end to end through the public API from pinned host buffers: every step
    # copies its inputs in (one copy: the step's inputs are packed into one
    # buffer on both sides), runs, and copies its output back
    ds0 = dss[0]
    host_ins = [d.host_inputs() for d in dss]
    host_out = torch.empty(ds0.out.shape, dtype=torch.int16).pin_memory()
    h2d = host_ins[0].numel()
    d2h = host_out.numel() * host_out.element_size()

    def e2e_graph(r):
        d, hin = dss[r], host_ins[r]

        def copies_in():
            d.inputs.copy_(hin, non_blocking=True)

        def copy_out():
            host_out.copy_(d.out.view(torch.int16), non_blocking=True)
        return d.capture("fused", prologue=copies_in, epilogue=copy_out)

    e2e_graphs = [e2e_graph(r) for r in range(copies)]
    for i in range(args.warmup):
        e2e_graphs[i % copies].replay()
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    with clocks.window() if clocks else _nullctx():
        e2e_ms = timed_loop([g.replay for g in e2e_graphs], stream, args.steps)
    barrier(world)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_value = bytes_all / (e2e_ms / 1e3) / 1e9
    del dss, host_ins, ds0, step_graphs, attn_graphs, e2e_graphs
    torch.cuda.empty_cache()
    mixed = None if args.no_mixed else bench_mixed(args, dev, stream, world, clocks)
    planner = None if args.no_planner or rank != 0 else bench_planner(args, dev, stream)
    clk = clocks.stop() if clocks else None

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    peaks = load_peaks()
    achieved = bytes_rank / (attn_ms_max / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": DECODE_TRAFFIC_BYTES, "traffic_unit": "bytes per launch (ncu)",
                "kernel": "decode_splitk_kernel<64,false,4,4,false> (attention call without the fused cache write)",
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
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 5),
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
            "attention_ms": round(attn_ms_max, 5),
            "launch": launch,
            "graph_replay_ms_per_step": round(graph_step_ms, 5),
            "stream_launch_ms_per_step": round(stream_step_ms, 5),
            "attention_graph_replay_ms": round(attn_graph_ms, 5),
            "gpu_launches": args.steps,
            "mixed_step": mixed,
            "plan_step": planner,
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "ms_per_step": round(e2e_ms, 4),
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
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
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_ours(args)


if __name__ == "__main__":
    main()
