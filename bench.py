"""Benchmark of the BigBird ITC block-sparse attention forward on B200.

One step = one forward pass (every row of the pattern: global rows, second
rows, middle rows, epilogue) over one batch of the BigBird-base attention
workload (B=4, H=12, L=4096, d=64, block=64, r=3, bf16, valid lengths
U[2048, 4096]) by default. Metric: sparse TFLOP/s = 4 * B * H * L *
keys_per_row * d / t.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

With N > 1 (launched by torch.distributed.run) every rank runs its own batch
of the workload (weak scaling: heads/batches are independent; no data-path
collective); time = max over ranks. `--impl reference` times the fp64 CPU
oracle on a bounded sample of the same workload on the host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "block-sparse attention TFLOP/s and % of BF16 tensor peak at L=4096, 1×B200"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "bigbird_base_l4096"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one forward
# kernel launch per workload, from an ncu capture of the current kernel
# source; an entry is removed whenever the kernel changes.
# Share of one forward call taken by the fp16 attention kernel in the ncu
# launch list of the same workload (cold-cache, serialised launches: the share,
# not the absolute, carries over to the live timing).
FWD_KERNEL_SHARE: dict = {"bigbird_base_l4096": 103.23 / (103.23 + 10.19)}
BWD_DRAM_BYTES_PER_LAUNCH: dict = {
    # 146.70 MB read + 81.14 MB written, dk/dv launch (d = 64), mean of 11 launches
    "bigbird_base_l4096": 227.842141e6,
}
FWD_DRAM_BYTES_PER_LAUNCH: dict = {
    # 84.66 MB read + 10.06 MB written, split-row kernel's fp16 instance (d = 64), mean of 30 launches
    "bigbird_base_l4096": 94.724471e6,
}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """nvidia-smi clock/throttle sampling; keeps the samples taken inside the
    timed window [t0, t1] (host wall clock)."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"bb_clocks_{os.getpid()}.csv")
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        from datetime import datetime
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[2]), float(f[3]), f[6], f[7], f[8], f[9]))
            except ValueError:
                continue
        os.unlink(self.path)
        inside = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= self.t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for r in inside:
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 r[3:]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r[1] for r in inside])), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside)}


def _oracle_sample(w, inp, ra, budget_s: float):
    """Time the oracle, as it stands, on whole (b, h) heads until budget_s is
    spent. Returns (sparse FLOPs processed, seconds, heads, threads)."""
    import oracle
    from threadpoolctl import threadpool_info

    threads = max([t.get("num_threads", 1) for t in threadpool_info()] or [1])
    per_head = oracle.sparse_flops(1, 1, w.L, w.d, w.block, w.r)
    done, heads = 0.0, 0
    t0 = time.perf_counter()
    for b in range(w.B):
        for h in range(w.H):
            sub = {x: inp[x][b:b + 1, h:h + 1] for x in "qkv"}
            sm = None if inp["seq_mask"] is None else inp["seq_mask"][b:b + 1].numpy()
            oracle.attention(sub["q"], sub["k"], sub["v"], None if ra is None else ra[h:h + 1], sm, w.block, w.r)
            done += per_head
            heads += 1
            if time.perf_counter() - t0 >= budget_s:
                return done, time.perf_counter() - t0, heads, threads
    return done, time.perf_counter() - t0, heads, threads


def _sparse_ref_sample(w, inp, ra, budget_s: float):
    """Time the C/OpenMP sparse brute-force reference (oracle/sparse_ref.c) on
    whole (b, h) heads, all host cores, until budget_s is spent. Returns
    (sparse FLOPs processed, seconds, heads, threads)."""
    import oracle
    from oracle import sparse_ref

    threads = len(os.sched_getaffinity(0))
    sparse_ref.build()
    per_head = oracle.sparse_flops(1, 1, w.L, w.d, w.block, w.r)
    done, heads = 0.0, 0
    t0 = time.perf_counter()
    for b in range(w.B):
        for h in range(w.H):
            sub = {x: inp[x][b:b + 1, h:h + 1] for x in "qkv"}
            sm = None if inp["seq_mask"] is None else inp["seq_mask"][b:b + 1].numpy()
            sparse_ref.sparse_attention(sub["q"], sub["k"], sub["v"], None if ra is None else ra[h:h + 1], sm,
                                        w.block, w.r, threads=threads)
            done += per_head
            heads += 1
            if time.perf_counter() - t0 >= budget_s:
                return done, time.perf_counter() - t0, heads, threads
    return done, time.perf_counter() - t0, heads, threads


def run_reference(args):
    """The oracle on the host cores: the reference arm of this benchmark."""
    world, rank, _ = _dist_env()
    if rank != 0:
        return 0
    import oracle
    from block_sparse_long_attention_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS[args.workload]
    inp = make_inputs(w)
    ra = None if oracle.is_fallback(w.L, w.block, w.r) else oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
    step_budget = float(os.environ.get("BB_REF_STEP_SECONDS", "5"))
    for _ in range(args.warmup):
        _oracle_sample(w, inp, ra, 0.0)
    tot_flops, tot_s, heads, threads = 0.0, 0.0, 0, 1
    for _ in range(args.steps):
        f, s, hh, threads = _oracle_sample(w, inp, ra, step_budget)
        tot_flops += f
        tot_s += s
        heads += hh
    value = tot_flops / tot_s / 1e12
    sample = f"{heads} whole (b,h) heads of {w.name} over {args.steps} steps (~{step_budget:.0f} s each)"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": _config(w, world), "l2": "oracle on host cores; no L2 flush (CPU)",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(w, world):
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d, "block": w.block, "r": w.r,
            "padding": "none" if w.pad is None else str(w.pad), "global_batch": w.B * world,
            "seq_len": w.L, "parallelism": f"dp{world} (independent batches per GPU)"}


L2_NOTE = "L2 flushed (2x L2 write) before every timed step"


def run_cuda(args):
    import torch
    import torch.distributed as dist

    import block_sparse_long_attention_b200 as bb
    from block_sparse_long_attention_b200.workloads import WORKLOADS, make_inputs

    world, rank, local = _dist_env()
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, seed=w.seed + rank)
    nb = w.L // w.block
    sparse = not bb.is_fallback(w.L, w.block, w.r)
    ra_h = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed) if sparse else None

    # device-resident inputs
    q, k, v = (inp[x].to(dev) for x in "qkv")
    sm = None if inp["seq_mask"] is None else inp["seq_mask"].to(dev)
    ra = None if ra_h is None else torch.from_numpy(ra_h).to(dev)
    out = torch.empty_like(q)
    ws = torch.zeros(max(bb.workspace_size(w.B, w.H, w.L, w.d, w.block, w.r), 1), dtype=torch.uint8, device=dev)
    props = torch.cuda.get_device_properties(dev)
    flush = torch.empty(2 * int(props.L2_cache_size) // 4 + (1 << 20), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        bb.fwd(q, k, v, ra, sm, block=w.block, r=w.r, out=out, workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if bb.device_status() != 0:
        raise RuntimeError("device error during warm-up")

    # The K timed steps are repeated until the timed region lasts about a
    # second, so that the clock sampler (one sample per 50 ms) sees it; the
    # estimate comes from one untimed pass, and every rank uses rank 0's count.
    t_est = time.perf_counter()
    for _ in range(args.steps):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    t_est = time.perf_counter() - t_est
    reps = max(int(args.repeat), int(np.ceil(float(args.min_timed_s) / max(t_est, 1e-6))))
    if world > 1:
        rt = torch.tensor([reps], device=dev, dtype=torch.int64)
        dist.broadcast(rt, 0)
        reps = int(rt.item())
    n_timed = reps * args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_timed)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n_timed)]
    sampler = ClockSampler(dev.index if world == 1 else local)
    sampler.start()
    time.sleep(1.0)  # nvidia-smi start-up
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.t0 = time.time()
    for i in range(n_timed):
        flush.zero_()  # L2 flush between timed iterations (outside the events)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    sampler.t1 = time.time()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms = float(np.mean([s.elapsed_time(e) for s, e in zip(starts, ends)]))
    if bb.device_status() != 0:
        raise RuntimeError("device error during the timed region")

    # the same calls back to back with a warm L2 (no flush between them)
    n_warm = min(args.steps, 1000)
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step()
    w0.record(stream)
    for _ in range(n_warm):
        step()
    w1.record(stream)
    torch.cuda.synchronize(dev)
    warm_ms = w0.elapsed_time(w1) / n_warm

    # end to end through the public API: pinned host inputs in, host result
    # out, through bigbird_attn_fwd_host (copies in, compute and copies out of
    # consecutive sequences overlap on the library's own streams)
    pin = {x: inp[x].contiguous().pin_memory() for x in "qkv"}
    sm_pin = None if inp["seq_mask"] is None else inp["seq_mask"].contiguous().pin_memory()
    ra_pin = None if ra_h is None else torch.from_numpy(ra_h).pin_memory()
    out_pin = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(pin[x].numel() * pin[x].element_size() for x in "qkv")
    h2d += 0 if sm_pin is None else sm_pin.numel()
    h2d += 0 if ra_pin is None else ra_pin.numel() * 4
    d2h = out_pin.numel() * out_pin.element_size()
    host_scratch = torch.empty(max(1, bb.fwd_host_scratch_bytes(w.B, w.H, w.L, w.d, w.block, w.r)),
                               dtype=torch.uint8, device=dev)

    def e2e_step():
        bb.fwd_host(pin["q"], pin["k"], pin["v"], ra_pin, sm_pin, out_pin, block=w.block, r=w.r,
                    scratch=host_scratch)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize(dev)
    e_steps = max(3, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e_steps

    if world > 1:
        t = torch.tensor([ms, e2e_ms, warm_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, e2e_ms, warm_ms = float(t[0]), float(t[1]), float(t[2])

    import oracle  # work accounting only (FLOP count formula)
    flops = oracle.sparse_flops(w.B, w.H, w.L, w.d, w.block, w.r)
    value = flops * world / (ms * 1e-3) / 1e12
    e2e_value = flops * world / (e2e_ms * 1e-3) / 1e12
    peaks, src = _peaks()
    achieved = flops / (ms * 1e-3) / 1e12
    # The tensor-core path launches the fp16 attention kernel and its bf16
    # instance (which merges the split global rows' key ranges, and redoes the
    # call first only when V holds a value fp16 cannot represent). It is the
    # path that takes a workspace; the CUDA-core path launches one kernel.
    ws_bytes = bb.workspace_size(w.B, w.H, w.L, w.d, w.block, w.r)
    generic = ws_bytes == 0
    launches_per_call = 1 if generic else 2
    if generic:
        # the CUDA-core kernel: fp32 peak from unit counts and clocks
        sm_mhz = (clocks or {}).get("sm_max_mhz") or 1965.0
        peak = props.multi_processor_count * 128 * 2 * float(sm_mhz) * 1e-6
        roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": None, "kernel": "bigbird_generic_fwd_kernel (fp32 CUDA cores)",
                "peak_source": "SMs x 128 fp32 FMA lanes x 2 x max SM clock"}
    else:
        peak = float(peaks["bf16_tflops"])
        traffic = FWD_DRAM_BYTES_PER_LAUNCH.get(w.name) if world == 1 else None
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "kernel": "bigbird_fwd2_kernel<fp16> (d = 64); the duration is the whole call, which adds its bf16 "
                          "instance (here only the global-row merge), launched as its programmatic "
                          "dependent, so this is a lower bound on the attention kernel's own rate",
                "peak_source": f"{src} bf16 dense burst (kernel timed alone)"}
        share = FWD_KERNEL_SHARE.get(w.name)
        if share:
            # the attention kernel alone: the call's time times its share in
            # the ncu launch list
            roof["dominant_kernel"] = {"name": "bigbird_fwd2_kernel<fp16>", "share_of_call": share,
                                       "achieved": achieved / share, "frac": achieved / share / peak,
                                       "share_source": "ncu launch list of this workload (gpu__time_duration.sum)"}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(w, world), "l2": L2_NOTE,
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": e2e_ms},
        "gpu_launches": n_timed * launches_per_call,
        "timed_repeats": reps,
        "warm_l2": {"ms_per_step": warm_ms, "value": flops * world / (warm_ms * 1e-3) / 1e12, "unit": UNIT,
                    "steps": n_warm, "note": "same calls back to back, no L2 flush (not the headline)"},
        "clocks": clocks,
    }
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            budget = float(os.environ.get("BB_CPU_BASELINE_SECONDS", "15"))
            ra_o = None if ra_h is None else oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
            f, s, heads, threads = _oracle_sample(w, inp, ra_o, budget)
            line["cpu_baseline"] = {"value": f / s / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
                                    "sample": f"{heads} whole (b,h) heads of {w.name} ({s:.1f} s)"}
            budget2 = float(os.environ.get("BB_CPU_SPARSE_SECONDS", "8"))
            f2, s2, heads2, threads2 = _sparse_ref_sample(w, inp, ra_o, budget2)
            line["cpu_sparse_baseline"] = {
                "value": f2 / s2 / 1e12, "unit": UNIT, "cores": threads2,
                "kind": "C/OpenMP sparse brute force, fp64 (oracle/sparse_ref.c, pinned to the oracle)",
                "sample": f"{heads2} whole (b,h) heads of {w.name} ({s2:.1f} s)"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_bwd(args):
    """Backward pass (bigbird_attn_bwd) on the same workload: one step = the
    gradients dq, dk, dv of one batch, with the forward's out and lse (from
    bigbird_attn_fwd_train) and dout resident. Single GPU."""
    import torch

    import block_sparse_long_attention_b200 as bb
    from block_sparse_long_attention_b200.workloads import WORKLOADS, make_inputs

    world, rank, local = _dist_env()
    if rank != 0:
        return 0
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    inp = make_inputs(w)
    sparse = not bb.is_fallback(w.L, w.block, w.r)
    q, k, v = (inp[x].to(dev) for x in "qkv")
    sm = None if inp["seq_mask"] is None else inp["seq_mask"].to(dev)
    ra = torch.from_numpy(bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)).to(dev) if sparse else None
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(w.seed)).to(torch.bfloat16).to(dev)
    out, lse = bb.fwd_train(q, k, v, ra, sm, block=w.block, r=w.r)
    props = torch.cuda.get_device_properties(dev)
    flush = torch.empty(2 * int(props.L2_cache_size) // 4 + (1 << 20), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ws = torch.zeros(max(1, bb.bwd_workspace_size(w.B, w.H, w.L, w.d, w.block, w.r)), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        bb.bwd(q, k, v, out, dout, lse, ra, sm, block=w.block, r=w.r, workspace=ws)
    torch.cuda.synchronize(dev)
    # as in the forward: the timed calls are repeated until the timed region
    # lasts about min_timed_s, so that the clock sampler sees it
    steps = min(args.steps, 50)
    t_est = time.perf_counter()
    for _ in range(steps):
        flush.zero_()
        bb.bwd(q, k, v, out, dout, lse, ra, sm, block=w.block, r=w.r, workspace=ws)
    torch.cuda.synchronize(dev)
    t_est = time.perf_counter() - t_est
    reps = max(int(args.repeat), int(np.ceil(float(args.min_timed_s) / max(t_est, 1e-6))))
    steps *= reps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(1.0)
    torch.cuda.synchronize(dev)
    sampler.t0 = time.time()
    for i in range(steps):
        flush.zero_()
        starts[i].record(stream)
        bb.bwd(q, k, v, out, dout, lse, ra, sm, block=w.block, r=w.r, workspace=ws)
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    sampler.t1 = time.time()
    clocks = sampler.stop()
    if bb.device_status() != 0:
        raise RuntimeError("device error during the timed region")
    ms = float(np.mean([a.elapsed_time(b) for a, b in zip(starts, ends)]))
    import oracle  # work accounting only (FLOP count formula)
    flops = oracle.backward_flops(w.B, w.H, w.L, w.d, w.block, w.r)
    value = flops / (ms * 1e-3) / 1e12
    peaks, src = _peaks()
    peak = float(peaks["bf16_tflops"])
    # row dot, dk/dv kernel, dq kernel, and the partial-sum launch when the
    # global rows are split into key ranges
    launches = 3 + (1 if bb.bwd_workspace_size(w.B, w.H, w.L) > 256 + 4 * w.B * w.H * w.L + 255 else 0)
    line = {
        "metric": "block-sparse attention backward TFLOP/s (dq, dk, dv) at L=4096, 1xB200", "value": value,
        "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "pass": "bwd",
        "config": _config(w, 1), "l2": L2_NOTE,
        "roofline": {"bound": "tensor", "achieved": value, "peak": peak, "unit": "TFLOP/s", "frac": value / peak,
                     # DRAM bytes of one dk/dv launch (the larger kernel), from an ncu capture of
                     # the current source (None until one is taken)
                     "traffic": BWD_DRAM_BYTES_PER_LAUNCH.get(w.name),
                     "kernel": "bwd_kernel<dq> + bwd_kernel<dk,dv> (tcgen05, bf16 operands); the duration is the "
                               "whole call (row dot and partial sums included), the work the algorithmic 5 GEMM-"
                               "shaped products; traffic is the dk/dv kernel's",
                     "peak_source": f"{src} bf16 dense burst"},
        "gpu_launches": steps * launches, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_probs(args):
    """Attention-probability export (bigbird_attn_probs, packed block-sparse
    layout, fp32) on the same workload: one step = the weights of every
    attended (query, key) pair of one batch, with q, k and the forward's lse
    resident. HBM-bound: the algorithmic bytes are the weights written plus
    q, k, lse and the mask read once. Single GPU."""
    import torch

    import block_sparse_long_attention_b200 as bb
    from block_sparse_long_attention_b200.workloads import WORKLOADS, make_inputs

    world, rank, local = _dist_env()
    if rank != 0:
        return 0
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    inp = make_inputs(w)
    sparse = not bb.is_fallback(w.L, w.block, w.r)
    q, k, v = (inp[x].to(dev) for x in "qkv")
    sm = None if inp["seq_mask"] is None else inp["seq_mask"].to(dev)
    ra = torch.from_numpy(bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)).to(dev) if sparse else None
    _, lse = bb.fwd_train(q, k, v, ra, sm, block=w.block, r=w.r)
    G, nbr, slots = bb.probs_layout(w.L, w.block, w.r, w.d)
    props = torch.cuda.get_device_properties(dev)
    flush = torch.empty(2 * int(props.L2_cache_size) // 4 + (1 << 20), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    res = {}
    for dtype, esize in ((torch.float32, 4), (torch.bfloat16, 2)):
        pg = torch.empty((w.B, w.H, G, w.block, w.L), dtype=dtype, device=dev)
        pb = torch.empty((w.B, w.H, nbr, slots, w.block, w.block), dtype=dtype, device=dev) if nbr else None

        def step():
            bb.probs(q, k, lse, ra, sm, block=w.block, r=w.r, out_dtype=dtype, out=(pg, pb))

        for _ in range(args.warmup):
            flush.zero_()
            step()
        torch.cuda.synchronize(dev)
        steps = min(args.steps, 4000)  # ~1 s of timed region: long enough for the clock samples
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        sampler = ClockSampler(dev.index)
        sampler.start()
        time.sleep(1.0)
        torch.cuda.synchronize(dev)
        sampler.t0 = time.time()
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        sampler.t1 = time.time()
        clocks = sampler.stop()
        if bb.device_status() != 0:
            raise RuntimeError("device error during the timed region")
        ms = float(np.mean([a.elapsed_time(b) for a, b in zip(starts, ends)]))
        out_bytes = (pg.numel() + (0 if pb is None else pb.numel())) * esize
        in_bytes = 2 * q.numel() * 2 + lse.numel() * 4 + (0 if sm is None else sm.numel())
        res[str(dtype).split(".")[-1]] = (ms, out_bytes, in_bytes, steps, clocks)
    ms, out_bytes, in_bytes, steps, clocks = res["float32"]
    peaks, src = _peaks()
    peak = float(peaks["hbm_gbs"])
    gbs = (out_bytes + in_bytes) / (ms * 1e-3) / 1e9
    bms, bout, bin_, _, _ = res["bfloat16"]
    bgbs = (bout + bin_) / (bms * 1e-3) / 1e9
    import oracle  # work accounting only (attended pairs)
    pairs = w.B * w.H * w.L * oracle.keys_per_row(w.L, w.block, w.r)
    line = {
        "metric": "block-sparse attention-probability export GB/s (packed layout, fp32) at L=4096, 1xB200",
        "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 (bf16 inputs)",
        "data": "synthetic", "pass": "probs",
        "config": _config(w, 1), "l2": L2_NOTE,
        # traffic: one fp32 export launch at the BigBird-base workload, ncu
        # (59.05 MB read + 431.25 MB written)
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": 490.295296e6 if w.name == "bigbird_base_l4096" else None,
                     "kernel": "bigbird_probs_kernel",
                     "algorithmic_bytes": out_bytes + in_bytes,
                     "peak_source": f"{src} HBM copy bandwidth"},
        "pairs_per_s": pairs / (ms * 1e-3),
        "bf16_output": {"ms_per_step": bms, "value": bgbs, "unit": "GB/s", "frac": bgbs / peak,
                        "algorithmic_bytes": bout + bin_},
        "gpu_launches": steps, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--repeat", type=int, default=1, help="repeat the timed loop at least this many times")
    ap.add_argument("--min-timed-s", type=float, default=1.0,
                    help="repeat the K timed steps until the timed region lasts about this long (clock samples)")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd", "probs"],
                    help="fwd (default, the headline), bwd (the backward pass) or probs (probability export)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.pass_ == "bwd":
        return run_bwd(args)
    if args.pass_ == "probs":
        return run_probs(args)
    return run_cuda(args)


if __name__ == "__main__":
    sys.exit(main())
