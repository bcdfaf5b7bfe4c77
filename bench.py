#!/usr/bin/env python
"""Benchmark of exact fused linear cross-entropy (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload packed]
    python bench.py --impl reference ...      # the CPU oracle arm

One step = flce_forward + flce_backward over one synthetic batch of the
workload (inputs resident in HBM).  Credited work is 8*C*D*V FLOP per step
(forward 2CDV, backward 6CDV).  With N > 1 (torchrun) each rank runs its own
independent batch (replicas, weak scaling; the loss has no cross-rank
exchange), and the time is the max over ranks.  Rank 0 prints one JSON line.

Other modes (not the default line):
  --vocab-parallel   one vocabulary slice per rank with the NCCL exchanges of
                     a vocabulary-parallel step (strong scaling)
  --vocab-shards P   all P slices' kernels on each GPU in turn
  --filter-eps E     the backward with gradient filtering (approximate)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused linear-CE fwd+bwd TFLOP/s (8·C·D·V) & % bf16 TC peak; peak MiB"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_SOURCES = ["lm_head_projection_supervised_b200/csrc/gemm.cuh",
                "lm_head_projection_supervised_b200/csrc/ptx.cuh"]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="flce", choices=["flce", "reference"])
    p.add_argument("--workload", default="packed")
    p.add_argument("--cpu-rows", type=int, default=4096,
                   help="supervised rows in the CPU-oracle baseline sample")
    p.add_argument("--ref-rows", type=int, default=64,
                   help="supervised rows per step of the reference (oracle) arm")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--vocab-shards", type=int, default=1,
                   help="P > 1: the vocabulary-sliced form, all P slices on each GPU in turn "
                        "(the kernels of a P-way vocabulary-parallel step, exchanges in place)")
    p.add_argument("--vocab-parallel", action="store_true",
                   help="one vocabulary slice per rank (P = number of ranks, a one-rank NCCL "
                        "group without torchrun), statistics all-gathered and dH all-reduced "
                        "with NCCL; strong scaling (the whole vocabulary is split)")
    p.add_argument("--panel-backward", action="store_true",
                   help="the panel form of the backward where the single-kernel form applies "
                        "(D <= 64)")
    p.add_argument("--filter-eps", type=float, default=0.0,
                   help="> 0: the backward with gradient filtering (an approximation; see "
                        "flce_backward_filtered)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(paths):
    """Hash of the kernel sources' code: comments and blank space removed, so
    that a capture stays valid across comment-only edits."""
    import re
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_kind, workload):
    """DRAM bytes per launch of `kernel_kind` from the committed ncu summary,
    or None when absent, taken on another workload or on a different version
    of the kernel."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel_kind)
    if not e or e.get("source_hash") != source_hash(GEMM_SOURCES) or \
            e.get("workload", "packed") != workload:
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks sampled while the timed region runs
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = "".join(c for c in uuid.lower() if c in "0123456789abcdef")
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [[x.strip() for x in line.split(",")] for line in out.strip().splitlines()]
        rows = [r for r in rows if len(r) >= 9]
        mine = [r for r in rows
                if "".join(c for c in r[0].lower() if c in "0123456789abcdef").endswith(self.uuid)]
        if mine:
            rows = mine
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for parts in rows:
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        load = [s for s, p in zip(sm, power) if p > 300.0] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "matched_uuid": bool(mine),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample of supervised rows
# ---------------------------------------------------------------------------
_DECODED = {}


def oracle_sample_run(inp, rows_wanted, seed=0):
    """Times the oracle's dense forward + backward on a seeded sample of
    supervised rows (inputs decoded to float64 outside the timed call)."""
    import numpy as np
    import torch
    from oracle import flce_oracle as orc
    idx, C = orc.supervised_rows(inp.labels, inp.mask)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(idx, size=min(rows_wanted, C), replace=False))
    key = id(inp)
    if key not in _DECODED:
        _DECODED.clear()
        _DECODED[key] = (inp.W64(), inp.b64())
    W64, b64 = _DECODED[key]
    H64 = inp.H64()[rows]
    y = inp.labels[rows]
    mk = inp.mask[rows]
    t0 = time.perf_counter()
    orc.forward_backward(H64, W64, b64, y, mk, lam=inp.lam, row_block=256)
    dt = time.perf_counter() - t0
    Cs = orc.supervised_rows(y, mk)[1]
    return dt, Cs, torch.get_num_threads()


def run_reference(args, inp, spec):
    """The oracle as the reference arm: each step is a bounded row sample."""
    from oracle import flce_oracle as orc  # noqa: F401
    times, Cs, cores = [], 0, 0
    for i in range(args.warmup + args.steps):
        dt, Cs, cores = oracle_sample_run(inp, args.ref_rows, seed=i)
        if i >= args.warmup:
            times.append(dt)
    step_s = statistics.mean(times)
    value = 8.0 * Cs * inp.D * inp.V / step_s / 1e12
    sample = (f"{Cs} supervised rows of {spec.name} per step (full V={inp.V}, D={inp.D}), "
              "fp64 dense forward+backward")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(spec, inp, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(spec, inp, n):
    import numpy as np
    C = int(np.count_nonzero((inp.labels != -100) & (inp.mask != 0)))
    w_mb = inp.V * inp.D * 2 / 1e6
    l2 = (f"inputs larger than L2 (W alone is {w_mb:.0f} MB > 126 MB); no flush" if w_mb > 126
          else f"W is {w_mb:.0f} MB, may stay L2-resident between steps (not flushed)")
    return {"workload": f"{spec.name}: N={inp.N} D={inp.D} V={inp.V} {spec.dtype}"
                        f"{' +bias' if inp.b is not None else ''}, C={C}",
            "N": inp.N, "D": inp.D, "V": inp.V, "C": C, "dtype": spec.dtype,
            "labels": spec.label_dist, "parallelism": f"replicas{n}", "l2": l2}


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank value over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_tflops(flop_step: float, steps: int, ms_max: float, world: int) -> float:
    """Whole-job throughput: every rank runs `steps` steps of `flop_step` FLOP."""
    return world * flop_step * steps / (ms_max * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_vocab_parallel(args, spec, rank, world, dev):
    """One vocabulary slice per rank: the NCCL exchanges of a vocabulary-
    parallel step are inside the timed region and are also timed on their
    own (all-gather of the per-row statistics, all-reduce of dH)."""
    import datetime
    import socket
    import numpy as np
    import torch
    import torch.distributed as dist
    from lm_head_projection_supervised_b200 import binding
    from lm_head_projection_supervised_b200 import vocab_parallel as vpar
    from lm_head_projection_supervised_b200 import workloads as wl

    if not dist.is_initialized():
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            if "MASTER_PORT" not in os.environ:
                with socket.socket() as so:
                    so.bind(("127.0.0.1", 0))
                    os.environ["MASTER_PORT"] = str(so.getsockname()[1])
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    P = dist.get_world_size()
    inp = wl.make_inputs(spec)  # the same batch on every rank: H and labels are replicated
    v0, n = vpar.vocab_slice(inp.V, P, rank)
    cfg = workload_config(spec, inp, P)
    cfg["parallelism"] = f"vocab{P}"
    cfg["slice"] = [v0, n]
    C = cfg["C"]
    tdt = torch.bfloat16 if spec.dtype == "bf16" else torch.float16
    H = torch.from_numpy(inp.H.view(np.int16)).view(tdt).to(dev)
    Ws = torch.from_numpy(inp.W[v0:v0 + n].view(np.int16)).view(tdt).to(dev)
    bs = None if inp.b is None else torch.from_numpy(inp.b[v0:v0 + n].view(np.int16)).view(
        tdt).to(dev)
    y = torch.from_numpy(inp.labels).to(dev)
    mk = torch.from_numpy(inp.mask).to(dev)
    ws = binding.Workspace(inp.N, inp.D, n, tdt, dev)
    cws = binding.CombineWorkspace(inp.N, dev)
    st = torch.empty((inp.N, 4), dtype=torch.float32, device=dev)
    dH = torch.empty((inp.N, inp.D), dtype=torch.float32, device=dev)
    dW = torch.empty((n, inp.D), dtype=torch.float32, device=dev)
    db = None if bs is None else torch.empty(n, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(marks=None):
        binding.shard_forward(H, Ws, bs, y, mk, -100, v0=v0, V_total=inp.V, ws=ws, out=st)
        if marks:
            marks[0].record(stream)
        allst = vpar.gather_stats(st)
        if marks:
            marks[1].record(stream)
        _, m, logs = binding.shard_combine(allst, y, mk, -100, ws=cws)
        binding.shard_backward(H, Ws, bs, y, mk, -100, m, logs, v0=v0, V_total=inp.V,
                               lam=inp.lam, ws=ws, out=(dH, dW, db))
        if marks:
            marks[2].record(stream)
        dist.all_reduce(dH, op=dist.ReduceOp.SUM)
        if marks:
            marks[3].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    if binding.device_status(ws) != 0 or binding.device_status(cws) != 0:
        raise RuntimeError("device error during warm-up")
    marks = [[ev() for _ in range(4)] for _ in range(args.steps)]
    e0, e1 = ev(), ev()
    dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(str(torch.cuda.get_device_properties(dev).uuid))
    sampler.start()
    e0.record(stream)
    for k in range(args.steps):
        step(marks[k])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clocks = sampler.stop()
    total_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    gather_ms = max_over_ranks(statistics.median(mk_[0].elapsed_time(mk_[1]) for mk_ in marks), dev)
    reduce_ms = max_over_ranks(statistics.median(mk_[2].elapsed_time(mk_[3]) for mk_ in marks), dev)
    flop_step = 8.0 * C * inp.D * inp.V  # the whole vocabulary, split over the ranks
    line = {"metric": METRIC, "value": flop_step * args.steps / (total_ms * 1e-3) / 1e12,
            "unit": UNIT, "n_gpus": P, "steps": args.steps, "warmup": max(args.warmup, 3),
            "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": spec.dtype, "data": "synthetic", "config": cfg,
            "exchange": {"allgather_stats_bytes": 16 * P * inp.N,
                         "allreduce_dH_bytes": 4 * inp.N * inp.D,
                         "allgather_ms": gather_ms, "allreduce_ms": reduce_ms,
                         "note": "NCCL collectives through torch.distributed, timed with events "
                                 "on the compute stream; medians over steps, max over ranks"},
            "clocks": clocks, "e2e": None,
            "note": "vocabulary-parallel mode; the default mode runs independent replicas"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.destroy_process_group()


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    from lm_head_projection_supervised_b200 import workloads as wl
    spec = wl.SPECS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return
        inp = wl.make_inputs(spec)
        run_reference(args, inp, spec)
        return

    if args.vocab_parallel:
        import torch
        torch.cuda.set_device(local_rank)
        run_vocab_parallel(args, spec, rank, world, torch.device("cuda", local_rank))
        return

    import numpy as np
    import torch
    from lm_head_projection_supervised_b200 import binding

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    inp = wl.make_inputs(spec, seed=wl.SEED_BASE + spec.k + 1000 * rank)
    cfg = workload_config(spec, inp, world)
    cfg["backward"] = ("single-kernel" if inp.D <= 64 and not args.panel_backward and
                       args.filter_eps <= 0 else "panel")
    if args.filter_eps > 0:
        cfg["filter_eps"] = args.filter_eps
        cfg["note"] = "backward with gradient filtering: an approximation, not the exact path"
    C = cfg["C"]
    flop_step = 8.0 * C * inp.D * inp.V

    # CPU baseline first (rank 0, one GPU): no GPU work has started yet.
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, Cs, cores = oracle_sample_run(inp, args.cpu_rows)
        cpu_baseline = {"value": 8.0 * Cs * inp.D * inp.V / dt / 1e12, "unit": UNIT,
                        "cores": cores, "kind": "oracle",
                        "sample": f"{Cs} supervised rows of {spec.name} (full V={inp.V}, "
                                  f"D={inp.D}), fp64 dense forward+backward, {dt:.1f} s"}

    tdt = torch.bfloat16 if spec.dtype == "bf16" else torch.float16
    torch.cuda.reset_peak_memory_stats(dev)
    H = torch.from_numpy(inp.H.view(np.int16)).view(tdt).to(dev)
    W = torch.from_numpy(inp.W.view(np.int16)).view(tdt).to(dev)
    b = None if inp.b is None else torch.from_numpy(inp.b.view(np.int16)).view(tdt).to(dev)
    y = torch.from_numpy(inp.labels).to(dev)
    mk = torch.from_numpy(inp.mask).to(dev)
    in_mib = sum(t.numel() * t.element_size() for t in (H, W, y, mk) + ((b,) if b is not None
                                                                            else ())) / 2**20
    ws = binding.Workspace(inp.N, inp.D, inp.V, tdt, dev)
    dH = torch.empty((inp.N, inp.D), dtype=torch.float32, device=dev)
    dW = torch.empty((inp.V, inp.D), dtype=torch.float32, device=dev)
    db = None if b is None else torch.empty(inp.V, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    P = args.vocab_shards
    if P > 1:
        from lm_head_projection_supervised_b200 import vocab_parallel as vpar
        bounds = [vpar.vocab_slice(inp.V, P, r) for r in range(P)]
        ws = binding.Workspace(inp.N, inp.D, max(n for _, n in bounds), tdt, dev)
        stats = torch.empty((P, inp.N, 4), dtype=torch.float32, device=dev)
        cws = binding.CombineWorkspace(inp.N, dev)
        cfg["vocab_shards"] = P

        def fwd(x):
            H, W, b, y, mk = x
            for r, (v0, n) in enumerate(bounds):
                binding.shard_forward(H, W[v0:v0 + n], None if b is None else b[v0:v0 + n], y,
                                      mk, -100, v0=v0, V_total=inp.V, ws=ws, out=stats[r])
            return binding.shard_combine(stats, y, mk, -100, ws=cws)

        def bwd(x, m, logs):
            H, W, b, y, mk = x
            for r, (v0, n) in enumerate(bounds):
                binding.shard_backward(H, W[v0:v0 + n], None if b is None else b[v0:v0 + n], y,
                                       mk, -100, m, logs, v0=v0, V_total=inp.V, lam=inp.lam,
                                       ws=ws, accumulate_dh=r > 0,
                                       panel_backward=args.panel_backward,
                                       out=(dH, dW[v0:v0 + n],
                                            None if db is None else db[v0:v0 + n]))
    else:
        def fwd(x):
            H, W, b, y, mk = x
            return binding.forward(H, W, b, y, mk, -100, ws=ws)

        def bwd(x, m, logs):
            H, W, b, y, mk = x
            # the forward's compaction and gathered rows are still in ws
            binding.backward(H, W, b, y, mk, -100, m, logs, lam=inp.lam, ws=ws,
                             out=(dH, dW, db), reuse_forward=True, filter_eps=args.filter_eps,
                             panel_backward=args.panel_backward)

    inputs = (H, W, b, y, mk)

    def step(x=inputs):
        loss, m, logs = fwd(x)
        bwd(x, m, logs)
        return loss

    def device_status():
        st = binding.device_status(ws)
        return st if st != 0 or P == 1 else binding.device_status(cws)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    n_warm = max(args.warmup, 3)
    for _ in range(n_warm):
        step()
    torch.cuda.synchronize(dev)
    st = device_status()
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {binding.status_string(st)}")

    sampler = ClockSampler(str(torch.cuda.get_device_properties(dev).uuid))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    binding.profile_begin()
    for k in range(args.steps):
        e0, e1, e2 = evs[k]
        e0.record(stream)
        loss, m, logs = fwd(inputs)
        e1.record(stream)
        bwd(inputs, m, logs)
        e2.record(stream)
    torch.cuda.synchronize(dev)
    prof = binding.profile_end()
    barrier()
    clocks = sampler.stop()
    st = device_status()
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {binding.status_string(st)}")
    total_ms = evs[0][0].elapsed_time(evs[-1][2])
    fwd_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    value = weak_scaling_tflops(flop_step, args.steps, total_ms, world)
    peak_mib = torch.cuda.max_memory_allocated(dev) / 2**20
    launches = sum(n for _, n in prof.values())
    # The library allocates no device memory: every buffer of the step is one
    # of these.  None may be the size of the N x V logits in 16 bits (checked
    # where that size is what the method avoids: 1 GiB and up).
    bufs = [t for t in (H, W, b, y, mk, dH, dW, db) if t is not None] + [ws.buf]
    largest = max(t.numel() * t.element_size() for t in bufs)
    logits_bytes = inp.N * inp.V * 2
    if logits_bytes >= 2**30 and largest >= logits_bytes:
        raise RuntimeError(f"a {largest} B buffer is as large as the {logits_bytes} B logits")

    # e2e: every step's inputs copied from pinned host memory and its loss read
    # back, all inside the timed region.  The inputs of step k+1 are copied on
    # a second stream into the other of two device buffer sets while step k
    # computes (as a data loader would); a step waits for its own copy only.
    e2e = None
    if not args.no_e2e:
        host = tuple(None if t is None else t.cpu().pin_memory() for t in inputs)
        bufs = (inputs, tuple(None if t is None else torch.empty_like(t) for t in inputs))
        loss_host = torch.empty((), dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host if t is not None)
        copy_stream = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        freed = [torch.cuda.Event() for _ in range(2)]

        def copy_in(k):
            j = k % 2
            with torch.cuda.stream(copy_stream):
                if k >= 2:
                    copy_stream.wait_event(freed[j])  # step k-2 is done with buffer j
                for d, h in zip(bufs[j], host):
                    if d is not None:
                        d.copy_(h, non_blocking=True)
                copied[j].record(copy_stream)

        barrier()
        torch.cuda.synchronize(dev)
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        copy_stream.wait_event(s0)
        copy_in(0)
        for k in range(args.steps):
            if k + 1 < args.steps:
                copy_in(k + 1)
            stream.wait_event(copied[k % 2])
            loss = step(bufs[k % 2])
            freed[k % 2].record(stream)
            loss_host.copy_(loss, non_blocking=True)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(s0.elapsed_time(s1), dev)
        e2e = {"value": weak_scaling_tflops(flop_step, args.steps, e2e_ms, world),
               "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": 4,
               "loss": float(loss_host.item()),
               "note": "inputs double-buffered: step k+1's host-to-device copy overlaps step k; "
                       "the loss is read back every step, the gradients dH, dW (db) stay on "
                       "the device for an on-device optimizer step"}

        # The same through the nn.Module a training loop calls
        # (binding.LinearCrossEntropyLoss + loss.backward(): autograd, one
        # workspace for both passes, gradients cast to the parameters' dtype).
        crit = binding.LinearCrossEntropyLoss(ignore_index=-100)

        def module_step(x):
            Hb, Wb, bb, yb, mb = x
            Hp = Hb.detach().requires_grad_(True)
            Wp = Wb.detach().requires_grad_(True)
            bp = None if bb is None else bb.detach().requires_grad_(True)
            loss = crit(Hp, yb, Wp, bias=bp, mask=mb)
            (loss * inp.lam).backward()
            return loss.detach()

        for _ in range(2):  # untimed: the allocator's first blocks for this path
            module_step(inputs)
        barrier()
        torch.cuda.synchronize(dev)
        s0.record(stream)
        copy_stream.wait_event(s0)
        copy_in(0)
        for k in range(args.steps):
            if k + 1 < args.steps:
                copy_in(k + 1)
            stream.wait_event(copied[k % 2])
            loss = module_step(bufs[k % 2])
            freed[k % 2].record(stream)
            loss_host.copy_(loss, non_blocking=True)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        mod_ms = max_over_ranks(s0.elapsed_time(s1), dev)
        e2e["module"] = {"value": weak_scaling_tflops(flop_step, args.steps, mod_ms, world),
                         "unit": UNIT, "loss": float(loss_host.item()),
                         "note": "LinearCrossEntropyLoss forward + loss.backward(), the same "
                                 "host-to-device copies; includes autograd and the casts of "
                                 "dH, dW to the parameters' dtype (torch kernels)"}

    # roofline of the dominant kernel (largest share of device time)
    peaks, peak_src = load_peaks()
    flop_per_step = {"fwd_gemm": 2.0 * C * inp.D * inp.V,   # algorithmic FLOP per step
                     "bwd_gemm": 6.0 * C * inp.D * inp.V}
    # algorithmic DRAM bytes per step: inputs read once and outputs written once
    # (16-bit W and H_c, fp32 dW and dH); the forward reads W and H_c, the
    # backward reads W and H_c again and writes dW and dH.
    esz = 2
    in_w = inp.V * inp.D * esz
    in_hc = C * inp.D * esz
    bytes_per_step = {"fwd_gemm": float(in_w + in_hc),
                      "bwd_gemm": float(in_w + in_hc + inp.V * inp.D * 4 + inp.N * inp.D * 4)}
    dom = max(flop_per_step, key=lambda k: prof[k][0])
    ms_tot, n_l = prof[dom]
    avg_ms = ms_tot / max(n_l, 1)
    flop_per_launch = flop_per_step[dom] * args.steps / max(n_l, 1)
    achieved = flop_per_launch / (avg_ms * 1e-3) / 1e12
    # The timed region is well under a second (tens of ms per step), so the
    # burst figure is the roofline; the sustained one is printed beside it.
    # fp16 and bf16 share the dense tensor-core rate on this part.
    peak = peaks.get("bf16_tflops")
    peak_sus = peaks.get("bf16_tflops_sustained")
    tb = ncu_traffic(dom, spec.name) if not cfg.get("backward", "").startswith("single") else None
    alg_launch = bytes_per_step[dom] * args.steps / max(n_l, 1)
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_note": f"burst dense bf16, {peak_src} (sub-second timed region)",
                "frac_sustained": achieved / peak_sus,
                "traffic": tb, "algorithmic_bytes": alg_launch,
                "traffic_over_algorithmic": (tb / alg_launch) if tb else None,
                "algorithmic_bytes_per_step": bytes_per_step["fwd_gemm"] +
                bytes_per_step["bwd_gemm"],
                "flop_per_launch": flop_per_launch, "avg_launch_ms": avg_ms,
                "launches": n_l,
                "kernel_share": {k: round(v[0] / max(1e-9, sum(x[0] for x in prof.values())), 4)
                                 for k, v in prof.items()}}

    burst = peaks.get("bf16_tflops")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": n_warm, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": spec.dtype, "data": "synthetic",
            "config": cfg, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
            "fwd_tflops": 2.0 * C * inp.D * inp.V / (fwd_ms * 1e-3) / 1e12,
            "bwd_tflops": 6.0 * C * inp.D * inp.V / (bwd_ms * 1e-3) / 1e12,
            "pct_bf16_peak": 100.0 * (value / world) / burst,
            "pct_bf16_peak_sustained": 100.0 * (value / world) / peaks.get(
                "bf16_tflops_sustained"),
            "peak_note": f"bf16 peak {burst} TFLOP/s burst, {peak_src}",
            "peak_mib": peak_mib, "input_mib": in_mib,
            "logits_mib_avoided": inp.N * inp.V * 2 / 2**20, "largest_alloc_mib": largest / 2**20,
            "clocks": clocks, "e2e": e2e, "gpu_launches": launches,
            "roofline": roofline, "cpu_baseline": cpu_baseline}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
