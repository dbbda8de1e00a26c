#!/usr/bin/env python
"""Benchmark of the fused HAD attention forward pass (tokens/s).

One step = one ``had_attention_fwd`` call over one batch of the long-context
workload (B=4, H=16, n=4096, d=64, N=512, bf16; tau = 1/8), inputs resident
in HBM.  Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl had|reference]

N > 1 runs under torchrun, one process per GPU; every rank processes its own
batch of independent (b, h) problems (weak scaling, no collective on the data
path) and the timing is the max over ranks.  ``--impl reference`` times the
CPU oracle (the only reference this method has) on bounded row samples of the
same workload, on rank 0 only.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "long"
L2_FLUSH_BYTES = 256 << 20
SM_COUNT = 148
ALU_LANES_PER_SM = 128


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["had", "reference"], default="had")
    ap.add_argument("--config", default=WORKLOAD, choices=sorted(synth.CONFIGS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-settle", action="store_true",
                    help="skip the timed-loop warm-up of the clocks (for profiler captures, "
                         "whose launch counts must be fixed; numbers taken under a profiler "
                         "are not reported)")
    ap.add_argument("--mode", choices=["attention", "unfused", "mass", "causal", "soft", "bwd"],
                    default="attention",
                    help="attention: the forward (the default line); unfused: the four-call "
                         "composition (binarize, top-N, softmax-V) stage by stage; mass: the "
                         "top-N mass-retention diagnostic; causal: the causal forward; soft: "
                         "the soft-code (tanh) forward; bwd: forward + straight-through backward")
    return ap.parse_args()


def metric_name(cfg):
    """The headline metric, named for the workload it is measured on."""
    return (f"HAD attention tokens/sec at n={cfg.n},d={cfg.d},N={cfg.N}; "
            f"% of int8-TC/HBM roofline")


# --------------------------------------------------------------------------- peaks


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "sm_max_mhz": float(p.get("sm_max_mhz", 1965.0)), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


def roofline_model(cfg, peaks):
    """Algorithmic work of one call and its roofline time.

    work   = 2*B*H*n^2*d (int8 logit ops, counted once) + 2*B*H*n*N*d (AV flops)
    T_roof = max(T_HBM, T_TC, T_ALU):
      T_HBM = (3*B*H*n*d*2 + B*H*n*d*4) bytes / HBM bandwidth   (read Q,K,V; write O)
      T_TC  = logit ops / int8 peak + AV flops / bf16 peak, int8 peak = 2 x bf16 peak
      T_ALU = B*H*n^2 logits / (SMs * 128 lanes * max SM clock), one op per logit
    """
    B, H, n, d, N = cfg.B, cfg.H, cfg.n, cfg.d, cfg.N
    elt = 2 if cfg.dtype == "bf16" else 4
    logit_ops = 2.0 * B * H * n * n * d
    av_flops = 2.0 * B * H * n * N * d
    hbm_bytes = 3.0 * B * H * n * d * elt + B * H * n * d * 4
    bf16 = peaks["bf16_tflops"] * 1e12
    i8 = 2.0 * bf16
    t_hbm = hbm_bytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = logit_ops / i8 + av_flops / bf16
    alu = SM_COUNT * ALU_LANES_PER_SM * peaks["sm_max_mhz"] * 1e6
    t_alu = B * H * n * n / alu
    return {"work": logit_ops + av_flops, "hbm_bytes": hbm_bytes, "t_hbm": t_hbm,
            "t_tc": t_tc, "t_alu": t_alu, "t_roof": max(t_hbm, t_tc, t_alu)}


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        mhz, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                maxs.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(mhz)}


# --------------------------------------------------------------------------- dist


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "had" else "gloo"
        if args.impl == "had":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value, world, device):
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(tokens_per_rank, ms_local, world, device):
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    ms = max_over_ranks(ms_local, world, device)
    return tokens_per_rank * world / (ms * 1e-3), ms


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------------- oracle


def oracle_baseline(cfg, target_seconds, steps=1):
    """Time the CPU oracle on bounded row samples; returns (tokens/s, details)."""
    import numpy as np
    import oracle
    q, k, v, sgq, sgk = synth.make_inputs(cfg)
    t0 = time.time()
    sq = oracle.binarize(synth.to_oracle_array(q), sgq.numpy())
    sk = oracle.binarize(synth.to_oracle_array(k), sgk.numpy())
    t_bin = time.time() - t0
    vo = synth.to_oracle_array(v)
    threads = oracle.max_threads()
    probe = np.arange(0, cfg.rows, max(1, cfg.rows // 64))[:64]
    t0 = time.time()
    oracle.attention_rows(sq, sk, vo, cfg.tau, cfg.N, probe, threads=threads)
    per_row = (time.time() - t0) / len(probe)
    count = int(max(64, min(cfg.rows, target_seconds / max(per_row, 1e-9))))
    times, rows_done = [], 0
    for s in range(steps):
        rows = synth.sample_rows(cfg, count, seed=100 + s)
        t0 = time.time()
        oracle.attention_rows(sq, sk, vo, cfg.tau, cfg.N, rows, threads=threads)
        times.append(time.time() - t0)
        rows_done += len(rows)
    total = sum(times)
    # binarizing the whole tensors once is part of the work; charge it pro rata
    total += t_bin * rows_done / cfg.rows
    tokens = rows_done / cfg.H
    return tokens / total, {
        "cores": threads,
        "sample": (f"{rows_done} query rows (of {cfg.rows}) of the {cfg.name} workload over "
                   f"{steps} step(s), all heads; plus whole-tensor binarization pro rata; "
                   f"tokens = rows / H"),
        "seconds": total,
    }


def run_reference(args, world, rank):
    cfg = synth.CONFIGS[args.config]
    if rank != 0:
        return
    steps = max(1, args.steps)
    per_step = max(1.0, min(args.cpu_seconds, 150.0 / (steps + args.warmup)))
    if args.warmup:
        oracle_baseline(cfg, per_step * 0.2, steps=1)
    value, info = oracle_baseline(cfg, per_step, steps=steps)
    line = {
        "impl": "reference", "metric": metric_name(cfg), "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
        "ms_per_step": info["seconds"] * 1e3 / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int32+f64", "data": "synthetic",
        "config": {"workload": cfg.describe(), "B": cfg.B, "H": cfg.H, "seq_len": cfg.n,
                   "d": cfg.d, "N": cfg.N, "parallelism": "rank 0 only (CPU oracle)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": info["cores"],
                         "kind": "oracle", "sample": info["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- had


def source_digest():
    """sha256 of the fused path's sources: its kernels, the helpers they
    include and its launch code (ties stored ncu counters to a build)."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_attention_sigma_b200", "csrc")
    for name in ("had_fwd_tc.cuh", "had_fused.cuh", "had_tc.cuh", "had_prep.cuh",
                 "had_pack.cuh", "had_common.cuh", "had_fwd_launch.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def fused_kernel_name(cfg):
    """The fused kernel had_attention_core runs for this workload (no debug outputs)."""
    return "attention_tc_kernel"


def stored_traffic(cfg):
    """DRAM bytes per launch of the fused kernel from the committed ncu summary,
    or None when the summary belongs to other sources or another workload."""
    path = os.path.join(ROOT, "profiles", f"{fused_kernel_name(cfg)}_{cfg.name}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    if fields.get("source_sha256") != source_digest():
        return None
    try:
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def run_had(args, world, rank, local):
    from sparse_attention_sigma_b200 import had
    cfg = synth.CONFIGS[args.config]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    model = roofline_model(cfg, peaks)

    q, k, v, sgq, sgk = synth.make_inputs(cfg)
    gq, gk, gv = q.to(dev), k.to(dev), v.to(dev)
    gsq, gsk = sgq.to(dev), sgk.to(dev)
    out = torch.empty((cfg.B, cfg.H, cfg.n, cfg.d), dtype=torch.float32, device=dev)
    ws = had.workspace(cfg.B, cfg.H, cfg.n, cfg.d, cfg.N, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    launches = (had.had_launch_count(had.HAD_OP_ATTENTION_PREPARE, cfg.B, cfg.H, cfg.n, cfg.d,
                                     cfg.N) +
                had.had_launch_count(had.HAD_OP_ATTENTION_CORE, cfg.B, cfg.H, cfg.n, cfg.d,
                                     cfg.N))

    # One step is had_attention_fwd, issued as its two stages so that the
    # dominant stage (the fused kernel and its fix-up) has its own events.
    def prepare():
        had.had_attention_prepare(gq, gk, gv, gsq, gsk, cfg.N, ws)

    def core():
        had.had_attention_core(gv, cfg.N, cfg.tau, ws, out=out)

    for _ in range(max(3, args.warmup)):
        prepare()
        core()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    t_end = time.time() + (0.0 if args.no_settle else 1.5)   # clocks settle under load first
    while time.time() < t_end:
        for _ in range(20):
            prepare()
            core()
        torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))                 # evict L2 between steps (outside the events)
        ev[i][0].record(stream)
        prepare()
        ev[i][1].record(stream)
        core()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clock_info = clocks.stop()
    if clock_info is not None:
        clock_info["window"] = "1.5 s of back-to-back calls ending with the timed steps"
    ms_local = sum(e[0].elapsed_time(e[2]) for e in ev) / args.steps
    core_local = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    value, ms = aggregate(cfg.tokens, ms_local, world, dev)
    core_ms = max_over_ranks(core_local, world, dev)

    achieved = model["work"] / (core_ms * 1e-3) / 1e12
    peak_eff = model["work"] / model["t_roof"] / 1e12
    traffic = stored_traffic(cfg)
    misses = had.had_attention_window_misses(ws, cfg.B, cfg.H, cfg.n, cfg.d, cfg.N)
    core_med = max_over_ranks(statistics.median(e[1].elapsed_time(e[2]) for e in ev), world, dev)
    ms_med = max_over_ranks(statistics.median(e[0].elapsed_time(e[2]) for e in ev), world, dev)

    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(had, cfg, q, k, v, gsq, gsk, ws, dev, max(3, args.steps // 2), world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, info = oracle_baseline(cfg, args.cpu_seconds)
        cpu = {"value": val, "unit": "tokens/s", "cores": info["cores"], "kind": "oracle",
               "sample": info["sample"]}

    if rank != 0:
        return
    line = {
        "metric": metric_name(cfg), "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.describe(), "B": cfg.B, "H": cfg.H, "seq_len": cfg.n,
                   "d": cfg.d, "N": cfg.N, "global_batch": cfg.B * world,
                   "parallelism": f"weak: {world} rank(s), one batch of independent heads each",
                   "l2": "flushed between steps (256 MiB write outside the timed events)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_eff,
                     "unit": "TFLOP/s", "frac": achieved / peak_eff, "traffic": traffic,
                     "kernel": f"had_attention_core: {fused_kernel_name(cfg)} + fixup_rows_kernel",
                     "core_ms": core_ms, "core_ms_median": core_med, "ms_median": ms_med,
                     "whole_call_frac": model["t_roof"] / (ms * 1e-3),
                     "t_roof_us": model["t_roof"] * 1e6, "t_hbm_us": model["t_hbm"] * 1e6,
                     "t_tc_us": model["t_tc"] * 1e6, "t_alu_us": model["t_alu"] * 1e6,
                     "peaks": peaks["source"]},
        "gpu_launches": launches * args.steps,
        "window_misses": {"rows": misses, "of": cfg.B * cfg.H * cfg.n,
                          "note": "rows the exact fix-up kernel recomputed in the last step"},
        "clocks": clock_info,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def end_to_end(had, cfg, q, k, v, gsq, gsk, ws, dev, steps, world):
    """Same call with inputs copied from pinned host memory and O copied back.

    Every step copies its Q, K, V host -> device, runs had_attention_fwd and
    copies its O device -> host.  Steps are pipelined the way a serving loop
    would run them: two sets of device buffers, the upload of step i + 1 on
    one stream, the compute of step i on another and the download of step
    i - 1 on a third, ordered by events.  The timed region runs from before
    the first upload to after the last download.
    """
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    ho = [torch.empty((cfg.B, cfg.H, cfg.n, cfg.d), dtype=torch.float32).pin_memory()
          for _ in range(2)]
    bufs = []
    for i in range(2):
        bufs.append({"q": torch.empty_like(q, device=dev), "k": torch.empty_like(k, device=dev),
                     "v": torch.empty_like(v, device=dev),
                     "out": torch.empty(ho[0].shape, dtype=torch.float32, device=dev),
                     "ws": ws if i == 0 else had.workspace(cfg.B, cfg.H, cfg.n, cfg.d, cfg.N,
                                                         device=dev)})
    s_up, s_comp, s_down = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev = lambda: torch.cuda.Event(enable_timing=False)
    up_done = [ev(), ev()]
    comp_done = [ev(), ev()]
    down_done = [ev(), ev()]
    used = [False, False]

    def step(i):
        b, h = bufs[i % 2], ho[i % 2]
        with torch.cuda.stream(s_up):
            if used[i % 2]:
                s_up.wait_event(comp_done[i % 2])     # the compute of step i - 2 read them
            b["q"].copy_(hq, non_blocking=True)
            b["k"].copy_(hk, non_blocking=True)
            b["v"].copy_(hv, non_blocking=True)
            up_done[i % 2].record(s_up)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(up_done[i % 2])
            if used[i % 2]:
                s_comp.wait_event(down_done[i % 2])   # out of step i - 2 is on the host
            had.had_attention_fwd(b["q"], b["k"], b["v"], gsq, gsk, cfg.N, cfg.tau,
                                  out=b["out"], ws=b["ws"], stream=s_comp)
            comp_done[i % 2].record(s_comp)
        with torch.cuda.stream(s_down):
            s_down.wait_event(comp_done[i % 2])
            h.copy_(b["out"], non_blocking=True)
            down_done[i % 2].record(s_down)
        used[i % 2] = True

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    barrier(world)
    s.record(s_up)
    for i in range(steps):
        step(i)
    for st in (s_up, s_comp):
        s_down.wait_stream(st)
    e.record(s_down)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e) / steps, world, dev)
    h2d = (q.numel() + k.numel() + v.numel()) * q.element_size()
    return {"value": cfg.tokens * world / (ms * 1e-3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": ho[0].numel() * 4,
            "ms_per_step": ms,
            "pipelining": "two buffer sets; upload, compute and download on three streams"}


def run_unfused(args, world, rank, local):
    """The four-call composition of the forward (had_binarize_pack on Q and
    K, had_hamming_topn, had_sparse_softmax_av) timed stage by stage, each
    against its own roofline:
      pack   HBM: read Q and K, write their packed bits;
      top-N  popcount pipe: two passes of d/32 popcounts per (query, key)
             pair at 16 popcounts per clock per SM;
      AV     HBM: read the kept set (6 B per kept pair) and V, write O.
    The value is tokens per second of the three stages together."""
    from sparse_attention_sigma_b200 import had
    cfg = synth.CONFIGS[args.config]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    q, k, v, sgq, sgk = synth.make_inputs(cfg)
    gq, gk, gv = q.to(dev), k.to(dev), v.to(dev)
    gsq, gsk = sgq.to(dev), sgk.to(dev)
    shape = (cfg.B, cfg.H, cfg.n)
    qb = torch.empty(shape + (cfg.d // 32,), dtype=torch.int32, device=dev)
    kb = torch.empty_like(qb)
    idx = torch.empty(shape + (cfg.N,), dtype=torch.int32, device=dev)
    lg = torch.empty(shape + (cfg.N,), dtype=torch.int16, device=dev)
    out = torch.empty(shape + (cfg.d,), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def stages():
        had.had_binarize_pack(gq, gsq, bits=qb)
        had.had_binarize_pack(gk, gsk, bits=kb)
        yield
        had.had_hamming_topn(qb, kb, cfg.d, cfg.N, idx=idx, logits=lg)
        yield
        had.had_sparse_softmax_av(idx, lg, gv, cfg.tau, out=out)
        yield

    for _ in range(max(3, args.warmup)):
        for _ in stages():
            pass
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))
        ev[i][0].record(stream)
        for j, _ in enumerate(stages()):
            ev[i][j + 1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clock_info = clocks.stop()
    per = [[e[j].elapsed_time(e[j + 1]) for e in ev] for j in range(3)]
    stage_ms = [max_over_ranks(statistics.median(x), world, dev) for x in per]
    value, ms = aggregate(cfg.tokens, sum(sum(x) for x in per) / args.steps, world, dev)
    B, H, n, d, N = cfg.B, cfg.H, cfg.n, cfg.d, cfg.N
    elt = 2 if cfg.dtype == "bf16" else 4
    hbm = peaks["hbm_gbs"] * 1e9
    pack_bytes = 2.0 * B * H * n * d * (elt + 1.0 / 8)
    popc = 2.0 * B * H * n * n * (d // 32)
    popc_peak = SM_COUNT * 16 * peaks["sm_max_mhz"] * 1e6
    av_bytes = B * H * n * (6.0 * N + d * elt + d * 4)
    frac = lambda work, t_ms, peak: work / (t_ms * 1e-3) / peak
    if rank != 0:
        return
    print(json.dumps({
        "metric": "HAD unfused forward (binarize, top-N, softmax-V) tokens/sec", "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "impl": "had_binarize_pack x2 + had_hamming_topn + had_sparse_softmax_av",
        "config": {"workload": cfg.describe(),
                   "l2": "flushed between steps (256 MiB write outside the timed events)"},
        "stage_ms_median": {"binarize_pack_qk": stage_ms[0], "hamming_topn": stage_ms[1],
                            "sparse_softmax_av": stage_ms[2]},
        "stage_roofline": {
            "binarize_pack_qk": {"bound": "hbm", "bytes": pack_bytes, "unit": "GB/s",
                                 "achieved": pack_bytes / (stage_ms[0] * 1e-3) / 1e9,
                                 "peak": peaks["hbm_gbs"],
                                 "frac": frac(pack_bytes, stage_ms[0], hbm)},
            "hamming_topn": {"bound": "alu (popcount pipe)", "popc": popc, "unit": "Tpopc/s",
                             "achieved": popc / (stage_ms[1] * 1e-3) / 1e12,
                             "peak": popc_peak / 1e12,
                             "frac": frac(popc, stage_ms[1], popc_peak)},
            "sparse_softmax_av": {"bound": "hbm", "bytes": av_bytes, "unit": "GB/s",
                                  "achieved": av_bytes / (stage_ms[2] * 1e-3) / 1e9,
                                  "peak": peaks["hbm_gbs"],
                                  "frac": frac(av_bytes, stage_ms[2], hbm)},
            "peaks": peaks["source"]},
        "gpu_launches": 4 * args.steps,
        "clocks": clock_info,
    }), flush=True)


def run_mass(args, world, rank, local):
    """The top-N mass-retention diagnostic (had_topn_mass) on the workload's
    binarized Q and K: rows per second, against the popcount roofline of its
    histogram pass (d/32 popcounts per (query, key) pair at 16 per clock per
    SM)."""
    from sparse_attention_sigma_b200 import had
    cfg = synth.CONFIGS[args.config]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q, k, _, sgq, sgk = synth.make_inputs(cfg)
    qb = had.had_binarize_pack(q.to(dev), sgq.to(dev))
    kb = had.had_binarize_pack(k.to(dev), sgk.to(dev))
    p = [0.9, 0.95, 0.99]
    nmin = torch.empty((cfg.B, cfg.H, cfg.n, len(p)), dtype=torch.int32, device=dev)
    step = lambda: had.had_topn_mass(qb, kb, cfg.d, cfg.tau, p, nmin=nmin)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    barrier(world)
    s.record()
    for _ in range(args.steps):
        step()
    e.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e) / args.steps, world, dev)
    rows = cfg.B * cfg.H * cfg.n * world
    popc = cfg.B * cfg.H * cfg.n * cfg.n * (cfg.d // 32) * world
    peak = SM_COUNT * 16 * 1.965e9 * world
    med = nmin.reshape(-1, len(p)).float().median(dim=0).values.tolist()
    if rank == 0:
        print(json.dumps({
            "metric": "top-N mass-retention diagnostic rows/sec", "value": rows / (ms * 1e-3),
            "unit": "rows/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "dtype": "u32/f64",
            "data": "synthetic", "impl": "had_topn_mass",
            "config": {"workload": cfg.describe(),
                       "p": p},
            "median_nmin": dict(zip([str(x) for x in p], med)),
            "roofline": {"bound": "alu", "achieved": popc / (ms * 1e-3) / 1e12,
                         "peak": peak / 1e12, "unit": "Tpopc/s",
                         "frac": popc / (ms * 1e-3) / peak,
                         "note": "popcount pipe, 16/clk/SM at 1.965 GHz"},
            "gpu_launches": args.steps,
        }), flush=True)


def run_causal(args, world, rank, local):
    """The causal forward: had_attention_causal_fwd (the fused tensor-core
    path, each CTA streaming keys only up to its last row) timed as the
    value, and the unfused composition (binarize, causal top-N, softmax-V)
    timed stage by stage beside it.  Roofline as the non-causal call with the
    causal work: n (n + 1) / 2 visible pairs a head, sum_i min(N, i + 1) kept
    pairs."""
    from sparse_attention_sigma_b200 import had
    cfg = synth.CONFIGS[args.config]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    q, k, v, sgq, sgk = synth.make_inputs(cfg)
    gq, gk, gv = q.to(dev), k.to(dev), v.to(dev)
    gsq, gsk = sgq.to(dev), sgk.to(dev)
    shape = (cfg.B, cfg.H, cfg.n)
    qb = torch.empty(shape + (cfg.d // 32,), dtype=torch.int32, device=dev)
    kb = torch.empty_like(qb)
    idx = torch.empty(shape + (cfg.N,), dtype=torch.int32, device=dev)
    lg = torch.empty(shape + (cfg.N,), dtype=torch.int16, device=dev)
    out = torch.empty(shape + (cfg.d,), dtype=torch.float32, device=dev)
    out_u = torch.empty_like(out)
    ws = torch.empty(had.had_workspace_bytes(had.HAD_OP_ATTENTION_CAUSAL, cfg.B, cfg.H, cfg.n,
                                             cfg.d, cfg.N), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    launches = had.had_launch_count(had.HAD_OP_ATTENTION_CAUSAL, cfg.B, cfg.H, cfg.n, cfg.d,
                                    cfg.N)

    def fused():
        had.had_attention_causal_fwd(gq, gk, gv, gsq, gsk, cfg.N, cfg.tau, out=out, ws=ws)

    def stages():
        had.had_binarize_pack(gq, gsq, bits=qb)
        had.had_binarize_pack(gk, gsk, bits=kb)
        yield
        had.had_hamming_topn_causal(qb, kb, cfg.d, cfg.N, idx=idx, logits=lg)
        yield
        had.had_sparse_softmax_av(idx, lg, gv, cfg.tau, out=out_u)
        yield

    for _ in range(max(3, args.warmup)):
        fused()
        for _ in stages():
            pass
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    t_end = time.time() + (0.0 if args.no_settle else 1.0)   # clocks settle under load first
    while time.time() < t_end:
        for _ in range(10):
            fused()
        torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))
        ev[i][0].record(stream)
        fused()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clock_info = clocks.stop()
    fused_local = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    value, ms = aggregate(cfg.tokens, fused_local, world, dev)

    usteps = max(1, min(args.steps, 5))
    uev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(usteps)]
    for i in range(usteps):
        flush.fill_(float(i))
        uev[i][0].record(stream)
        for j, _ in enumerate(stages()):
            uev[i][j + 1].record(stream)
    torch.cuda.synchronize()
    stage_ms = [sum(e[j].elapsed_time(e[j + 1]) for e in uev) / usteps for j in range(3)]

    B, H, n, d, N = cfg.B, cfg.H, cfg.n, cfg.d, cfg.N
    pairs = B * H * n * (n + 1) / 2
    kept = B * H * (min(N, n) * (min(N, n) + 1) / 2 + max(n - N, 0) * N)
    bf16 = peaks["bf16_tflops"] * 1e12
    elt = 2 if cfg.dtype == "bf16" else 4
    t_hbm = (3.0 * B * H * n * d * elt + B * H * n * d * 4) / (peaks["hbm_gbs"] * 1e9)
    t_tc = 2.0 * pairs * d / (2 * bf16) + 2.0 * kept * d / bf16
    t_alu = pairs / (SM_COUNT * 128 * peaks["sm_max_mhz"] * 1e6)
    t_roof = max(t_hbm, t_tc, t_alu)
    work = 2.0 * pairs * d + 2.0 * kept * d
    if rank != 0:
        return
    print(json.dumps({
        "metric": "HAD causal attention tokens/sec", "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic", "impl": "had_attention_causal_fwd (fused)",
        "config": {"workload": cfg.describe(), "causal": True,
                   "l2": "flushed between steps (256 MiB write outside the timed events)"},
        "unfused_stage_ms": {"binarize_pack": stage_ms[0], "hamming_topn_causal": stage_ms[1],
                             "sparse_softmax_av": stage_ms[2]},
        "roofline": {"bound": "tensor", "achieved": work / (ms * 1e-3) / 1e12,
                     "peak": work / t_roof / 1e12, "unit": "TFLOP/s",
                     "frac": t_roof / (ms * 1e-3), "traffic": None,
                     "kernel": "whole call: prep + attention_fwd_kernel<causal> + fix-up",
                     "t_roof_us": t_roof * 1e6, "t_hbm_us": t_hbm * 1e6, "t_tc_us": t_tc * 1e6,
                     "t_alu_us": t_alu * 1e6, "peaks": peaks["source"]},
        "gpu_launches": launches * args.steps,
        "clocks": clock_info,
    }), flush=True)


def run_soft(args, world, rank, local):
    """The soft-code forward (had_soft_attention_fwd, tanh training stages) on
    the workload with c = 1: tokens per second, issued as its three stages.
    The top-N stage is dominated by the fp32 logit kernel (2 d flops per
    (query, key) pair on the CUDA cores); its roofline is the FMA pipe."""
    from sparse_attention_sigma_b200 import had
    cfg = synth.CONFIGS[args.config]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    c = 1.0
    q, k, v, sgq, sgk = synth.make_inputs(cfg)
    gq, gk, gv = q.to(dev), k.to(dev), v.to(dev)
    gsq, gsk = sgq.to(dev), sgk.to(dev)
    shape = (cfg.B, cfg.H, cfg.n)
    tq = torch.empty(shape + (cfg.d,), dtype=torch.float32, device=dev)
    tk = torch.empty_like(tq)
    idx = torch.empty(shape + (cfg.N,), dtype=torch.int32, device=dev)
    lg = torch.empty(shape + (cfg.N,), dtype=torch.float32, device=dev)
    out = torch.empty(shape + (cfg.d,), dtype=torch.float32, device=dev)
    ws = torch.empty(had.had_workspace_bytes(had.HAD_OP_SOFT_TOPN, cfg.B, cfg.H, cfg.n, cfg.d,
                                             cfg.N), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    launches = (2 + had.had_launch_count(had.HAD_OP_SOFT_TOPN, cfg.B, cfg.H, cfg.n, cfg.d, cfg.N)
                + 1)

    def stages():
        had.had_soft_binarize(gq, gsq, c, t=tq)
        had.had_soft_binarize(gk, gsk, c, t=tk)
        yield
        had.had_soft_topn(tq, tk, cfg.N, idx=idx, logits=lg, ws=ws)
        yield
        had.had_soft_softmax_av(idx, lg, gv, cfg.tau, out=out)
        yield

    for _ in range(max(3, args.warmup)):
        for _ in stages():
            pass
    ref = had.had_soft_attention_fwd(gq, gk, gv, gsq, gsk, c, cfg.N, cfg.tau)
    torch.cuda.synchronize()
    if not torch.equal(ref, out):
        raise RuntimeError("had_soft_attention_fwd differs from its three stages")
    del ref
    clocks = ClockSampler(local)
    clocks.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))
        ev[i][0].record(stream)
        for j, _ in enumerate(stages()):
            ev[i][j + 1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clock_info = clocks.stop()
    stage_ms = [sum(e[j].elapsed_time(e[j + 1]) for e in ev) / args.steps for j in range(3)]
    value, ms = aggregate(cfg.tokens, sum(stage_ms), world, dev)
    topn_ms = max_over_ranks(stage_ms[1], world, dev)
    flops = 2.0 * cfg.B * cfg.H * cfg.n * cfg.n * cfg.d
    peak = SM_COUNT * 128 * 2 * 1.965e9
    if rank != 0:
        return
    print(json.dumps({
        "metric": "HAD soft-code (tanh) attention tokens/sec", "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "impl": "had_soft_attention_fwd",
        "config": {"workload": cfg.describe(), "c": c,
                   "l2": "flushed between steps (256 MiB write outside the timed events)"},
        "stage_ms": {"soft_binarize": stage_ms[0], "soft_topn": stage_ms[1],
                     "soft_softmax_av": stage_ms[2]},
        "roofline": {"bound": "alu", "achieved": flops / (topn_ms * 1e-3) / 1e12,
                     "peak": peak / 1e12, "unit": "TFLOP/s", "frac": flops / (topn_ms * 1e-3) / peak,
                     "kernel": "had_soft_topn stage: soft_logits_kernel + soft_select_kernel",
                     "note": "fp32 FMA pipe, 128 lanes/SM at 1.965 GHz; 2 d flops per "
                             "(query, key) pair of the logits"},
        "gpu_launches": launches * args.steps,
        "clocks": clock_info,
    }), flush=True)


def run_bwd(args, world, rank, local):
    """One step of the straight-through training stage on the workload: the
    fused forward (keeping its kept set) and had_attention_bwd on that set.
    Tokens per second of the pair; each half has its own events.  The
    roofline is the backward's algorithmic HBM traffic: Q, K, V read, dO
    read, dQ, dK, dV written, and the kept set (6 B per kept pair) read."""
    from sparse_attention_sigma_b200 import had
    cfg = synth.CONFIGS[args.config]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    q, k, v, sgq, sgk = synth.make_inputs(cfg)
    gq, gk, gv = q.to(dev), k.to(dev), v.to(dev)
    gsq, gsk = sgq.to(dev), sgk.to(dev)
    shape = (cfg.B, cfg.H, cfg.n)
    dout = torch.randn(shape + (cfg.d,), generator=torch.Generator().manual_seed(5)).to(dev)
    out = torch.empty(shape + (cfg.d,), dtype=torch.float32, device=dev)
    idx = torch.empty(shape + (cfg.N,), dtype=torch.int32, device=dev)
    lg = torch.empty(shape + (cfg.N,), dtype=torch.int16, device=dev)
    grads = [torch.empty(shape + (cfg.d,), dtype=torch.float32, device=dev) for _ in range(3)]
    fws = had.workspace(cfg.B, cfg.H, cfg.n, cfg.d, cfg.N, device=dev)
    bws = torch.empty(had.had_workspace_bytes(had.HAD_OP_ATTENTION_BWD, cfg.B, cfg.H, cfg.n,
                                              cfg.d, cfg.N), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    launches = (had.had_launch_count(had.HAD_OP_ATTENTION_FWD, cfg.B, cfg.H, cfg.n, cfg.d, cfg.N)
                + had.had_launch_count(had.HAD_OP_ATTENTION_BWD, cfg.B, cfg.H, cfg.n, cfg.d,
                                       cfg.N) - 1)      # the kept set is given: no recompute

    def fwd():
        had.had_attention_fwd(gq, gk, gv, gsq, gsk, cfg.N, cfg.tau, out=out, dbg_idx=idx,
                              dbg_logits=lg, ws=fws)

    def bwd():
        had.had_attention_bwd(gq, gk, gv, gsq, gsk, dout, cfg.N, cfg.tau, 1.0, idx=idx,
                              logits=lg, dq=grads[0], dk=grads[1], dv=grads[2], ws=bws)

    for _ in range(max(3, args.warmup)):
        fwd()
        bwd()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))
        ev[i][0].record(stream)
        fwd()
        ev[i][1].record(stream)
        bwd()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clock_info = clocks.stop()
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    bwd_local = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    value, ms = aggregate(cfg.tokens, fwd_ms + bwd_local, world, dev)
    bwd_ms = max_over_ranks(bwd_local, world, dev)
    elt = 2 if cfg.dtype == "bf16" else 4
    elems = cfg.B * cfg.H * cfg.n * cfg.d
    nbytes = elems * (3 * elt + 4 + 12) + cfg.B * cfg.H * cfg.n * cfg.N * 6
    peak = peaks["hbm_gbs"]
    if rank != 0:
        return
    print(json.dumps({
        "metric": "HAD straight-through training step (forward + backward) tokens/sec",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "impl": "had_attention_fwd + had_attention_bwd",
        "config": {"workload": cfg.describe(), "clip": 1.0,
                   "l2": "flushed between steps (256 MiB write outside the timed events)"},
        "stage_ms": {"forward": fwd_ms, "backward": bwd_ms},
        "roofline": {"bound": "hbm", "achieved": nbytes / (bwd_ms * 1e-3) / 1e9, "peak": peak,
                     "unit": "GB/s", "frac": nbytes / (bwd_ms * 1e-3) / 1e9 / peak,
                     "kernel": "had_attention_bwd (7 launches)", "peaks": peaks["source"],
                     "note": "algorithmic bytes: Q,K,V,dO read, dQ,dK,dV written, kept set read"},
        "gpu_launches": launches * args.steps,
        "clocks": clock_info,
    }), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.mode == "unfused":
            run_unfused(args, world, rank, local)
        elif args.mode == "mass":
            run_mass(args, world, rank, local)
        elif args.mode == "causal":
            run_causal(args, world, rank, local)
        elif args.mode == "soft":
            run_soft(args, world, rank, local)
        elif args.mode == "bwd":
            run_bwd(args, world, rank, local)
        else:
            run_had(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
