#!/usr/bin/env python
"""Benchmark: action chunks/s of the WAM attention stack at 19.2 s of context on B200.

One step = one whole action chunk (every stage a3-a8) over one synthetic episode:
30-layer history prefill with the cache store and fusion epilogue, 4 imagination passes x 30
layers, the final cache pass, 10 Euler steps x 30 action layers (8 reading a fused pair).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

Prints ONE JSON line on rank 0.  Under torchrun (N > 1) every rank runs its own episode
(independent replicas, no collective on the data path; weak scaling); the timed region is
bracketed by a barrier + synchronize and the reported time is the max over ranks.

`--impl reference` times the fp64 CPU oracle (the only reference this path has) on the
host cores, on a bounded sample of the same workload, extrapolated to a whole chunk.
"""

from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import signal
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from cached_kv_attention_b200 import synth  # noqa: E402

METRIC = "action chunks/s at 19.2 s context (1 B200); % HBM / tensor-core roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--workload", default="ctx19.2s_bf16", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--fusion", default="epilogue", choices=["epilogue", "standalone"])
    ap.add_argument("--no-graph", action="store_true", help="issue the chunk eagerly")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--profile-call", default=None, choices=["history", "future", "action", "action_nvfp4"],
                    help="launch one stage call of the workload --repeat times and exit "
                         "(a small case for ncu captures; prints nothing)")
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--processes", type=int, default=2,
                    help="at N = 1, repeat the timed steps in this many processes in all and report "
                         "each one's median step time")
    ap.add_argument("--child", action="store_true", help=argparse.SUPPRESS)
    return ap.parse_args()


# ------------------------------------------------------------------------------ work model

def algorithmic_work(w: synth.Workload, pad: np.ndarray) -> dict:
    """Allowed work of one chunk, counting only allowed (query, key) pairs and valid keys.

    prefill FLOPs = 4 D H T^2 x sum over calls and valid query frames of the valid key
    frames it reads; action bytes = fused valid keys x H x D x 2 (K, V) x 2 B per interaction
    read plus Q/K/V (bf16) and O (fp32) of every action call."""
    T, D, H = w.T, w.D, w.H
    pair = 4.0 * D * H * T * T
    hist_pairs = fut_pairs = 0
    valid_keys = 0
    for b in range(w.B):
        valid = [f for f in range(w.F) if not pad[b, f]]
        valid_keys += len(valid) * T
        for f in range(w.F_h):
            if not pad[b, f] and (not w.slide or f == w.F_h - 1):  # sliding window: newest only
                hist_pairs += sum(1 for g in valid if g <= f)
        for f in range(w.F_h, w.F):
            fut_pairs += sum(1 for g in valid if g <= f)
    # future-frame passes: the imagination steps and the cache pass, or one per joint step
    n_pass_fut = w.n_euler_steps if w.joint else w.n_video_steps + 1
    flops_hist = pair * hist_pairs * w.L
    flops_fut = pair * fut_pairs * w.L * n_pass_fut
    act_qkvo = w.n_act * H * D * (3 * 2 + 4) * w.B
    reads = w.M * w.n_euler_steps
    calls = w.L * w.n_euler_steps
    # bytes of one fused K or V row of one head: bf16, or NVFP4 (D / 2 bytes of E2M1 codes and
    # D / 16 E4M3 block scales)
    row = D * 2 if w.kv_format == "bf16" else D // 2 + D // 16
    fused_read_bytes = valid_keys * H * row * 2  # one fused pair read (K and V)
    action_bytes = fused_read_bytes * reads + act_qkvo * calls
    return {
        "imag_flops_per_launch": pair * fut_pairs,
        "prefill_flops": flops_hist + flops_fut,
        "prefill_launches": w.L * (1 + n_pass_fut),
        "action_bytes": action_bytes,
        "action_launches": calls,
        "action_reads": reads,
        "fused_read_bytes": fused_read_bytes,
        "valid_keys": valid_keys,
    }


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples (200 ms) taken while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.path = index, None, None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.send_signal(signal.SIGTERM)
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9:
                rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# ------------------------------------------------------------------------------ distributed

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def replica_throughput(ms_local: float, world: int):
    """Whole-job throughput of N independent replicas (one episode per rank, weak scaling):
    the step time is the slowest rank's, and the job completes one chunk per rank per step.
    Returns (ms per step, chunks/s over all ranks)."""
    ms = max_over_ranks(ms_local, world)
    return ms, world * 1000.0 / ms


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------ CPU oracle

def oracle_sample_seconds(w: synth.Workload, pad: np.ndarray, n_heads: int, n_layers: int,
                          seed: int, row_stride: int = 1) -> float:
    """Time the oracle (as it stands) over every stage of one chunk for n_heads heads and
    n_layers layers (inputs drawn per head, same distributions), computing every
    row_stride-th video query row (rows are independent).  Returns seconds."""
    from oracle import wam_oracle as O
    T, D = w.T, w.D
    hist, fut = w.F_h * T, w.F_f * T
    g = lambda name, tok, *i: synth.normal((w.B, tok, n_heads, D), seed, "cpu_" + name, *i,
                                           std=w.qkv_std, dtype=torch.bfloat16).double().numpy()
    layers = list(range(n_layers))
    hq = [g("hq", hist, l) for l in layers]
    hk = [g("hk", hist, l) for l in layers]
    hv = [g("hv", hist, l) for l in layers]
    # future-frame passes: imagination steps + the cache pass, or one per joint step (the
    # co-denoising chunk does the same work in another order)
    n_fut = w.n_euler_steps if w.joint else w.n_video_steps + 1
    iq = [[g("iq", fut, s, l) for l in layers] for s in range(n_fut)]
    ik = [[g("ik", fut, s, l) for l in layers] for s in range(n_fut)]
    iv = [[g("iv", fut, s, l) for l in layers] for s in range(n_fut)]
    aq = [[g("aq", w.n_act, i, l) for l in layers] for i in range(w.n_euler_steps)]
    ak = [[g("ak", w.n_act, i, l) for l in layers] for i in range(w.n_euler_steps)]
    av = [[g("av", w.n_act, i, l) for l in layers] for i in range(w.n_euler_steps)]
    xf = np.zeros((w.B, fut, w.C))
    vf = np.ones((w.B, fut, w.C))
    xa = np.zeros((w.B, w.n_act, w.A))
    va = np.ones((w.B, w.n_act, w.A))
    N = w.F * T
    t0 = time.perf_counter()
    kc = [O.cache_store(np.zeros((w.B, N, n_heads, D)), hk[l], pad, T, 0, w.F_h) for l in layers]
    vc = [O.cache_store(np.zeros((w.B, N, n_heads, D)), hv[l], pad, T, 0, w.F_h) for l in layers]
    rows_h = np.arange((w.F_h - 1) * T if w.slide else 0, hist, row_stride)
    rows_f = np.arange(0, fut, row_stride)
    for l in layers:
        O.video_prefill(hq[l], hk[l], hv[l], None, None, pad, None, T, 0, w.F_h, rows=rows_h)
    n_ode = n_fut if w.joint else w.n_video_steps
    sv = O.flow_schedule(n_ode, 0.0 if w.joint else w.sigma_star) if n_ode > 0 else None
    for s in range(n_fut):
        for l in layers:
            O.video_prefill(iq[s][l], ik[s][l], iv[s][l], kc[l], vc[l], pad, None, T, w.F_h, w.F,
                            rows=rows_f)
        if s < n_ode:
            xf = O.euler_step(xf, vf, sv[s + 1] - sv[s])
    for l in layers:
        kc[l] = O.cache_store(kc[l], ik[-1][l], pad, T, w.F_h, w.F)
        vc[l] = O.cache_store(vc[l], iv[-1][l], pad, T, w.F_h, w.F)
    wts = O.fuse_weights(np.zeros(n_layers))
    fk = O.fuse_interval(kc, wts)
    fv = O.fuse_interval(vc, wts)
    sa = O.flow_schedule(w.n_euler_steps)
    interaction = max(1, round(n_layers * w.M / w.L))
    for i in range(w.n_euler_steps):
        for j, l in enumerate(layers):
            video = j < interaction
            O.action_attention(aq[i][l], ak[i][l], av[i][l], fk if video else None,
                               fv if video else None, pad, T)
        xa = O.euler_step(xa, va, sa[i + 1] - sa[i])
    return time.perf_counter() - t0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w: synth.Workload, pad: np.ndarray, seed: int) -> dict:
    n_heads, n_layers = 1, 4
    sec = oracle_sample_seconds(w, pad, n_heads, n_layers, seed)
    scale = (w.H / n_heads) * (w.L / n_layers)
    chunk_s = sec * scale
    return {"value": 1.0 / chunk_s, "unit": "chunks/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"all stages of one chunk for {n_heads}/{w.H} heads x {n_layers}/{w.L} layers "
                      f"({sec:.1f} s of fp64 CPU work), extrapolated x{scale:.0f} to a whole chunk"}


def parity_sample(w: synth.Workload, pad: np.ndarray) -> dict:
    """Parity of this library against the oracle on a sample of the workload: the same chunk
    (frames, padding, schedules, Euler steps) on 1 head and 4 layers (one fusion interval read
    by layer 3), run through the chunk runner and through the oracle's chunk on the same seeded
    inputs.  Per stage: the worst max|err| / max|ref| and the worst mean relative error
    sum|err| / sum|ref| over the stage's output tensors."""
    from cached_kv_attention_b200 import chunk as C
    from oracle import wam_oracle as O
    if w.slide:
        return None
    ws = w.replace(name=w.name + "_parity", H=1, L=4, seed=w.seed + 77)

    def tree(x, fn):
        return [tree(y, fn) for y in x] if isinstance(x, list) else fn(x)

    to64 = lambda t: t.float().cpu().double().numpy()
    inp_cpu = C.make_inputs(ws, "cpu")
    inp = {k: tree(v, lambda t: t.cuda()) for k, v in inp_cpu.items()}
    r = C.ChunkRunner(ws, inp, pad=pad, distinct_out=True).prepare()
    r.run()
    torch.cuda.synchronize()
    inp64 = {k: tree(v, to64) for k, v in inp_cpu.items()}
    inp64["fuse_weights"] = [O.fuse_weights(x) for x in inp64.pop("fuse_logits")]
    kw = dict(L=ws.L, S=ws.S, T=ws.T, F_h=ws.F_h, F_f=ws.F_f, pad=pad)
    if ws.joint:
        ref = O.chunk_joint(inp64, n_steps=ws.n_euler_steps, **kw)
    else:
        ref = O.chunk(inp64, n_video_steps=ws.n_video_steps, n_euler_steps=ws.n_euler_steps,
                      sigma_star=ws.sigma_star, **kw)
    rows = lambda f0, f1: np.repeat(~pad[:, f0:f1].astype(bool), ws.T, axis=1)
    out = {}

    def add(stage, got, want, mask=None):
        got, want = to64(got), np.asarray(want)
        if mask is not None:
            got, want = got[mask], want[mask]
        err = np.abs(got - want)
        mx = float(err.max() / max(np.abs(want).max(), 1e-300))
        mean = float(err.sum() / max(np.abs(want).sum(), 1e-300))
        o = out.setdefault(stage, {"max_rel": 0.0, "mean_rel": 0.0})
        o["max_rel"], o["mean_rel"] = max(o["max_rel"], mx), max(o["mean_rel"], mean)

    for l in range(ws.L):
        add("history", r.hist_o[l], ref["hist_o"][l], rows(0, ws.F_h))
        if not ws.joint:
            add("final", r.final_o[l], ref["final_o"][l], rows(ws.F_h, ws.F))
            for s_ in range(ws.n_video_steps):
                add("imagination", r.imag_o[s_ * ws.L + l], ref["imag_o"][s_][l], rows(ws.F_h, ws.F))
    reader = set(C.interaction_layers(ws.L, ws.S))
    for i in range(ws.n_euler_steps):
        for l in range(ws.L):
            add("fused read" if l in reader else "self-only read", r.act_o[i * ws.L + l], ref["act_o"][i][l])
    for m in range(ws.M):
        add("fused pairs", r.fused_k[m], ref["fused_k"][m], rows(0, ws.F))
        add("fused pairs", r.fused_v[m], ref["fused_v"][m], rows(0, ws.F))
    add("x_act", r.x_act, ref["x_act"])
    return {"sample": f"the chunk on 1/{w.H} heads and 4/{w.L} layers (one fusion interval)",
            "bounds": {"bf16": {"max_rel": 1e-2, "mean_rel": 2e-3}, "f32": {"max_rel": 1e-5}},
            "stages": out}


# ------------------------------------------------------------------------------ reference arm

def run_reference(args, world, rank):
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    pad = synth.pad_mask(w).numpy()
    n_heads, n_layers, stride = 1, 1, 4
    scale = (w.H / n_heads) * (w.L / n_layers)
    for i in range(args.warmup):
        oracle_sample_seconds(w, pad, n_heads, n_layers, seed=1000 + i, row_stride=stride)
    times = [oracle_sample_seconds(w, pad, n_heads, n_layers, seed=2000 + i, row_stride=stride)
             for i in range(args.steps)]
    # the video stages were sampled on 1/stride of their query rows: time them at full rows
    full = oracle_sample_seconds(w, pad, n_heads, n_layers, seed=3000, row_stride=1)
    part = oracle_sample_seconds(w, pad, n_heads, n_layers, seed=3000, row_stride=stride)
    step_s = sum(times) / len(times)
    # one timed step does this fraction of a chunk's work (its rows on 1 / stride of the video
    # queries, timed against one full-row step, and 1 / scale of the heads x layers)
    chunks_per_step = 1.0 / ((full / part) * scale)
    value = chunks_per_step / step_s
    sample = (f"each step: all stages of one chunk for {n_heads}/{w.H} heads x {n_layers}/{w.L} "
              f"layers on every {stride}th video query row, scaled to all rows by one full-row "
              f"step (x{full / part:.2f}) and x{scale:.0f} to a whole chunk")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "chunks/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "chunks_per_step": chunks_per_step,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "L": w.L, "H": w.H, "D": w.D, "T": w.T,
                   "F_h": w.F_h, "F_f": w.F_f, "pad_frames": int(pad.sum()), "n_act": w.n_act,
                   "n_video_steps": w.n_video_steps, "n_euler_steps": w.n_euler_steps},
        "cpu_baseline": {"value": value, "unit": "chunks/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "chunks/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ this library

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one imagination-pass prefill
# launch, from one ncu capture of the same kernel (`bench.py --profile-call future`); the
# stride variants launch the identical imagination pass, other workloads report None.
# None: the kernel has changed since its last capture (80.47 MB per launch, before the prefill
# kernel became one instantiation per pairing mode); the next capture fills it in again.
IMAG_TRAFFIC_BYTES = {"ctx19.2s_bf16": None}
# The same for one fused-cache action read (`bench.py --profile-call action`, and
# `--workload nvfp4_ctx19.2s_bf16 --profile-call action_nvfp4` for the NVFP4 read); the stride
# variants issue the identical bf16 read.
ACTION_TRAFFIC_BYTES = {"ctx19.2s_bf16": 67.70e6, "nvfp4_ctx19.2s_bf16": 19.27e6}


def time_fused_read(runner, stream, n=20) -> float:
    """Mean device time (ms) of one fused-cache action read: the chunk's own interaction reads of
    its first Euler step (one per fused pair, M launches, 8 x 66 MB at 19.2 s: larger than L2),
    captured back to back in one CUDA graph and replayed after a 256 MB write that flushes the L2
    and a 256 MB read of another buffer (so no dirty line is left to write back), with CUDA events
    around the replay; the time divided by the number of reads."""
    calls = runner.calls
    first = runner.fused_read_call
    reads = [i for i in range(first, len(calls))
             if calls[i][0] is calls[first][0] and calls[i][1][2] is not None][:runner.w.M]
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    clean = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    total = torch.zeros((), dtype=torch.float32, device="cuda")
    for i in reads:  # once outside capture (one-time per-device set-up)
        fn, args = calls[i]
        if fn(*args):
            raise RuntimeError("fused read call failed")
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in reads:
            fn, args = calls[i]
            if fn(*args):
                raise RuntimeError("fused read call failed")
    ts = []
    for i in range(n + 3):
        flush.fill_(float(i))
        torch.sum(clean, dim=0, out=total)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(a.elapsed_time(b) / len(reads))
    del g, flush, clean, total
    return statistics.mean(ts)


def run_mine(args, world, rank, local):
    from cached_kv_attention_b200 import chunk as C
    from cached_kv_attention_b200 import wam

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w0 = synth.WORKLOADS[args.workload]
    w = w0.replace(seed=w0.seed + 1000 * rank)  # each rank: its own episode
    pad = synth.pad_mask(w0).numpy()
    work = algorithmic_work(w, pad)

    inp = C.make_inputs(w, device="cuda")
    torch.cuda.synchronize()
    # one dedicated stream: the chunk is prepared, warmed up, captured and replayed on it
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    runner = C.ChunkRunner(w, inp, pad=pad, distinct_out=False, fusion=args.fusion).prepare(stream)
    launches = runner.launches_per_chunk()

    ev = {name: (torch.cuda.Event(enable_timing=True, external=True),
                 torch.cuda.Event(enable_timing=True, external=True))
          for name, _, _ in runner.stages}
    if w.slide:
        runner.prime()  # the state the first streamed chunk continues from
    runner.run()  # first call: one-time per-device set-up outside any capture
    torch.cuda.synchronize()
    wam.device_error()
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            runner.run(events=ev, stream=stream)
        step = graph.replay
    else:
        step = lambda: runner.run(events=ev, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stage_ms = {k: [] for k in ev}
    # one event between consecutive steps: the whole region for the mean, each step for the median
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        marks[0].record(stream)
        for i in range(args.steps):
            step()
            marks[i + 1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = marks[0].elapsed_time(marks[-1])
    step_times = [marks[i].elapsed_time(marks[i + 1]) / runner.chunks_per_run for i in range(args.steps)]
    if args.child:
        print(json.dumps({"median_ms": statistics.median(step_times)}), flush=True)
        return
    # Stage events are re-recorded by every step: read the last timed step's stage times,
    # then time up to 10 more steps one by one for the stage averages.
    for k, (a, b) in ev.items():
        stage_ms[k].append(a.elapsed_time(b))
    for _ in range(min(args.steps, 10)):
        step()
        torch.cuda.synchronize()
        for k, (a, b) in ev.items():
            stage_ms[k].append(a.elapsed_time(b))
    wam.device_error()
    # a run is one chunk, or two streamed chunks in the sliding-window mode
    ms, value = replica_throughput(total_ms / args.steps / runner.chunks_per_run, world)
    st_ms = {k: statistics.mean(v) for k, v in stage_ms.items()}
    if w.joint:  # co-denoising: per joint step a video stage (future passes) and an action stage
        fut_ms = sum(v for k, v in st_ms.items() if k.startswith("video"))
        st_ms = {"history": st_ms["history"], "joint_video": fut_ms,
                 "action": sum(v for k, v in st_ms.items() if k.startswith("action"))}
        video_ms = st_ms["history"] + fut_ms
    else:
        video_ms = (st_ms["history"] + st_ms["imagination"] + st_ms["final"] + st_ms.get("copy", 0.0) +
                    st_ms.get("quantize", 0.0))
    action_ms = st_ms["action"]
    fused_ms = time_fused_read(runner, stream)

    peaks = {}
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk):
        peaks = json.load(open(pk))
    tflops_peak = peaks.get("bf16_tflops_sustained")
    hbm_peak = peaks.get("hbm_gbs")
    peak_src = "measured" if peaks else "fallback"
    if tflops_peak is None:
        tflops_peak = 1400.0
    if hbm_peak is None:
        hbm_peak = 6650.0

    # Dominant kernel: the imagination-pass prefill (4 passes x L layers per chunk, the largest
    # share of the step).  Its launch time is the imagination stage over its prefill launches
    # (the stage's four Euler launches, ~3 us each, are included).
    # (With no imagination step, the one-shot variant, the final pass stands in: same shape,
    # plus the cache store and fusion epilogue.)
    pass_name = ("joint_video" if w.joint else "imagination" if w.n_video_steps > 0 else "final")
    n_imag = (w.n_euler_steps * w.L if w.joint else
              w.n_video_steps * w.L if w.n_video_steps > 0 else w.L)
    imag_ms = st_ms[pass_name] / n_imag
    imag_tflops = work["imag_flops_per_launch"] / (imag_ms * 1e-3) / 1e12
    same_launch = (w.n_video_steps > 0 and not w.joint and
                   w0.replace(name="ctx19.2s_bf16", S=4) == synth.WORKLOADS["ctx19.2s_bf16"])
    roofline = {"bound": "tensor", "achieved": imag_tflops, "peak": tflops_peak,
                "unit": "TFLOP/s", "frac": imag_tflops / tflops_peak,
                "traffic": IMAG_TRAFFIC_BYTES["ctx19.2s_bf16"] if same_launch else None,
                "kernel": f"prefill_tc_kernel, {pass_name} pass (wam_video_prefill_kv)",
                "peak_kind": f"{peak_src} bf16 sustained",
                "flops_per_launch": work["imag_flops_per_launch"], "ms_per_launch": imag_ms,
                "video_stage_tflops": work["prefill_flops"] / (video_ms * 1e-3) / 1e12}
    fused_bytes = work["fused_read_bytes"] + w.n_act * w.H * w.D * (3 * 2 + 4) * w.B
    fused_gbs = fused_bytes / (fused_ms * 1e-3) / 1e9
    traffic_key = "ctx19.2s_bf16" if w.name.startswith("stride") and w.name.endswith("_ctx19.2s_bf16") else w.name
    action_traffic = ACTION_TRAFFIC_BYTES.get(traffic_key)
    roofline_action = {"bound": "hbm", "achieved": fused_gbs, "peak": hbm_peak, "unit": "GB/s",
                       "frac": fused_gbs / hbm_peak,
                       "kernel": ("action_nvfp4_kernel, one NVFP4 fused-cache read (wam_action_attn_nvfp4)"
                                  if w.kv_format == "nvfp4" else
                                  "action_umma_kernel, one fused-cache read (wam_action_attn)"),
                       "peak_kind": f"{peak_src} copy bandwidth", "bytes_per_launch": fused_bytes,
                       "traffic": action_traffic,
                       "ms_per_launch": fused_ms,
                       "method": "one Euler step's interaction reads (one per fused pair) back to back "
                                 "in a CUDA graph after an L2 flush, time / reads",
                       "action_stage_gbs": work["action_bytes"] / (action_ms * 1e-3) / 1e9}

    protocol = {"warmup": args.warmup, "samples": args.steps,
                "median_ms_per_process": [statistics.median(step_times)],
                "mean_ms": total_ms / args.steps / runner.chunks_per_run}
    if rank == 0 and world == 1 and args.processes > 1:
        protocol["median_ms_per_process"] += other_process_medians(args, args.processes - 1)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, w, runner, inp, step, pad, world)

    cpu = parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, pad, seed=7)
        parity = parity_sample(w, pad)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "chunks/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "L": w.L, "H": w.H, "D": w.D, "T": w.T,
                       "F_h": w.F_h, "F_f": w.F_f, "pad_frames": int(pad.sum()),
                       "valid_keys": work["valid_keys"], "n_act": w.n_act,
                       "n_video_steps": w.n_video_steps, "n_euler_steps": w.n_euler_steps,
                       "fusion_stride": w.S, "fusion": args.fusion, "fused_cache": w.kv_format,
                       "launch": "cuda graph" if graph is not None else "eager",
                       "l2": "inputs larger than L2: ~25 GB of distinct per-layer buffers per chunk",
                       "parallelism": f"replicas x{world}"},
            "stage_ms": {**st_ms, "video": video_ms},
            "protocol": protocol,
            "roofline": roofline,
            "roofline_action": roofline_action,
            "cpu_baseline": cpu,
            "parity": parity,
            "e2e": e2e,
            "gpu_launches": launches * args.steps,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if graph is not None:
        del graph


def other_process_medians(args, n: int) -> list:
    """Median step time (ms) of the same timed steps in n more processes, run one after another
    (the pages time 5 warm-ups + 30 samples in two processes and report medians)."""
    out = []
    for _ in range(n):
        cmd = [sys.executable, os.path.abspath(__file__), "--steps", str(args.steps), "--warmup",
               str(args.warmup), "--workload", args.workload, "--fusion", args.fusion, "--child"]
        if args.no_graph:
            cmd.append("--no-graph")
        r = subprocess.run(cmd, capture_output=True, text=True)
        lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
        if r.returncode != 0 or not lines:
            raise RuntimeError(f"bench child process failed (rc {r.returncode}): {r.stderr[-2000:]}")
        out.append(json.loads(lines[-1])["median_ms"])
    return out


def measure_e2e(args, w, runner, inp, step, pad, world) -> dict:
    """Chunks/s through the public API with the chunk's inputs in pinned HOST memory: every
    step copies the inputs it reads (the non-padding frames of every Q/K/V tensor, the
    velocities and initial noise) host -> device, runs the chunk and reads x_act back."""
    stream = torch.cuda.current_stream()
    valid = [f for f in range(w.F) if not pad[0, f]] if w.B == 1 else None
    copies = []  # (device tensor view, host tensor view)
    pools = {}

    def host_like(key, t, slot):
        k = (key, slot)
        if k not in pools:
            pools[k] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            pools[k].copy_(t.cpu() if t.numel() < (1 << 26) else torch.ones(t.shape, dtype=t.dtype))
        return pools[k]

    def add(key, t, slot, frame_rows=None):
        h = host_like(key, t, slot)
        if frame_rows is None:
            copies.append((t, h))
        else:
            for r0, r1 in frame_rows:
                copies.append((t[:, r0:r1], h[:, r0:r1]))

    T = w.T
    runs = []
    if valid is not None:
        hv = [f for f in valid if f < w.F_h]
        if hv:
            s0 = hv[0]
            prev = s0
            for f in hv[1:] + [None]:
                if f is None or f != prev + 1:
                    runs.append((s0 * T, (prev + 1) * T))
                    if f is not None:
                        s0 = f
                if f is not None:
                    prev = f
    else:
        runs = None
    for name in (("new_q", "new_k", "new_v") if w.slide else ("hist_q", "hist_k", "hist_v")):
        for l, t in enumerate(inp[name]):
            add(name, t, l % 2, None if w.slide else runs)
    for name in ("imag_q", "imag_k", "imag_v", "act_q", "act_k", "act_v", "joint_q", "joint_k", "joint_v"):
        for i, row in enumerate(inp[name]):
            for l, t in enumerate(row):
                add(name, t, (i + l) % 2)
    for name in ("final_q", "final_k", "final_v"):
        for l, t in enumerate(inp[name]):
            add(name, t, l % 2)
    for name in ("v_future", "v_act"):
        for i, t in enumerate(inp[name]):
            add(name, t, i % 2)
    add("x_future", runner.x_future, 0)
    add("x_act", runner.x_act, 0)
    h2d = sum(d.numel() * d.element_size() for d, _ in copies)
    out_host = torch.empty(runner.x_act.shape, dtype=torch.float32, pin_memory=True)
    d2h = out_host.numel() * 4
    # Step i + 1's inputs cross PCIe on a copy stream into a staging set while step i's chunk
    # runs; each step then moves its staged inputs into the chunk's buffers (device to device,
    # on the compute stream) before replaying the chunk.
    staged = [torch.empty_like(d) for d, _ in copies]
    copy_stream = torch.cuda.Stream()

    def h2d_into_staging():
        with torch.cuda.stream(copy_stream):
            for (_, h), s_ in zip(copies, staged):
                s_.copy_(h, non_blocking=True)
        e = torch.cuda.Event()
        e.record(copy_stream)
        return e

    def run(n_steps):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        copy_stream.wait_event(start)
        ready = h2d_into_staging()
        for i in range(n_steps):
            stream.wait_event(ready)
            for (d, _), s_ in zip(copies, staged):
                d.copy_(s_, non_blocking=True)
            free = torch.cuda.Event()
            free.record(stream)
            if i + 1 < n_steps:
                copy_stream.wait_event(free)
                ready = h2d_into_staging()
            step()
            out_host.copy_(runner.x_act, non_blocking=True)
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    run(1)
    barrier(world)
    total = run(args.e2e_steps)
    ms = max_over_ranks(total / args.e2e_steps / runner.chunks_per_run, world)
    cpr = runner.chunks_per_run
    return {"value": world * 1000.0 / ms, "unit": "chunks/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d // cpr, "d2h_bytes_per_step": d2h // cpr,
            "h2d_gbs": h2d / cpr / (ms * 1e-3) / 1e9,
            "note": "inputs in pinned host memory; the non-padding frames of every Q/K/V tensor, "
                    "the velocities and initial noise copied host->device every step (timed), on "
                    "a copy stream overlapping the previous step's chunk, then moved into the "
                    "chunk's buffers; x_act read back every step; bound by the host link "
                    "(48.5 GB/s with 1, 2 or 4 copy streams)"}


def profile_call(args):
    """One stage call of one layer at the workload's full size, repeated: the history prefill
    (with the cache store and a fusion epilogue), a future-frame prefill reading the cache,
    or a fused action read."""
    from cached_kv_attention_b200 import wam
    w = synth.WORKLOADS[args.workload]
    pad = synth.pad_mask(w).numpy()
    lay = wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, pad)
    bf = torch.bfloat16
    g = lambda n, tok: synth.normal((w.B, tok, w.H, w.D), w.seed, "prof_" + n, std=w.qkv_std,
                                    dtype=bf, device="cuda")
    shape = (w.B, w.N, w.H, w.D)
    kc, vc = g("kc", w.N), g("vc", w.N)
    if args.profile_call == "history":
        q, k, v = g("q", w.F_h * w.T), g("k", w.F_h * w.T), g("v", w.F_h * w.T)
        o = torch.empty((w.B, w.F_h * w.T, w.H, w.D), device="cuda")
        acc_k = torch.zeros(shape, device="cuda")
        acc_v = torch.zeros(shape, device="cuda")
        epi = wam.FuseEpilogue(0.25, False, False, acc_k, acc_v, None, None)
        call = lambda: wam.video_prefill_kv(lay, 0, w.F_h, q, k, v, kc, vc, o, True, epi)
    elif args.profile_call == "future":
        q, k, v = g("q", w.F_f * w.T), g("k", w.F_f * w.T), g("v", w.F_f * w.T)
        o = torch.empty((w.B, w.F_f * w.T, w.H, w.D), device="cuda")
        call = lambda: wam.video_prefill_kv(lay, w.F_h, w.F, q, k, v, kc, vc, o, False)
    elif args.profile_call == "action":
        qa, ka, va = g("qa", w.n_act), g("ka", w.n_act), g("va", w.n_act)
        o = torch.empty((w.B, w.n_act, w.H, w.D), device="cuda")
        call = lambda: wam.action_attn(lay, kc, vc, qa, ka, va, o)
    else:  # the NVFP4 read over the cache encoded once
        qa, ka, va = g("qa", w.n_act), g("ka", w.n_act), g("va", w.n_act)
        o = torch.empty((w.B, w.n_act, w.H, w.D), device="cuda")
        cache = wam.Nvfp4Cache(lay, 2)
        wam.fused_to_nvfp4(lay, [kc, vc], cache)
        call = lambda: wam.action_attn_nvfp4(lay, cache, 0, 1, qa, ka, va, o)
    for _ in range(args.repeat):
        call()
    torch.cuda.synchronize()
    wam.device_error()


def main():
    args = parse()
    if args.profile_call:
        profile_call(args)
        return
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            if not torch.cuda.is_available():
                raise SystemExit("bench.py: this implementation needs a CUDA GPU (B200)")
            run_mine(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
