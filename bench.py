#!/usr/bin/env python
"""Benchmark: MoE-layer tokens/s for single-token decode of the 2-bit MoE FFN layer.

Workload (one step): DECODE_BURST single-token decode passes (B = 1) through
the decode layer -- d=4096, 256 routed experts (IQ2X gate/up, Q2K down),
f=2048, top-8, bf16 shared expert f=2048 -- each pass = route + gate/up +
down/combine.  Successive passes rotate over LAYERS resident layers, so the
weights read between two uses of a layer (~330 MB) exceed the 126 MB L2: no
flush is needed and none of a pass's weights is served from L2 by the previous
pass.  The timed region replays a CUDA graph of one step K times.

Also reported: the dominant kernel's roofline (the gate/up GEMV, HBM-bound),
an end-to-end number through the public Python API with host<->device copies,
the CPU oracle as baseline, a prefill measurement (T=4096, grouped GEMM) and,
on one GPU, the other workloads: the tiny latency case, the batched decode
sweep (B = 1, 4, 16, 64) and the Q4K layer (T=16384 prefill, B=1 decode).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: data-parallel replicas (each rank decodes its own token stream);
no collective on the data path.
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
sys.path.insert(0, ROOT)

from bit_quantized_moe_02_b200 import synth  # noqa: E402

DECODE_BURST = 256
LAYERS = 4
METRIC = "MoE-layer decode tokens/s (B=1)"
UNIT = "tokens/s"


def workload_config(wl, extra=None):
    s = wl.shape
    c = {"workload": "decode d=%d E=%d f=%d k=%d shared_f=%d B=1, IQ2X gate/up + Q2K down, bf16 shared"
                     % (s.d, s.E, s.f, s.k, s.f_shared),
         "tokens_per_step": DECODE_BURST, "layers_rotated": LAYERS,
         "l2": "inputs larger than L2: %d layers rotated, %.0f MB of weights read per pass" % (
             LAYERS, layer_bytes(wl) / 1e6)}
    if extra:
        c.update(extra)
    return c


def layer_bytes(wl):
    """Algorithmic bytes of one B=1 decode pass: k experts' packed blocks, shared bf16 weights, router, x, out."""
    s = wl.shape
    routed = s.k * (2 * s.f * (s.d // 256) * 66 + s.d * (s.f // 256) * 84)
    return routed + s.shared_bytes + s.router_bytes + s.d * 2 + s.d * 4


def step_bytes(shape, n_unique, B):
    """Algorithmic bytes of one decode step of B tokens that touches n_unique distinct experts: each touched
    expert's packed blocks once, the shared expert and router once, x in (bf16) and out (fp32)."""
    return n_unique * shape.expert_bytes + shape.shared_bytes + shape.router_bytes + B * shape.d * (2 + 4)


def gateup_bytes(wl):
    s = wl.shape
    return s.k * 2 * s.f * (s.d // 256) * 66 + 2 * s.f_shared * s.d * 2 + s.d * 2


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [v.strip() for v in l.split(",")]
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args=None):
    """One process per GPU under torchrun (RANK / WORLD_SIZE / LOCAL_RANK from the environment).  The process
    group carries only the barrier and the max-over-ranks timing (replicas: no data-path collective): NCCL on
    GPUs, gloo where no GPU is present (the CPU tests)."""
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    gpu = torch.cuda.is_available()
    if gpu:
        torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=600)
        if gpu:
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, ws):
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------------------------------------
# CPU oracle legs


def oracle_tokens_per_s(wl, n_tokens, nthreads, seed_stream=7):
    """Time the oracle (as it stands) on n_tokens decode tokens of layer 0, nthreads host threads."""
    import oracle
    L = synth.make_layer(wl, layer=0)
    x = synth.activations(wl, n_tokens, stream=seed_stream)
    ids, _, _, _ = oracle.route(x, L.wr, L.bias, wl.shape.k)
    for e in np.unique(ids):  # generate the touched experts before the clock starts
        for w in ("gate", "up", "down"):
            L.expert(w, int(e))
    t0 = time.perf_counter()
    oracle.layer_forward(L.shape, x, L.wr, L.bias, L.grid, L.expert, (L.sh_gate, L.sh_up, L.sh_down),
                         nthreads=nthreads)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


def workload_cpu_baselines(cores):
    """The oracle timed on each other workload's layer (bounded samples of a few seconds each, all host threads):
    tokens/s on the tiny layer, on the batched-decode layer (router bias N(0,1); the oracle's per-token cost does
    not depend on the batch size), on the prefill layer (tokens of the T=4096 input) and on the Q4K layer."""
    res = {}
    for name, per_thread in (("tiny", 256), ("batched", 4), ("prefill", 4), ("q4", 2)):
        wl = synth.WORKLOADS[name]
        n = per_thread * cores
        tps, dt = oracle_tokens_per_s(wl, n, cores)
        res[name] = {"value": tps, "unit": UNIT, "cores": cores, "kind": "oracle",
                     "sample": "%d tokens of the %s workload's layer 0 (%d per host thread), %.1f s"
                               % (n, name, per_thread, dt)}
    return res


def run_reference(args, ws, rank):
    wl = synth.WORKLOADS["decode"]
    if rank != 0:
        return
    cores = os.cpu_count() or 1
    if args.warmup:
        oracle_tokens_per_s(wl, min(args.warmup, cores), min(args.warmup, cores), seed_stream=8)
    tps, dt = oracle_tokens_per_s(wl, args.steps, cores)
    cb = {"value": tps, "unit": UNIT, "cores": min(cores, args.steps), "kind": "oracle",
          "sample": "%d decode tokens (one per step), plain C oracle, fp32 dequant + fp64 contraction" % args.steps}
    line = {"impl": "reference", "metric": METRIC, "value": tps, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, {"tokens_per_step": 1}), "cpu_baseline": cb,
            "e2e": {"value": tps, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------------------
# our arm


GATEUP_KERNEL = "decode_gateup_kernel<0, 8, 4>"
GATEUP_SRC = os.path.join(ROOT, "bit_quantized_moe_02_b200", "csrc", "decode_gemv.cuh")


def gateup_traffic():
    """DRAM bytes (read + write) of one gate/up launch from the committed ncu summary, or None when the kernel
    source has changed since those counters were taken (the summary records the source's SHA-256)."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", "decode_gateup_traffic.json")
    try:
        rec = json.load(open(prof))
        sha = hashlib.sha256(open(GATEUP_SRC, "rb").read()).hexdigest()
        if rec.get("kernel") == GATEUP_KERNEL and rec.get("source_sha256") == sha:
            return rec.get("bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


def run_ours(args, ws, rank, local):
    import torch
    from bit_quantized_moe_02_b200 import ds4moe

    torch.manual_seed(0)
    wl = synth.WORKLOADS["decode"]
    s = wl.shape
    t_setup = time.perf_counter()
    layers = [ds4moe.DeviceLayer(synth.make_layer(wl, layer=l + 16 * rank), max_tokens=1) for l in range(LAYERS)]
    xs = [torch.from_numpy(synth.activations(wl, DECODE_BURST, layer=rank, stream=i)).cuda().view(torch.bfloat16)
          for i in range(1)][0]
    outs = torch.empty((DECODE_BURST, s.d), dtype=torch.float32, device="cuda")
    ids_buf = torch.empty((DECODE_BURST, s.k), dtype=torch.int32, device="cuda")
    w_buf = torch.empty((DECODE_BURST, s.k), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    setup_s = time.perf_counter() - t_setup

    def one_pass(i):
        Lr = layers[i % LAYERS]
        ds4moe.route(xs[i:i + 1], Lr.wr, Lr.bias, s.k, ws=Lr.route_ws, ids=ids_buf[i:i + 1], weights=w_buf[i:i + 1])
        ds4moe.expert_ffn_decode(Lr.ex, xs[i:i + 1], ids_buf[i:i + 1], w_buf[i:i + 1], Lr.ws, out=outs[i:i + 1])

    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for i in range(DECODE_BURST):  # eager warm-up of every launch
            one_pass(i)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(DECODE_BURST):
                one_pass(i)
        for _ in range(args.warmup):
            graph.replay()
        stream.synchronize()
        assert ds4moe.last_device_error() == 0

        # ---- timed region: exactly K steps (graph replays) ----
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(ws)
        torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
            torch.cuda.synchronize()
        barrier(ws)
        t_ms = e0.elapsed_time(e1)
    t_max = max_over_ranks(t_ms, ws)
    tokens = DECODE_BURST * args.steps * ws
    value = tokens / (t_max / 1e3)

    # ---- dominant kernel: gate/up GEMV, timed with events around each launch inside a graph ----
    hbm, tf, tf_sus, peak_kind = peaks()
    with torch.cuda.stream(stream):
        ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for _ in range(DECODE_BURST)]
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            for i in range(DECODE_BURST):
                Lr = layers[i % LAYERS]
                ds4moe.route(xs[i:i + 1], Lr.wr, Lr.bias, s.k, ws=Lr.route_ws, ids=ids_buf[i:i + 1],
                             weights=w_buf[i:i + 1])
                ev[i][0].record(stream)
                ds4moe.decode_gateup(Lr.ex, xs[i:i + 1], ids_buf[i:i + 1], Lr.ws)
                ev[i][1].record(stream)
                ds4moe.decode_down(Lr.ex, ids_buf[i:i + 1], w_buf[i:i + 1], Lr.ws, outs[i:i + 1])
                ev[i][2].record(stream)
        g2.replay()
        g2.replay()
        stream.synchronize()
    gu_ms = float(np.mean([a.elapsed_time(b) for a, b, _ in ev]))
    dn_ms = float(np.mean([b.elapsed_time(c) for _, b, c in ev]))
    gu_bytes = gateup_bytes(wl)
    achieved = gu_bytes / (gu_ms / 1e3) / 1e9
    traffic = gateup_traffic()

    # ---- end to end through the public API: pinned H2D of x, decode, D2H of the output, every step ----
    # headline: DecodeGraph (the binding's graph-replayed single-token decode); also the eager forward()
    n_e2e = min(DECODE_BURST, 256)
    x_host = torch.from_numpy(synth.activations(wl, n_e2e, layer=rank, stream=5)).pin_memory()
    out_host = torch.empty((1, s.d), dtype=torch.float32).pin_memory()
    x_dev = torch.empty((1, s.d), dtype=torch.int16, device="cuda")

    def e2e_tokens_per_s(step):
        runs = []
        for _ in range(3):  # host wall clock on a shared machine: the median of three 256-token runs
            barrier(ws)
            t0 = time.perf_counter()
            for i in range(n_e2e):
                out_host.copy_(step(i), non_blocking=True)
                stream.synchronize()
            runs.append(max_over_ranks(time.perf_counter() - t0, ws))
        return n_e2e * ws / sorted(runs)[1]

    def eager_step(i):
        x_dev.copy_(x_host[i:i + 1], non_blocking=True)
        return layers[i % LAYERS].forward(x_dev.view(torch.bfloat16))

    def host_io_tokens_per_s(graphs):
        # the graph holds the H2D copy of x from its pinned input buffer and the D2H copy of the output: per
        # token one host copy of x into that buffer, one graph launch and one synchronization
        runs = []
        for _ in range(3):
            barrier(ws)
            t0 = time.perf_counter()
            for i in range(n_e2e):
                graphs[i % LAYERS](x_host[i:i + 1])
                stream.synchronize()
            runs.append(max_over_ranks(time.perf_counter() - t0, ws))
        return n_e2e * ws / sorted(runs)[1]

    with torch.cuda.stream(stream):
        graphs = [layers[l].decode_graph() for l in range(LAYERS)]
        graphs_io = [layers[l].decode_graph(host_io=True) for l in range(LAYERS)]
        for i in range(16):
            graphs[i % LAYERS](x_host[i:i + 1])
            graphs_io[i % LAYERS](x_host[i:i + 1])
            stream.synchronize()
            eager_step(i)
        stream.synchronize()
        e2e_value = host_io_tokens_per_s(graphs_io)
        e2e_graph = e2e_tokens_per_s(lambda i: graphs[i % LAYERS](x_host[i:i + 1]))
        e2e_eager = e2e_tokens_per_s(eager_step)
    del graphs, graphs_io

    # ---- prefill: T=4096 grouped path (one layer, eager) ----
    prefill = None
    if not args.no_prefill:
        prefill = run_prefill(args, ds4moe, torch, stream, tf, tf_sus, peak_kind)

    workloads = None
    if ws == 1 and not args.no_workloads:
        try:
            workloads = run_workloads(ds4moe, torch, stream, hbm, tf, peak_kind)
        except Exception as exc:  # these are reported beside the main line, which is kept either way
            workloads = {"error": "%s: %s" % (type(exc).__name__, str(exc)[:200])}

    if rank != 0:
        return
    cpu = None
    if ws == 1 and not args.no_cpu:
        cores = os.cpu_count() or 1
        n_cpu = 12 * cores  # about a second per token and thread: a ~12 s sample
        tps, dt = oracle_tokens_per_s(wl, n_cpu, cores)
        cpu = {"value": tps, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": "%d decode tokens of layer 0 (12 per host thread), %.1f s" % (n_cpu, dt)}
        if isinstance(workloads, dict) and "error" not in workloads:
            for name, cb in workload_cpu_baselines(cores).items():
                entry = workloads.get(name) if name != "prefill" else prefill
                if isinstance(entry, dict) and "error" not in entry:
                    entry["cpu_baseline"] = cb
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_max / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 products / f32 accumulation (2-bit weights)", "data": "synthetic (seeded numpy; random-init weights)",
        "config": workload_config(wl, {"parallelism": "replicas x%d" % ws if ws > 1 else "1 GPU"}),
        "gpu_launches": 4 * DECODE_BURST * args.steps,
        "layer_bytes_per_token": layer_bytes(wl),
        "achieved_layer_GBps": layer_bytes(wl) * DECODE_BURST * args.steps / (t_ms / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "kernel": GATEUP_KERNEL, "achieved": achieved,
                     "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                     "peak_kind": peak_kind + " (burst copy)", "algorithmic_bytes_per_launch": gu_bytes,
                     "avg_launch_ms": gu_ms, "down_kernel_avg_ms": dn_ms,
                     "down_kernel_GBps": (layer_bytes(wl) - gu_bytes - s.router_bytes) / (dn_ms / 1e3) / 1e9},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": s.d * 2, "d2h_bytes_per_step": s.d * 4,
                "note": "one token per step through DecodeGraph(host_io=True): host copy of x into its pinned "
                        "input buffer, one graph launch (H2D of x, route + decode, D2H of out), sync; median of 3 "
                        "runs of 256 tokens",
                "graph_separate_copies_value": e2e_graph, "eager_forward_value": e2e_eager},
        "clocks": clk.summary(),
        "prefill": prefill,
        "workloads": workloads,
        "setup_s": setup_s,
    }
    print(json.dumps(line), flush=True)


def run_prefill(args, ds4moe, torch, stream, tf, tf_sus, peak_kind):
    wl = synth.WORKLOADS["prefill"]
    s = wl.shape
    T = wl.tokens[0]
    D = ds4moe.DeviceLayer(synth.make_layer(wl), max_tokens=T)
    x = torch.from_numpy(synth.activations(wl, T)).cuda().view(torch.bfloat16)
    y_perm = torch.empty((T * s.k, s.d), dtype=torch.float32, device="cuda")
    inv = torch.empty(T * s.k, dtype=torch.int32, device="cuda")
    ys = torch.empty((T, s.d), dtype=torch.float32, device="cuda")
    out = torch.empty((T, s.d), dtype=torch.float32, device="cuda")

    def deterministic():
        ids, w = D.route(x, ids=D.ids_buf[:T], weights=D.w_buf[:T])
        ds4moe.expert_ffn_grouped(D.ex, x, ids, w, D.ws, y_perm, inv, ys)
        ds4moe.combine(y_perm, inv, ys, T, s.d, s.k, out=out)

    def fused():
        D.forward_fused(x, out=out)

    flops = 2 * 3 * s.d * s.f * T * s.k + 2 * 3 * s.d * s.f_shared * T + 2 * T * s.E * s.d
    res = {"workload": "prefill T=%d, same layer, router bias N(0,1)" % T, "peak_tflops": tf, "peak_kind": peak_kind,
           "flops_per_step": flops}
    for name, step in (("deterministic", deterministic), ("fused", fused)):
        ms = device_ms(torch, stream, step, warmup=3, n=10)
        assert ds4moe.last_device_error() == 0
        res[name] = {"tokens_per_s": T / (ms / 1e3), "ms_per_step": ms, "tflops": flops / (ms / 1e3) / 1e12,
                     "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / tf}
    res["deterministic"]["calls"] = "route, expert_ffn_grouped (y_perm, y_shared), combine (fixed summation order)"
    res["fused"]["calls"] = "route, expert_ffn_grouped_fused (down GEMM adds into out; atomic summation order)"
    best = min(("deterministic", "fused"), key=lambda n: res[n]["ms_per_step"])
    res.update({k: res[best][k] for k in ("tokens_per_s", "ms_per_step", "tflops", "frac_of_bf16_peak")})
    res["headline_mode"] = best
    del D
    return res


def device_ms(torch, stream, step, warmup, n):
    """Mean device time of n back-to-back calls of step() on stream (CUDA events), after warmup calls."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            step()
        e1.record(stream)
        stream.synchronize()
    return e0.elapsed_time(e1) / n


class StepTimer:
    """Device time of single steps with L2 flushed in between: each step is bracketed by CUDA events on the
    stream, and a 1 GiB write (8x L2) runs between steps, outside the events.  The flush also keeps the GPU busy
    long enough for the host to enqueue the next step ahead of it, so host launch time normally does not enter."""

    def __init__(self, torch, stream):
        self.torch, self.stream = torch, stream
        self.flush = torch.empty(1 << 28, dtype=torch.float32, device="cuda")

    def mean_ms(self, step, n, warmup=2):
        torch, st = self.torch, self.stream
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        torch.cuda.synchronize()
        with torch.cuda.stream(st):
            for i in range(warmup):
                step(i)
            self.flush.zero_()
            self.flush.zero_()
            for i in range(n):
                ev[i][0].record(st)
                step(i)
                ev[i][1].record(st)
                self.flush.zero_()
            st.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in ev]))


def run_workloads(ds4moe, torch, stream, hbm, tf, peak_kind):
    """The other workloads of the layer, one GPU: the tiny latency case, the batched decode sweep (B = 1, 4, 16,
    64 with skewed routing: distinct experts touched, bytes, GB/s) and the Q4K layer (T=16384 prefill, then B=1
    decode).  Each runs the same entry points, at the same sizes, as the parity tests; a failure is reported in
    its entry instead of the numbers."""
    res = {}
    timer = StepTimer(torch, stream)

    def guarded(name, fn):
        try:
            res[name] = fn()
        except Exception as exc:  # report, keep the main line
            res[name] = {"error": "%s: %s" % (type(exc).__name__, str(exc)[:200])}

    def tiny():
        wl = synth.WORKLOADS["tiny"]
        D = ds4moe.DeviceLayer(synth.make_layer(wl), max_tokens=1)
        with torch.cuda.stream(stream):
            G = D.decode_graph()
            G(torch.from_numpy(synth.activations(wl, 1)).cuda())
            n = 2000
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for _ in range(20):
                G()
            e0.record(stream)
            for _ in range(n):
                G()
            e1.record(stream)
            stream.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / n
        s = wl.shape
        return {"workload": "tiny d=%d E=%d f=%d k=%d shared_f=%d B=1 (L2-resident: a latency case)"
                            % (s.d, s.E, s.f, s.k, s.f_shared),
                "us_per_token": us, "tokens_per_s": 1e6 / us, "bytes_per_token": step_bytes(s, s.k, 1),
                "timing": "%d back-to-back DecodeGraph replays (route + gate/up + down), CUDA events" % n}

    def batched():
        wl = synth.WORKLOADS["batched"]
        s = wl.shape
        D = ds4moe.DeviceLayer(synth.make_layer(wl), max_tokens=max(wl.tokens))
        n = 16
        rows = []
        for B in wl.tokens:
            x = torch.from_numpy(synth.activations(wl, B * n, stream=40 + B)).cuda().view(torch.bfloat16)
            ids = [None] * n

            def step(i):
                _, ids[i], _ = D.forward(x[i * B:(i + 1) * B], return_routing=True)

            ms = timer.mean_ms(step, n)
            assert ds4moe.last_device_error() == 0
            U = [len(np.unique(t.cpu().numpy())) for t in ids]
            nbytes = float(np.mean([step_bytes(s, u, B) for u in U]))
            rows.append({"B": B, "tokens_per_s": B / (ms / 1e3), "ms_per_step": ms,
                         "unique_experts_per_step": float(np.mean(U)), "bytes_per_step": nbytes,
                         "GBps": nbytes / (ms / 1e3) / 1e9, "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / hbm})
        return {"workload": "batched decode, decode layer with router bias N(0,1), B in %s" % (list(wl.tokens),),
                "timing": "mean of %d steps (distinct tokens each), L2 flushed between steps" % n,
                "peak_GBps": hbm, "peak_kind": peak_kind, "sweep": rows}

    def q4():
        wl = synth.WORKLOADS["q4"]
        s = wl.shape
        T = wl.tokens[0]
        D = ds4moe.DeviceLayer(synth.make_layer(wl), max_tokens=T)
        x = torch.from_numpy(synth.activations(wl, T)).cuda().view(torch.bfloat16)
        flops = 2 * 3 * s.d * s.f * T * s.k + 2 * 3 * s.d * s.f_shared * T + 2 * T * s.E * s.d
        prefill = {"T": T}
        for name, step in (("deterministic", lambda: D.forward_grouped(x)), ("fused", lambda: D.forward_fused(x))):
            ms = device_ms(torch, stream, step, warmup=2, n=5)
            assert ds4moe.last_device_error() == 0
            prefill[name] = {"tokens_per_s": T / (ms / 1e3), "ms_per_step": ms, "tflops": flops / (ms / 1e3) / 1e12,
                             "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / tf}
        del x
        n = 32
        x1 = torch.from_numpy(synth.activations(wl, n, stream=1)).cuda().view(torch.bfloat16)
        ms1 = timer.mean_ms(lambda i: D.forward(x1[i:i + 1]), n)
        assert ds4moe.last_device_error() == 0
        nb = step_bytes(s, s.k, 1)
        decode = {"B": 1, "tokens_per_s": 1e3 / ms1, "ms_per_token": ms1, "bytes_per_token": nb,
                  "GBps": nb / (ms1 / 1e3) / 1e9, "frac_of_hbm": nb / (ms1 / 1e3) / 1e9 / hbm,
                  "path": "single-token GEMV (Q4K)", "timing": "mean of %d tokens, L2 flushed between" % n}
        return {"workload": "q4: decode layer with Q4K gate/up/down, router bias N(0,1)", "prefill": prefill,
                "decode": decode, "peak_kind": peak_kind}

    guarded("tiny", tiny)
    guarded("batched", batched)
    guarded("q4", q4)
    del timer
    return res


def run_profile_case(args):
    """Small case for ncu captures, same kernels and shapes as the benchmark but fewer experts resident:
    the decode layer d=4096, f=2048, k=8, shared 2048 (IQ2X/Q2K, or Q4K throughout with --profile-layer q4) with
    E=16 experts (the 8 a token uses stream 56 MB of packed IQ2X/Q2K weights, 118 MB of Q4K, + 50 MB of shared
    weights per pass, about L2's size or more), 16 eager decode steps of --profile-batch tokens each; optionally
    a prefill of T tokens on E=64 experts (T=1024, k=8 keeps the prefill workload's 128 tokens per expert on
    average), in the deterministic and the fused-combine form."""
    import dataclasses

    import torch
    from bit_quantized_moe_02_b200 import ds4moe
    base = synth.WORKLOADS["decode" if args.profile_layer == "decode" else "q4"]
    wl = dataclasses.replace(base, shape=dataclasses.replace(base.shape, E=16))
    B = args.profile_batch
    D = ds4moe.DeviceLayer(synth.make_layer(wl), max_tokens=B)
    xs = torch.from_numpy(synth.activations(wl, 16 * B, stream=3)).cuda().view(torch.bfloat16)
    for i in range(16):
        D.forward(xs[i * B:(i + 1) * B])
    torch.cuda.synchronize()
    if args.profile_prefill:
        del D
        pb = synth.WORKLOADS["prefill" if args.profile_layer == "decode" else "q4"]
        wlp = dataclasses.replace(pb, shape=dataclasses.replace(pb.shape, E=64))
        T = args.profile_prefill
        P = ds4moe.DeviceLayer(synth.make_layer(wlp), max_tokens=T)
        x = torch.from_numpy(synth.activations(wlp, T)).cuda().view(torch.bfloat16)
        for _ in range(2):
            P.forward_grouped(x)
            P.forward_fused(x)
        torch.cuda.synchronize()
    assert ds4moe.last_device_error() == 0
    print(json.dumps({"profile_case": "ok", "layer": args.profile_layer, "batch": B,
                      "prefill_T": args.profile_prefill}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the tiny / batched / q4 measurements")
    ap.add_argument("--profile-case", action="store_true", help="small case for ncu captures (see profiles/)")
    ap.add_argument("--profile-prefill", type=int, default=0, help="with --profile-case: also run a T-token prefill")
    ap.add_argument("--profile-layer", default="decode", choices=["decode", "q4"],
                    help="with --profile-case: IQ2X/Q2K decode layer or its Q4K variant")
    ap.add_argument("--profile-batch", type=int, default=1, help="with --profile-case: tokens per decode step")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args)
        return
    if args.impl == "reference":
        ws, rank = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0"))
        run_reference(args, ws, rank)
        return
    ws, rank, local = dist_setup(args)
    try:
        run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
