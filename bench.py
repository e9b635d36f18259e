#!/usr/bin/env python
"""Benchmark of the fused MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
                    [--impl native|reference]

A step is one pass of the whole layer (route -> permute -> gather -> gate/up
GEMM -> [FP8 h quant] -> down GEMM -> combine) over one batch of every token
count of the workload, e.g. T = 1, 4, 16, 64 for the decode workload
(H=4096, I=14336, E=8, top-2, bf16).  Inputs are seeded synthetic tensors;
the expert weights (2.8 GB for decode) are larger than the 126 MB L2 and
four input batches rotate between steps.

Metric: layer tokens/s (whole job, all ranks).  N > 1 runs independent
replicas, one per GPU (the layer is single-GPU; there is no data-path
collective), timed on the device and reduced as the max over ranks.
`--impl reference` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import atexit
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import CONFIGS, make_batch, make_weights  # noqa: E402

WORKLOADS = {
    "decode": dict(cfg="decode", dtype=0, bound="hbm"),
    "prefill": dict(cfg="prefill", dtype=0, bound="tensor"),
    "fp8": dict(cfg="fp8", dtype=1, bound="tensor"),      # roofline entry at T=2048
    "skewed": dict(cfg="skewed", dtype=0, bound="tensor"),
}
NBATCH = 4
GRAPH_MAX_T = 64       # token counts that run as CUDA graphs
# DRAM bytes (read + write) of one gate/up launch from an ncu capture of the
# same kernel build, keyed by (workload, T); None until captured.
TRAFFIC = {("decode", 64): 1887167120, ("prefill", 4096): 1378159440,
           ("fp8", 2048): 876559360}
SMALL_T, CHUNK = 128, 2048   # the library's single-CTA route+permute limits
SMALL_AMAX = 32768           # x elements the single-CTA kernel also takes amax(x) of


def describe(name):
    c = CONFIGS[name]
    d = "fp8 e4m3" if WORKLOADS[name]["dtype"] else "bf16"
    return (f"{name} {d} H={c['H']} I={c['I']} E={c['E']} top-{c['k']} "
            f"T={','.join(str(t) for t in c['T'])}")


def kernels_per_forward(T, k, fp8, H):
    """Kernels one moe_forward launches (the cudaMemsetAsync is not a kernel)."""
    A = T * k
    small = T <= SMALL_T and A <= CHUNK
    if small:
        n = 1                                   # fused route + permute
    else:
        n = 1 + (1 if A <= CHUNK else 3)        # route, permute (1 or 3 kernels)
    n += 1                                      # gather
    n += 1 if fp8 and not (small and T * H <= SMALL_AMAX) else 0   # amax(x)
    n += 1                                      # gate/up GEMM
    n += 1 if fp8 else 0                        # h quantisation
    n += 2                                      # down GEMM + combine
    return n


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 25 ms; the summary
    keeps the samples that arrived between mark_start() and mark_end() (the
    timed regions), or all of them, flagged, when none did."""
    INTERVAL_MS = 25
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        u = str(uuid)
        self.uuid = u if u.startswith("GPU-") else "GPU-" + u
        self.proc, self.lines, self.err = None, [], ""
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
            threading.Thread(target=self._read, daemon=True).start()
            threading.Thread(target=self._read_err, daemon=True).start()
            time.sleep(0.3)   # the first samples arrive before the timed region starts
        except (OSError, ValueError) as e:
            self.proc, self.err = None, str(e)
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.perf_counter(), ln.strip()))

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def _read_err(self):
        for ln in self.proc.stderr:
            self.err += ln

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines
        window = "timed regions"
        if self.t0 is not None and self.t1 is not None:
            # a sample printed up to one interval after the region ends was taken inside it
            late = 2 * self.INTERVAL_MS / 1e3
            inside = [(t, ln) for t, ln in lines if self.t0 <= t <= self.t1 + late]
            if inside:
                lines = inside
            else:
                window = "no sample inside the timed regions; all samples"
        for _, ln in lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
               "reasons": sorted(reasons), "samples": len(sm), "window": window}
        if not sm:
            out["error"] = (self.err.strip() or "no samples")[:200]
        return out


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def gate_up_bytes(T, k, H, I, active, fp8):
    """Algorithmic bytes of one gate/up launch: the active experts' W_g and W_u,
    the T*k gathered activation rows read, the T*k rows of h written (bf16)."""
    wb = 1 if fp8 else 2
    return active * 2 * H * I * wb + T * k * H * wb + T * k * I * 2


def oracle_sample(W, dtype, Ts, budget_s=12.0):
    """The oracle on a bounded sample: tokens of the largest batch, one by one,
    until the time budget is spent.  Returns (tokens/s, cores, description)."""
    import numpy as np
    import oracle
    T = max(Ts)
    x, logits = make_batch(W, T, 0, 0)
    ids, w = oracle.route_topk(logits, W.k)
    used = sorted(set(int(e) for e in np.unique(ids)))
    remap = {e: i for i, e in enumerate(used)}
    Wg = W.Wg[used].cpu().to(torch.bfloat16)
    Wu = W.Wu[used].cpu().to(torch.bfloat16)
    Wd = W.Wd[used].cpu().to(torch.bfloat16)
    lid = np.vectorize(remap.get)(ids).astype(np.int32)
    n, t0 = 0, time.perf_counter()
    step = max(1, oracle.num_threads())
    while True:
        toks = [(n + i) % T for i in range(step)]
        if dtype == 0:
            oracle.moe_layer(x, lid, w, Wg, Wu, Wd, tokens=toks)
        else:   # the FP8 oracle needs every h row for its scale: whole batch
            oracle.moe_layer_fp8(x, lid, w, Wg, Wu, Wd, tokens=toks)
            n += T - step
        n += step
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    what = (f"oracle layer on {n} tokens of the T={T} batch ({budget_s:.0f} s budget), "
            f"{len(used)} experts")
    return n / el, oracle.num_threads(), what


def weight_device(name):
    """Where a workload's expert weights are drawn: the skewed workload's on the
    GPU (22.5 GB), the others on the CPU; both arms use the same rule."""
    return "cuda" if name == "skewed" and torch.cuda.is_available() else "cpu"


def aggregate_over_ranks(elapsed_ms, tokens_per_step, steps, world, dist=None, device=None):
    """Whole-job throughput of a timed region: the slowest rank's time (max over
    ranks) and the tokens all ranks processed in it.  Returns (ms, tokens/s)."""
    el = torch.tensor([float(elapsed_ms)], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(el, op=dist.ReduceOp.MAX)
    ms = float(el.item())
    return ms, tokens_per_step * steps * world / (ms / 1e3)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    # the same weights as the native arm (the skewed workload's 22.5 GB of
    # expert weights are drawn on the GPU there; the oracle copies the experts
    # its sample uses to the host)
    W = make_weights(wl["cfg"], 0, weight_device(wl["cfg"]))
    Ts = CONFIGS[wl["cfg"]]["T"]
    budget = args.ref_step_seconds
    for _ in range(args.warmup):
        oracle_sample(W, wl["dtype"], Ts, budget_s=min(1.0, budget))
    vals, cores, what = [], 1, ""
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, cores, what = oracle_sample(W, wl["dtype"], Ts, budget_s=budget)
        vals.append(v)
    el = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {"metric": "fused-MoE layer tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": describe(args.workload)},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": what},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_native(args):
    import mixture_experts_expert_route_b200 as moe
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    wl = WORKLOADS[args.workload]
    name, dtype = wl["cfg"], wl["dtype"]
    cfg = CONFIGS[name]
    Ts = tuple(int(t) for t in args.Ts.split(",")) if args.Ts else cfg["T"]
    k, E, H, I = cfg["k"], cfg["E"], cfg["H"], cfg["I"]
    W = make_weights(name, 0, weight_device(name))
    Wg, Wu, Wd = (t.to(dev, torch.bfloat16) for t in (W.Wg, W.Wu, W.Wd))
    layer = moe.MoELayer(Wg, Wu, Wd, k=k, dtype=dtype)
    del Wg, Wu, Wd
    batches = {T: [make_batch(W, T, 0, b) for b in range(NBATCH)] for T in Ts}
    dev_in = {T: [(x.to(dev), lg.to(dev)) for x, lg in batches[T]] for T in Ts}
    outs = {T: torch.empty((T, H), dtype=torch.bfloat16, device=dev) for T in Ts}
    for T in Ts:
        layer.workspace(T)
    stream = torch.cuda.current_stream()

    # active experts of every batch (for the algorithmic bytes)
    active = {}
    for T in Ts:
        active[T] = []
        for x, lg in dev_in[T]:
            ids, _ = moe.route_topk(lg, k)
            active[T].append(int(torch.unique(ids).numel()))

    # Small token counts (T <= 64) run as CUDA graphs, one per rotating batch:
    # there the layer is a short chain of short kernels and the launch cost
    # on the host would otherwise show.  Larger T launch directly.
    graphs, graph_note = {}, None

    def step(i, ev=None, direct=False):
        for T in Ts:
            if T in graphs and ev is None and not direct:
                graphs[T][i % NBATCH].replay()
                continue
            x, lg = dev_in[T][i % NBATCH]
            layer(x, lg, out=outs[T], events=None if ev is None else ev[T])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if layer.check() != 0:
        raise RuntimeError("device status word reports a fault")
    if not args.no_graphs:
        try:
            for T in Ts:
                if T > GRAPH_MAX_T:
                    continue
                gl = []
                for b in range(NBATCH):
                    x, lg = dev_in[T][b]
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        layer(x, lg, out=outs[T])
                    gl.append(g)
                graphs[T] = gl
            for i in range(args.warmup):
                step(i)
            torch.cuda.synchronize()
            if layer.check() != 0:
                raise RuntimeError("device status word reports a fault")
        except RuntimeError as ex:
            if "status word" in str(ex):
                raise
            graphs.clear()
            graph_note = "graph capture failed, direct launches: " + str(ex).splitlines()[0]

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    uuid = torch.cuda.get_device_properties(dev).uuid
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    # headline region: the layer exactly as a caller runs it (no stage events,
    # so consecutive kernels keep their programmatic-launch overlap)
    clk = ClockSampler(uuid).__enter__()
    atexit.register(clk.__exit__, None, None, None)   # stop the sampler on any exit path
    clk.mark_start()
    t_start.record(stream)
    for i in range(args.steps):
        step(i)
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    if layer.check() != 0:
        raise RuntimeError("device status word reports a fault")
    tokens_per_step = sum(Ts)
    elapsed_ms, value = aggregate_over_ranks(elapsed_ms, tokens_per_step, args.steps, world,
                                             dist if world > 1 else None, dev)

    # stage region: the same steps with CUDA events recorded between the
    # layer's stages on the launching stream (an event between two kernels
    # ends their overlap, so stage times are slightly pessimistic)
    evs = [{T: [torch.cuda.Event(enable_timing=True) for _ in range(7)] for T in Ts}
           for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        step(i, evs[i])
    torch.cuda.synchronize()
    clk.mark_end()     # the headline and stage regions, back to back
    clk.__exit__(None, None, None)

    # per-stage device times from the events recorded inside the timed region
    stage = {T: [[] for _ in range(6)] for T in Ts}
    for i in range(args.steps):
        for T in Ts:
            e = evs[i][T]
            for s in range(6):
                stage[T][s].append(e[s].elapsed_time(e[s + 1]))
    gu_ms = {T: statistics.mean(stage[T][2]) for T in Ts}
    dn_ms = {T: statistics.mean(stage[T][4]) for T in Ts}
    layer_ms = {T: statistics.mean([sum(stage[T][s][j] for s in range(6))
                                    for j in range(args.steps)]) for T in Ts}
    # whole-layer time of each T inside the headline region, from a third pass
    # of single-T steps timed without stage events (graph replays where the
    # headline uses them; the direct-launch time is reported beside it)
    layer_graph_ms = {}
    for T in graphs:
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            graphs[T][i % NBATCH].replay()
        e1.record(stream)
        torch.cuda.synchronize()
        layer_graph_ms[T] = e0.elapsed_time(e1) / args.steps
    layer_pdl_ms = {}
    for T in Ts:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        x, lg = dev_in[T][0]
        layer(x, lg, out=outs[T])
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(args.steps):
            x, lg = dev_in[T][i % NBATCH]
            layer(x, lg, out=outs[T])
        e1.record(stream)
        torch.cuda.synchronize()
        layer_pdl_ms[T] = e0.elapsed_time(e1) / args.steps
    fp8 = dtype == 1
    gu_bytes = {T: statistics.mean(gate_up_bytes(T, k, H, I, a, fp8) for a in active[T])
                for T in Ts}
    hbm, tf, src = peaks()
    tpeak = tf * (2 if fp8 else 1)   # e4m3 dense peak = 2x the measured bf16 peak (nominal ratio)
    # dominant kernel: the gate/up GEMM; its largest launch (the largest T)
    Tr = max(Ts)
    gu_flops = {T: 4.0 * T * k * H * I for T in Ts}      # 2 GEMMs of 2*H*I per assignment
    kname = "grouped_gemm_kernel<%s, gate/up> at T=%d" % ("e4m3" if fp8 else "bf16", Tr)
    if WORKLOADS[args.workload]["bound"] == "hbm":
        achieved = gu_bytes[Tr] / (gu_ms[Tr] / 1e3) / 1e9
        agg = sum(gu_bytes[T] for T in Ts) / (sum(gu_ms[T] for T in Ts) / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved / hbm, 4),
                    "traffic": TRAFFIC.get((args.workload, Tr)), "kernel": kname,
                    "bytes_per_launch": int(gu_bytes[Tr]),
                    "all_T_achieved": round(agg, 1), "all_T_frac": round(agg / hbm, 4),
                    "peak_source": src}
    else:
        achieved = gu_flops[Tr] / (gu_ms[Tr] / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tpeak,
                    "unit": "TFLOP/s", "frac": round(achieved / tpeak, 4),
                    "traffic": TRAFFIC.get((args.workload, Tr)), "kernel": kname,
                    "flops_per_launch": int(gu_flops[Tr]),
                    "peak_source": src + (" (bf16 burst x2 for e4m3)" if fp8 else " (bf16 burst)")}
    wb = 1 if fp8 else 2
    per_T = {}
    for T in Ts:
        a = statistics.mean(active[T])
        layer_bytes = a * 3 * H * I * wb + T * H * 2 * 2 + T * E * 4
        layer_flops = 6.0 * T * k * H * I
        lt = layer_graph_ms.get(T, layer_pdl_ms[T])
        per_T[str(T)] = {"layer_us": round(1e3 * lt, 2),
                         "layer_us_direct": round(1e3 * layer_pdl_ms[T], 2),
                         "cuda_graph": T in graphs,
                         "layer_tflops": round(layer_flops / (lt / 1e3) / 1e12, 1),
                         "layer_tensor_frac": round(layer_flops / (lt / 1e3) / 1e12 / tpeak, 4),
                         "layer_us_staged": round(1e3 * layer_ms[T], 2),
                         "gate_up_us": round(1e3 * gu_ms[T], 2),
                         "down_us": round(1e3 * dn_ms[T], 2),
                         "active_experts": a,
                         "layer_hbm_gbs": round(layer_bytes / (lt / 1e3) / 1e9, 1),
                         "layer_hbm_frac": round(layer_bytes / (lt / 1e3) / 1e9 / hbm, 4)}

    # end to end through the public call, host buffers, copies in the timed
    # region.  Uploads and read-backs run on two streams of their own,
    # double-buffered: the inputs of the next layer call go up while the
    # current one computes, and each output comes back while the next computes.  Every step still moves all
    # of its inputs and outputs across PCIe inside the timed region.
    e2e = None
    if not args.no_e2e:
        hx = {T: [x.pin_memory() for x, _ in batches[T]] for T in Ts}
        hl = {T: [lg.pin_memory() for _, lg in batches[T]] for T in Ts}
        ho = {T: [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
              for T in Ts}
        dx = {T: [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
              for T in Ts}
        dl = {T: [torch.empty((T, E), dtype=torch.float32, device=dev) for _ in range(2)]
              for T in Ts}
        do = {T: [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
              for T in Ts}
        h2d = torch.cuda.Stream(device=dev)
        d2h = torch.cuda.Stream(device=dev)
        jobs = [(T, i) for i in range(args.steps) for T in Ts]

        def run_jobs(jobs, start=None):
            """Pipelined H2D -> layer -> D2H over the job list; on return the
            compute stream waits for the last output to reach the host.  The
            copy streams first wait for `start` (the timed region's opening
            event), so no copy of the region begins before it."""
            done = {}      # slot -> event: layer finished reading/writing that slot
            back = {}      # slot -> event: D2H of that slot's output finished
            if start is not None:
                h2d.wait_event(start)
                d2h.wait_event(start)
            seen = {}
            for T, i in jobs:
                b = seen.get(T, 0)          # alternate the two buffers of each T
                seen[T] = b + 1
                b %= 2
                slot = (T, b)
                with torch.cuda.stream(h2d):
                    if slot in done:
                        h2d.wait_event(done[slot])    # the layer is done with this slot
                    dx[T][b].copy_(hx[T][i % NBATCH], non_blocking=True)
                    dl[T][b].copy_(hl[T][i % NBATCH], non_blocking=True)
                    up = torch.cuda.Event()
                    up.record(h2d)
                stream.wait_event(up)
                if slot in back:
                    stream.wait_event(back[slot])     # output slot read back already
                layer(dx[T][b], dl[T][b], out=do[T][b])
                ev = torch.cuda.Event()
                ev.record(stream)
                done[slot] = ev
                with torch.cuda.stream(d2h):
                    d2h.wait_event(ev)
                    ho[T][b].copy_(do[T][b], non_blocking=True)
                    bk = torch.cuda.Event()
                    bk.record(d2h)
                back[slot] = bk
            for bk in back.values():
                stream.wait_event(bk)

        run_jobs([(T, i) for i in range(args.warmup) for T in Ts])
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        run_jobs(jobs, start=a0)
        a1.record(stream)
        torch.cuda.synchronize()
        _, e_val = aggregate_over_ranks(a0.elapsed_time(a1), tokens_per_step, args.steps, world,
                                        dist if world > 1 else None, dev)
        e2e = {"value": e_val,
               "unit": "tokens/s",
               "h2d_bytes_per_step": sum(T * H * 2 + T * E * 4 for T in Ts),
               "d2h_bytes_per_step": sum(T * H * 2 for T in Ts),
               "copies": "pinned host buffers; uploads and read-backs on two streams, "
                         "double-buffered"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, what = oracle_sample(W, dtype, Ts)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": what}

    launches = args.steps * sum(kernels_per_forward(T, k, fp8, H) for T in Ts)
    if rank == 0:
        line = {"metric": "fused-MoE layer tokens/s", "value": value, "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "fp8" if fp8 else "bf16",
                "data": "synthetic (seeded; random-init weights of the workload's shape)",
                "config": {"workload": describe(args.workload), "global_batch": sum(Ts) * world,
                           "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                           "l2": "inputs larger than L2: expert weights "
                                 f"{3 * E * H * I * wb / 1e9:.2f} GB, {NBATCH} rotating batches",
                           "cuda_graphs": sorted(graphs) if graphs else (graph_note or "none"),
                           "per_T": per_T},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graphs", action="store_true",
                    help="launch every T directly (no CUDA graphs for T <= 64)")
    ap.add_argument("--ref-step-seconds", type=float, default=5.0)
    ap.add_argument("--Ts", default="", help="comma-separated subset of the token counts")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
