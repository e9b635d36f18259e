#!/usr/bin/env python
"""Benchmark of the fused MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all]
                    [--impl native|reference]

A step is one pass of the whole layer (route -> permute -> [gather] -> gate/up
GEMM -> [FP8 h quant] -> down GEMM -> combine) over one
batch of every token count of a workload, e.g. T = 1, 4, 16, 64 for the
decode workload (H=4096, I=14336, E=8, top-2, bf16).  Inputs are seeded
synthetic tensors; the expert weights are larger than the 126 MB L2 and four
input batches rotate between steps.

With the default ``--workload all`` the headline (``value``, ``roofline``,
``e2e``, ``cpu_baseline``) is the decode workload, and the same JSON line
carries a ``workloads`` block with the other workloads measured the same way
on the same GPU: fine-grained prefill (T=4096), FP8 (T = 1, 32, 256, 2048) and
the skewed large-expert-count layer (T=8192).

Metric: layer tokens/s (whole job, all ranks).  N > 1 runs independent
replicas, one per GPU (the layer is single-GPU; there is no data-path
collective), timed on the device and reduced as the max over ranks.
``--impl reference`` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import atexit
import hashlib
import json
import os
import platform
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
    # the prefill layer serving four rank-16 adapters (multi-LoRA)
    "prefill_lora": dict(cfg="prefill", dtype=0, bound="tensor", lora=(4, 16)),
}
HEADLINE = "decode"
NBATCH = 4
GRAPH_MAX_T = 64       # token counts that --graphs runs as CUDA graphs
# DRAM bytes (read + write) of one gate/up launch, from an ncu capture made
# offline (profiles/), keyed by (workload, T).  Each value records the hash of
# the GEMM's source files it was captured with; the bench reports it only
# while the sources still hash the same, and null (stale) otherwise.
GEMM_SOURCES = ("mixture_experts_expert_route_b200/csrc/grouped_gemm.cu",
                "mixture_experts_expert_route_b200/csrc/common.cuh")
# DRAM bytes (read + write) of one gate/up launch, from ncu captures of the
# committed profiling mode (`--calls N`, cold cache), keyed by (workload, T);
# each entry names the GEMM code it was taken on and is reported only while
# that code is unchanged.  The full-size skewed launch is captured with the
# three single-pass metrics only (duration, DRAM read and write bytes).
TRAFFIC = {
    ("decode", 64): {"bytes": 1885457152, "gemm_src": "b033dbd28027",
                     "capture": "profiles/grouped_gemm_decode_T64.md"},
    ("prefill", 4096): {"bytes": 1379271936, "gemm_src": "b033dbd28027",
                        "capture": "profiles/grouped_gemm_prefill_T4096.md"},
    ("fp8", 2048): {"bytes": 876748032, "gemm_src": "b033dbd28027",
                    "capture": "profiles/grouped_gemm_fp8_T2048.md"},
    ("skewed", 8192): {"bytes": 15107015168, "gemm_src": "b033dbd28027",
                       "capture": "profiles/grouped_gemm_skewed_T8192.md"},
    ("prefill_lora", 4096): {"bytes": 1460490752, "gemm_src": "b033dbd28027",
                             "capture": "profiles/grouped_gemm_prefill_lora_T4096.md"},
}
NO_TRAFFIC = {}
SMALL_T, CHUNK = 128, 2048   # the library's single-CTA route+permute limits
SMALL_AMAX = 32768           # x elements the single-CTA kernel also takes amax(x) of


def strip_comments(src):
    """C/C++ source without comments, trailing blanks and empty lines (string
    and character literals kept), so that the hash below follows the code."""
    out, i, n, quote = [], 0, len(src), None
    while i < n:
        c = src[i]
        if quote:
            out.append(c)
            if c == "\\" and i + 1 < n:
                out.append(src[i + 1])
                i += 2
                continue
            if c == quote:
                quote = None
            i += 1
        elif c in "\"'":
            quote = c
            out.append(c)
            i += 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "\n".join(ln.rstrip() for ln in "".join(out).splitlines() if ln.strip())


def gemm_source_hash():
    """Hash of the GEMM's code (comments stripped): the key under which a
    traffic capture stays valid."""
    h = hashlib.sha256()
    for p in GEMM_SOURCES:
        with open(os.path.join(ROOT, p)) as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:12]


def traffic_for(workload, T):
    """(bytes or None, note) for the roofline's `traffic` field."""
    rec = TRAFFIC.get((workload, T))
    if rec is None:
        return None, NO_TRAFFIC.get(workload, "no ncu capture of this GEMM code")
    if rec["gemm_src"] != gemm_source_hash():
        return None, f"stale: captured on GEMM sources {rec['gemm_src']} ({rec['capture']})"
    return rec["bytes"], f"ncu capture offline ({rec['capture']}), GEMM sources {rec['gemm_src']}"


def describe(name):
    wl = WORKLOADS[name]
    c = CONFIGS[wl["cfg"]]
    d = "fp8 e4m3" if wl["dtype"] else "bf16"
    lo = f", {wl['lora'][0]} adapters of rank {wl['lora'][1]}" if wl.get("lora") else ""
    return (f"{name} {d} H={c['H']} I={c['I']} E={c['E']} top-{c['k']} "
            f"T={','.join(str(t) for t in c['T'])}{lo}")


def gemm_token_cap(T, k, E):
    """The GEMMs' token-tile cap: twice the mean tokens per expert in steps of
    16 (16..256), rounded to 32 above 64 (CTA-pair tiles)."""
    n = max(16, ((2 * T * k + E - 1) // E + 15) // 16 * 16)
    if n > 64:
        n = (n + 31) // 32 * 32
    return min(n, 256)


def kernels_per_forward(T, k, E, fp8, H, lora=False):
    """Kernels one moe_forward launches."""
    A = T * k
    small = T <= SMALL_T and A <= CHUNK
    if small:
        n = 1                                   # fused route + permute
    elif A <= CHUNK:
        n = 2                                   # route, single-CTA permute
    else:
        n = 3                                   # route, count, scan + scatter
    # FP8: amax(x) and the codes of x (in the route kernel for small batches)
    n += 2 if fp8 and not (small and T * H <= SMALL_AMAX) else 0
    # gather (pair tiles and adapter layers; else in the GEMM), adapter shrinks
    n += 1 if gemm_token_cap(T, k, E) > 64 or lora else 0
    n += 2 if lora else 0
    n += 1                                      # gate/up GEMM
    n += 1 if fp8 else 0                        # h quantisation
    n += 2                                      # down GEMM + combine (or finalize)
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


def sustained_bf16():
    """bf16 dense peak under the power cap (a GEMM loop of seconds): the
    measured figure when the box has one, else the pool's earlier
    measurement (~1.4 PFLOP/s at ~1.3 GHz with sw_power_cap active)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops_sustained" in d:
            return d["bf16_tflops_sustained"], "measured"
    return 1400.0, "fallback"


def gate_up_bytes(T, k, H, I, active, fp8):
    """Algorithmic bytes of one gate/up launch: the active experts' W_g and W_u,
    the T tokens' activation rows read (each once), the T*k rows of h written."""
    wb = 1 if fp8 else 2
    return active * 2 * H * I * wb + T * H * wb + T * k * I * 2


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def oracle_sample(W, dtype, T, budget_s=12.0, max_tokens=None, threads=None):
    """The oracle on a bounded sample: tokens of batch 0 with T tokens, one
    call per `threads` tokens, until the time budget is spent.  Only the
    experts the first `max_tokens` tokens use are copied to the host.  The
    FP8 oracle needs every h row for its scale, so it runs whole batches.
    Returns (tokens/s, threads used, description)."""
    import numpy as np
    import oracle
    x, logits = make_batch(W, T, 0, 0)
    n_pool = T if max_tokens is None else min(T, max_tokens)
    x, logits = x[:n_pool], logits[:n_pool]
    ids, w = oracle.route_topk(logits, W.k)
    used = sorted(set(int(e) for e in np.unique(ids)))
    remap = np.zeros(W.E, np.int32)
    remap[used] = np.arange(len(used), dtype=np.int32)
    Wg = W.Wg[used].cpu().to(torch.bfloat16)
    Wu = W.Wu[used].cpu().to(torch.bfloat16)
    Wd = W.Wd[used].cpu().to(torch.bfloat16)
    lid = remap[ids]
    saved = oracle.num_threads()
    if threads is not None:
        oracle.set_num_threads(threads)
    used_threads = oracle.num_threads()
    try:
        n, t0 = 0, time.perf_counter()
        step = max(1, used_threads)
        while True:
            if dtype == 0:
                toks = [(n + i) % n_pool for i in range(step)]
                oracle.moe_layer(x, lid, w, Wg, Wu, Wd, tokens=toks)
                n += step
            else:
                oracle.moe_layer_fp8(x, lid, w, Wg, Wu, Wd)
                n += n_pool
            if time.perf_counter() - t0 >= budget_s:
                break
        el = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(saved)
    what = (f"oracle layer on {n} tokens from the first {n_pool} of the T={T} batch "
            f"({budget_s:.0f} s budget), {len(used)} experts, {used_threads} threads")
    return n / el, used_threads, what


def cpu_baseline(W, dtype, T, budget_s, max_tokens=None, single_thread=True):
    v, cores, what = oracle_sample(W, dtype, T, budget_s, max_tokens)
    out = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": what,
           "cpu_model": cpu_model()}
    if single_thread:
        v1, _, what1 = oracle_sample(W, dtype, T, budget_s, max_tokens, threads=1)
        out["single_thread_value"] = v1
        out["single_thread_sample"] = what1
    return out


# oracle sample per workload: (T of the batch it draws tokens from, the
# token pool: only the first tokens, whose experts are copied to the host;
# None = the whole batch).  The FP8 oracle runs whole batches (its h scale
# needs every row), hence its small batch.
ORACLE_SAMPLE = {"decode": (64, None), "prefill": (4096, 512), "fp8": (32, None),
                 "skewed": (8192, 32), "prefill_lora": (4096, 512)}


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


def headline_name(args):
    return HEADLINE if args.workload == "all" else args.workload


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = headline_name(args)
    if name == "split":
        name = SPLIT["cfg"]     # the split computes the decode layer
    wl = WORKLOADS[name]
    # the same weights as the native arm (the skewed workload's 22.5 GB of
    # expert weights are drawn on the GPU there; the oracle copies the experts
    # its sample uses to the host)
    W = make_weights(wl["cfg"], 0, weight_device(wl["cfg"]))
    T, pool = ORACLE_SAMPLE[name]
    budget = args.ref_step_seconds
    for _ in range(args.warmup):
        oracle_sample(W, wl["dtype"], T, budget_s=min(1.0, budget), max_tokens=pool)
    vals, cores, what = [], 1, ""
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, cores, what = oracle_sample(W, wl["dtype"], T, budget_s=budget, max_tokens=pool)
        vals.append(v)
    el = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {"metric": "fused-MoE layer tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": describe(name)},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": what, "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class Bench:
    """One workload on this rank's GPU: packed layer, rotating input batches,
    the timed regions and the derived roofline figures."""

    def __init__(self, name, args, dev, dist, world, Ts=None):
        import mixture_experts_expert_route_b200 as moe
        self.moe, self.name, self.args, self.dev, self.dist, self.world = \
            moe, name, args, dev, dist, world
        wl = WORKLOADS[name]
        self.dtype = wl["dtype"]
        self.fp8 = self.dtype == 1
        cfg = CONFIGS[wl["cfg"]]
        self.Ts = Ts or cfg["T"]
        self.k, self.E, self.H, self.I = cfg["k"], cfg["E"], cfg["H"], cfg["I"]
        self.W = make_weights(wl["cfg"], 0, weight_device(wl["cfg"]))
        Wg, Wu, Wd = (t.to(dev, torch.bfloat16) for t in (self.W.Wg, self.W.Wu, self.W.Wd))
        self.layer = moe.MoELayer(Wg, Wu, Wd, k=self.k, dtype=self.dtype)
        del Wg, Wu, Wd
        self.lora, self.adapters = None, {}
        if wl.get("lora"):
            from workloads import adapter_ids, make_lora
            n, r = wl["lora"]
            lw = make_lora(self.E, self.H, self.I, n_adapters=n, rank=r, seed=1)
            self.lora = moe.Lora(*(m.to(dev) for m in (lw.Ag, lw.Bg, lw.Au, lw.Bu, lw.Ad,
                                                         lw.Bd)), lw.scale)
            self.lora_rank = r
            self.adapters = {T: adapter_ids(T, n, seed=T).to(dev) for T in self.Ts}
        self.batches = {T: [make_batch(self.W, T, 0, b) for b in range(NBATCH)]
                        for T in self.Ts}
        self.dev_in = {T: [(x.to(dev), lg.to(dev)) for x, lg in self.batches[T]]
                       for T in self.Ts}
        self.outs = {T: torch.empty((T, self.H), dtype=torch.bfloat16, device=dev)
                     for T in self.Ts}
        for T in self.Ts:
            self.layer.workspace(T)
        self.stream = torch.cuda.current_stream()
        self.active = {}
        for T in self.Ts:
            self.active[T] = []
            for x, lg in self.dev_in[T]:
                ids, _ = moe.route_topk(lg, self.k)
                self.active[T].append(int(torch.unique(ids).numel()))
        self.graphs, self.graph_note = {}, None

    def release(self):
        for gl in self.graphs.values():
            for g in gl:
                g.reset()
        self.graphs.clear()
        del self.layer, self.dev_in, self.outs, self.batches
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    def check(self):
        if self.layer.check() != 0:
            raise RuntimeError(f"{self.name}: device status word reports a fault")

    def call(self, T, x, lg, out, ev=None):
        if self.lora is None:
            return self.layer(x, lg, out=out, events=ev)
        return self.moe.forward(self.dtype, x, lg, self.layer.packed, self.layer.scales, self.E,
                                self.I, self.k, out=out, status=self.layer.status,
                                ws=self.layer.workspace(T), events=ev, lora=self.lora,
                                adapter=self.adapters[T])

    def step(self, i, ev=None, direct=False):
        for T in self.Ts:
            if T in self.graphs and ev is None and not direct:
                self.graphs[T][i % NBATCH].replay()
                continue
            x, lg = self.dev_in[T][i % NBATCH]
            self.call(T, x, lg, self.outs[T], ev=None if ev is None else ev[T])

    def capture_graphs(self):
        """With --graphs, small token counts (T <= 64) run as CUDA graphs, one
        per rotating batch.  Off by default: measured on B200, the replays were
        slower on the device than direct launches (decode T=1 128.1 vs 124.6 us,
        FP8 T=1 52.2 vs 47.3 us; the layer is device-bound, and the direct
        chain keeps more of the programmatic-launch overlap)."""
        if not self.args.graphs:
            return
        try:
            for T in self.Ts:
                if T > GRAPH_MAX_T:
                    continue
                gl = []
                for b in range(NBATCH):
                    x, lg = self.dev_in[T][b]
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        self.call(T, x, lg, self.outs[T])
                    gl.append(g)
                self.graphs[T] = gl
            for i in range(self.args.warmup):
                self.step(i)
            torch.cuda.synchronize()
            self.check()
        except RuntimeError as ex:
            if "status word" in str(ex):
                raise
            self.graphs.clear()
            self.graph_note = "graph capture failed, direct launches: " + str(ex).splitlines()[0]

    def measure(self, clk):
        """Headline region (the layer as a caller runs it), stage region
        (events between the stages) and per-T regions.  Returns a result dict."""
        args, dist, world = self.args, self.dist, self.world
        for i in range(args.warmup):
            self.step(i)
        torch.cuda.synchronize()
        self.check()
        self.capture_graphs()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        clk.mark_start()     # the clock window: headline, stage and per-T regions
        t_start.record(self.stream)
        for i in range(args.steps):
            self.step(i)
        t_end.record(self.stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        elapsed_ms = t_start.elapsed_time(t_end)
        self.check()
        tokens_per_step = sum(self.Ts)
        elapsed_ms, value = aggregate_over_ranks(elapsed_ms, tokens_per_step, args.steps, world,
                                                 dist, self.dev)

        # stage region: the same steps with CUDA events recorded between the
        # layer's stages on the launching stream (an event between two kernels
        # ends their overlap, so stage times are slightly pessimistic)
        evs = [{T: [torch.cuda.Event(enable_timing=True) for _ in range(7)] for T in self.Ts}
               for _ in range(args.steps)]
        torch.cuda.synchronize()
        for i in range(args.steps):
            self.step(i, evs[i])
        torch.cuda.synchronize()
        stage = {T: [[] for _ in range(6)] for T in self.Ts}
        for i in range(args.steps):
            for T in self.Ts:
                e = evs[i][T]
                for s in range(6):
                    stage[T][s].append(e[s].elapsed_time(e[s + 1]))
        gu_ms = {T: statistics.mean(stage[T][2]) for T in self.Ts}
        dn_ms = {T: statistics.mean(stage[T][4]) for T in self.Ts}
        layer_ms = {T: statistics.mean([sum(stage[T][s][j] for s in range(6))
                                        for j in range(args.steps)]) for T in self.Ts}
        # whole-layer time of each T on its own (graph replays where the
        # headline uses them; the direct-launch time is reported beside it)
        layer_graph_ms = {}
        for T in self.graphs:
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            for i in range(args.steps):
                self.graphs[T][i % NBATCH].replay()
            e1.record(self.stream)
            torch.cuda.synchronize()
            layer_graph_ms[T] = e0.elapsed_time(e1) / args.steps
        layer_direct_ms = {}
        for T in self.Ts:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            x, lg = self.dev_in[T][0]
            self.call(T, x, lg, self.outs[T])
            torch.cuda.synchronize()
            e0.record(self.stream)
            for i in range(args.steps):
                x, lg = self.dev_in[T][i % NBATCH]
                self.call(T, x, lg, self.outs[T])
            e1.record(self.stream)
            torch.cuda.synchronize()
            layer_direct_ms[T] = e0.elapsed_time(e1) / args.steps
        clk.mark_end()
        self.check()
        return dict(elapsed_ms=elapsed_ms, value=value, gu_ms=gu_ms, dn_ms=dn_ms,
                    layer_ms=layer_ms, layer_graph_ms=layer_graph_ms,
                    layer_direct_ms=layer_direct_ms)

    def report(self, r, clocks=None):
        """roofline + per-T figures of a measure() result.  A tensor-bound
        workload whose timed region ran under the power cap (sw_power_cap
        active in `clocks`) is compared with the sustained peak, the others
        with the burst peak; the line carries the other fraction too."""
        k, E, H, I, fp8, Ts = self.k, self.E, self.H, self.I, self.fp8, self.Ts
        hbm, tf, src = peaks()
        burst = tf * (2 if fp8 else 1)   # e4m3 dense peak = 2x the measured bf16 peak (nominal)
        capped = bool(clocks) and "sw_power_cap" in clocks.get("reasons", [])
        if capped:
            sus, ssrc = sustained_bf16()
            tpeak = sus * (2 if fp8 else 1)
            peak_kind = f"sustained ({ssrc}; sw_power_cap active in the timed region)"
        else:
            tpeak, peak_kind = burst, "burst"
        gu_ms = r["gu_ms"]
        gu_bytes = {T: statistics.mean(gate_up_bytes(T, k, H, I, a, fp8)
                                       for a in self.active[T]) for T in Ts}
        gu_flops = {T: 4.0 * T * k * H * I for T in Ts}   # 2 GEMMs of 2*H*I per assignment
        Tr = max(Ts)
        kname = "grouped_gemm_kernel<%s, gate/up> at T=%d" % ("e4m3" if fp8 else "bf16", Tr)
        traffic, tnote = traffic_for(self.name, Tr)
        if WORKLOADS[self.name]["bound"] == "hbm":
            achieved = gu_bytes[Tr] / (gu_ms[Tr] / 1e3) / 1e9
            agg = sum(gu_bytes[T] for T in Ts) / (sum(gu_ms[T] for T in Ts) / 1e3) / 1e9
            roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                        "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": traffic,
                        "traffic_note": tnote, "kernel": kname,
                        "bytes_per_launch": int(gu_bytes[Tr]),
                        "all_T_achieved": round(agg, 1), "all_T_frac": round(agg / hbm, 4),
                        "peak_source": src + " (HBM copy)"}
        else:
            achieved = gu_flops[Tr] / (gu_ms[Tr] / 1e3) / 1e12
            roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tpeak,
                        "unit": "TFLOP/s", "frac": round(achieved / tpeak, 4),
                        "traffic": traffic, "traffic_note": tnote, "kernel": kname,
                        "flops_per_launch": int(gu_flops[Tr]), "peak_kind": peak_kind,
                        "frac_vs_burst": round(achieved / burst, 4),
                        "peak_source": src + (" (bf16 x2 for e4m3)" if fp8 else " (bf16)")}
        wb = 1 if fp8 else 2
        per_T = {}
        for T in Ts:
            a = statistics.mean(self.active[T])
            layer_bytes = a * 3 * H * I * wb + T * H * 2 * 2 + T * E * 4
            layer_flops = 6.0 * T * k * H * I
            if self.lora is not None:
                # each assignment of an adapted token: shrink and expand of its
                # own adapter on the three matrices (2r(H+I) MACs each)
                n_ad = int((self.adapters[T] >= 0).sum().item())
                layer_flops += 6.0 * n_ad * k * 2 * self.lora_rank * (H + I)
            # one token count: the primary timed region is that T's layer time (the
            # per-T region repeats it later, on a warmer, power-capped GPU)
            lt = (r["elapsed_ms"] / self.args.steps if len(Ts) == 1
                  else r["layer_graph_ms"].get(T, r["layer_direct_ms"][T]))
            per_T[str(T)] = {
                "layer_us": round(1e3 * lt, 2),
                "layer_us_direct": round(1e3 * r["layer_direct_ms"][T], 2),
                "cuda_graph": T in self.graphs,
                "tokens_per_s": round(T / (lt / 1e3), 1),
                "layer_tflops": round(layer_flops / (lt / 1e3) / 1e12, 1),
                "layer_tensor_frac": round(layer_flops / (lt / 1e3) / 1e12 / tpeak, 4),
                "layer_hbm_gbs": round(layer_bytes / (lt / 1e3) / 1e9, 1),
                "layer_hbm_frac": round(layer_bytes / (lt / 1e3) / 1e9 / hbm, 4),
                "layer_us_staged": round(1e3 * r["layer_ms"][T], 2),
                "gate_up_us": round(1e3 * gu_ms[T], 2),
                "gate_up_tensor_frac": round(gu_flops[T] / (gu_ms[T] / 1e3) / 1e12 / tpeak, 4),
                "gate_up_hbm_frac": round(gu_bytes[T] / (gu_ms[T] / 1e3) / 1e9 / hbm, 4),
                "down_us": round(1e3 * r["dn_ms"][T], 2),
                "active_experts": a}
        return roofline, per_T

    def e2e(self):
        """End to end through the public call, host buffers, copies in the timed
        region.  Uploads and read-backs run on two streams of their own,
        double-buffered: the inputs of the next layer call go up while the
        current one computes, and each output comes back while the next
        computes.  Every step still moves all of its inputs and outputs across
        PCIe inside the timed region."""
        args, dev, Ts, H, E = self.args, self.dev, self.Ts, self.H, self.E
        hx = {T: [x.pin_memory() for x, _ in self.batches[T]] for T in Ts}
        hl = {T: [lg.pin_memory() for _, lg in self.batches[T]] for T in Ts}
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
        stream, layer = self.stream, self.layer

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
        if self.dist:
            self.dist.barrier()
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        run_jobs([(T, i) for i in range(args.steps) for T in Ts], start=a0)
        a1.record(stream)
        torch.cuda.synchronize()
        self.check()
        _, e_val = aggregate_over_ranks(a0.elapsed_time(a1), sum(Ts), args.steps, self.world,
                                        self.dist, dev)
        return {"value": e_val,
                "unit": "tokens/s",
                "h2d_bytes_per_step": sum(T * H * 2 + T * E * 4 for T in Ts),
                "d2h_bytes_per_step": sum(T * H * 2 for T in Ts),
                "copies": "pinned host buffers; uploads and read-backs on two streams, "
                          "double-buffered"}

    def launches(self):
        return self.args.steps * sum(kernels_per_forward(T, self.k, self.E, self.fp8, self.H,
                                                         self.lora is not None)
                                     for T in self.Ts)


# The CPU/GPU expert split (FIDDLER): the decode workload's experts
# (Mixtral-8x7B-shaped) with half of them resident on the GPU (the ones a
# profiling batch hits most), the others in host memory, run on the host or
# copied to one of four staging slots per the measured latency model; decode
# batches (T = 1..64) and prefill chunks (T = 512 and 2048, ~128 and ~512
# tokens per expert).
SPLIT = dict(cfg="decode", budget=4, n_stage=4, profile_T=256, T=(1, 4, 16, 64, 512, 2048))
# "dynamic": the page's per-expert rule; "balanced": host and link in parallel
SPLIT_POLICIES = (("dynamic", 0), ("balanced", 3), ("all_cpu", 1), ("all_staged", 2))


def host_read_gbs(seconds=1.0):
    """Host memory read bandwidth: a torch sum over 1 GiB of float32 on all
    cores (the best of a few passes)."""
    a = torch.ones(1 << 28, dtype=torch.float32)
    best = 0.0
    t_end = time.perf_counter() + seconds
    while True:
        t0 = time.perf_counter()
        a.sum()
        best = max(best, a.numel() * 4 / (time.perf_counter() - t0) / 1e9)
        if time.perf_counter() > t_end:
            break
    del a
    return best


class SplitBench:
    """moe_split_forward on the decode workload: per token count, the layer
    under the dynamic plan and under the two fixed policies (every
    non-resident expert on the host, or every one copied in)."""

    def __init__(self, args, dev, Ts=None):
        import mixture_experts_expert_route_b200 as moe
        self.moe, self.args, self.dev = moe, args, dev
        cfg = CONFIGS[SPLIT["cfg"]]
        self.Ts = Ts or SPLIT["T"]
        self.k, self.E, self.H, self.I = cfg["k"], cfg["E"], cfg["H"], cfg["I"]
        W = make_weights(SPLIT["cfg"], 0, "cuda")
        master = [t.cpu() for t in (W.Wg, W.Wu, W.Wd)]
        W.Wg = W.Wu = W.Wd = None
        torch.cuda.empty_cache()
        self.W = W
        # offline placement from a profiling batch's expert hits
        xp, lp = make_batch(W, SPLIT["profile_T"], 1, 0)
        ids, _ = moe.route_topk(lp.to(dev), self.k)
        hits = torch.bincount(ids.flatten().long(), minlength=self.E).cpu().tolist()
        self.resident = moe.split_place(hits, SPLIT["budget"])
        self.layer = moe.SplitLayer(*master, self.k, self.resident, n_stage=SPLIT["n_stage"],
                                    device=dev)
        del master
        self.dev_in = {T: [tuple(t.to(dev) for t in make_batch(W, T, 0, b))
                           for b in range(NBATCH)] for T in self.Ts}
        self.outs = {T: torch.empty((T, self.H), dtype=torch.bfloat16, device=dev)
                     for T in self.Ts}
        # tokens per expert of each batch (for the launch count of a call)
        self.counts = {T: [torch.bincount(moe.route_topk(lg, self.k)[0].flatten().long(),
                                          minlength=self.E).cpu().tolist()
                           for _, lg in self.dev_in[T]] for T in self.Ts}

    def measure(self, clk):
        args, layer = self.args, self.layer
        res = {}
        expert_bytes = 3 * self.H * self.I * 2
        clk.mark_start()
        for T in self.Ts:
            for pname, pol in SPLIT_POLICIES:
                for i in range(args.warmup):
                    x, lg = self.dev_in[T][i % NBATCH]
                    layer(x, lg, out=self.outs[T], policy=pol)
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                places = {"resident": 0, "staged": 0, "cpu": 0}
                launches = 0
                # each call is bracketed by its own events (a call waits for the
                # routing once, so back-to-back calls do not overlap anyway); the
                # median of the calls is reported beside the mean, because the
                # host's cores are shared with other work on the machine
                evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(args.steps)]
                e0.record()
                for i in range(args.steps):
                    x, lg = self.dev_in[T][i % NBATCH]
                    evs[i][0].record()
                    layer(x, lg, out=self.outs[T], policy=pol)
                    evs[i][1].record()
                    w = list(layer.where)
                    places["resident"] += w.count(self.moe.SPLIT_RESIDENT)
                    places["staged"] += w.count(self.moe.SPLIT_STAGED)
                    places["cpu"] += w.count(self.moe.SPLIT_CPU)
                    launches += self.kernels_per_call(T, w, self.counts[T][i % NBATCH])
                e1.record()
                torch.cuda.synchronize()
                if layer.check() != 0:
                    raise RuntimeError("split: device status word reports a fault")
                per_call = [a.elapsed_time(b) for a, b in evs]
                ms = statistics.median(per_call)
                mean = {key: v / args.steps for key, v in places.items()}
                res[(T, pname)] = dict(ms=ms, mean_ms=e0.elapsed_time(e1) / args.steps,
                                       places=mean, launches=launches,
                                       bytes={key: v * expert_bytes for key, v in mean.items()})
        clk.mark_end()
        return res

    def kernels_per_call(self, T, where, counts):
        """Kernels one moe_split_forward launches: route, slot map, the
        permutation (one kernel up to 2048 assignments, else three), per GPU
        group of experts (resident, staged) a gate/up and a down GEMM plus a
        gather kernel for CTA-pair tiles, and the combine."""
        A = T * self.k
        n = 2 + (1 if A <= CHUNK else 2) + 1
        for kind in (self.moe.SPLIT_RESIDENT, self.moe.SPLIT_STAGED):
            ex = [e for e in range(self.E) if where[e] == kind]
            if not ex:
                continue
            n += 2
            if gemm_token_cap(sum(counts[e] for e in ex), 1, len(ex)) > 64:
                n += 1
        return n

    def report(self, res, clocks):
        hbm, _, src = peaks()
        c = self.layer.costs
        expert_bytes = 3 * self.H * self.I * 2
        link = expert_bytes / (c.xfer_us * 1e-6) / 1e9           # GB/s, measured copy
        host_bw = host_read_gbs()
        per_T = {}
        for T in self.Ts:
            d = res[(T, "dynamic")]
            b = d["bytes"]
            # the host experts' weights stream from host memory while the GPU
            # copies the staged ones over the link and streams the resident ones
            ideal_ms = max(b["cpu"] / (host_bw * 1e9),
                           b["staged"] / (link * 1e9) + (b["resident"] + b["staged"]) /
                           (hbm * 1e9)) * 1e3
            entry = {"layer_us": round(1e3 * d["ms"], 1),
                     "layer_us_mean": round(1e3 * d["mean_ms"], 1),
                     "tokens_per_s": round(T / (d["ms"] / 1e3), 1),
                     "experts_per_call": {k2: round(v, 2) for k2, v in d["places"].items()},
                     "ideal_us": round(1e3 * ideal_ms, 1),
                     "frac_of_ideal": round(ideal_ms / d["ms"], 4)}
            for pname, _ in SPLIT_POLICIES[1:]:
                o = res[(T, pname)]
                entry[f"{pname}_us"] = round(1e3 * o["ms"], 1)
                entry[f"speedup_vs_{pname}"] = round(o["ms"] / d["ms"], 3)
            bal = res[(T, "balanced")]
            bb = bal["bytes"]
            ideal_b = max(bb["cpu"] / (host_bw * 1e9),
                          bb["staged"] / (link * 1e9) + (bb["resident"] + bb["staged"]) /
                          (hbm * 1e9)) * 1e3
            entry["balanced_experts_per_call"] = {k2: round(v, 2)
                                                  for k2, v in bal["places"].items()}
            entry["balanced_frac_of_ideal"] = round(ideal_b / bal["ms"], 4)
            per_T[str(T)] = entry
        total_ms = sum(res[(T, "dynamic")]["ms"] for T in self.Ts)
        total_bal = sum(res[(T, "balanced")]["ms"] for T in self.Ts)
        return {"workload": f"split bf16 H={self.H} I={self.I} E={self.E} top-{self.k} "
                            f"T={','.join(str(t) for t in self.Ts)}, "
                            f"{SPLIT['budget']} experts resident, {SPLIT['n_stage']} staging slots",
                "value": round(sum(self.Ts) / (total_ms / 1e3), 1), "unit": "tokens/s",
                "ms_per_step": round(total_ms, 3), "dtype": "bf16",
                "policy": "dynamic (the per-expert rule); balanced_* fields: the host/link "
                          "balanced plan; *_us: median over the timed calls",
                "value_balanced": round(sum(self.Ts) / (total_bal / 1e3), 1),
                "resident": [int(v) for v in self.resident],
                "costs": {"cpu_us": round(c.cpu_us, 1),
                          "cpu_us_per_token": round(c.cpu_us_per_token, 1),
                          "xfer_us": round(c.xfer_us, 1), "gpu_us": c.gpu_us,
                          "gpu_us_per_token": c.gpu_us_per_token},
                "host_isa": ["portable", "avx512_bf16", "amx_bf16"][self.moe.host_isa()],
                "host_threads": os.cpu_count(), "cpu_model": cpu_model(),
                "roofline": {"bound": "host memory | host link | hbm",
                             "host_read_gbs": round(host_bw, 1),
                             "link_h2d_gbs": round(link, 1), "hbm_gbs": hbm,
                             "peak_source": src + " (HBM); host and link measured here",
                             "note": "ideal = max(host experts' bytes / host read bandwidth, "
                                     "staged bytes / link + GPU experts' bytes / HBM)"},
                "per_T": per_T, "clocks": clocks,
                "gpu_launches": sum(res[(T, "dynamic")]["launches"] for T in self.Ts),
                "gpu_launches_note": "timed calls of the dynamic policy: route, slot map, "
                                     "permutation, gate/up and down GEMMs (+ gather for pair "
                                     "tiles) per GPU group of experts, combine"}

    def host_kernel_rates(self, ns=(1, 16, 64, 128, 512)):
        """moe_host_expert_ffn alone on expert 0 (all host threads, the best of
        three runs per token count): weight bytes and FLOPs per second."""
        H, I = self.H, self.I
        out = {}
        for n in ns:
            x = torch.randn(n, H, generator=torch.Generator().manual_seed(n)).to(torch.bfloat16)
            w = torch.ones(n)
            self.moe.host_expert_ffn(self.layer.host_weights[0], x, w)
            best = 1e9
            for _ in range(3):
                t0 = time.perf_counter()
                self.moe.host_expert_ffn(self.layer.host_weights[0], x, w)
                best = min(best, time.perf_counter() - t0)
            out[str(n)] = {"ms": round(best * 1e3, 3),
                           "weight_gbs": round(3 * H * I * 2 / best / 1e9, 1),
                           "tflops": round(6.0 * n * H * I / best / 1e12, 2)}
        return out

    def release(self):
        del self.layer, self.dev_in, self.outs
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def run_split(args, dev, uuid):
    c = ClockSampler(uuid).__enter__()
    sb = SplitBench(args, dev)
    r = sb.measure(c)
    c.__exit__(None, None, None)
    blk = sb.report(r, c.summary())
    blk["host_kernel"] = sb.host_kernel_rates()
    sb.release()
    return blk


def run_native(args):
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
    uuid = torch.cuda.get_device_properties(dev).uuid
    clk = ClockSampler(uuid).__enter__()
    atexit.register(clk.__exit__, None, None, None)   # stop the sampler on any exit path
    head = headline_name(args)
    Ts = tuple(int(t) for t in args.Ts.split(",")) if args.Ts else None
    if head == "split":
        # one GPU and its host: with several ranks the host cores would be
        # shared between them, so only rank 0 measures
        clk.__exit__(None, None, None)
        if rank == 0:
            blk = run_split(args, dev, uuid)
            print(json.dumps({"metric": "CPU/GPU split layer tokens/s", **blk,
                              "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                              "higher_is_better": True,
                              "note": f"measured on rank 0 of {world}" if world > 1 else None}),
                  flush=True)
        if dist:
            dist.destroy_process_group()   # no barrier: rank 0's run outlasts the timeout
        return

    b = Bench(head, args, dev, dist, world, Ts)
    r = b.measure(clk)
    clk.__exit__(None, None, None)
    head_clocks = clk.summary()
    roofline, per_T = b.report(r, head_clocks)
    e2e = None if args.no_e2e else b.e2e()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        T, pool = ORACLE_SAMPLE[head]
        cpu = cpu_baseline(b.W, b.dtype, T, args.cpu_seconds, pool)
    line = {"metric": "fused-MoE layer tokens/s", "value": r["value"], "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": r["elapsed_ms"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp8" if b.fp8 else "bf16",
            "data": "synthetic (seeded; random-init weights of the workload's shape)",
            "config": {"workload": describe(head), "global_batch": sum(b.Ts) * world,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2: expert weights "
                             f"{3 * b.E * b.H * b.I * (1 if b.fp8 else 2) / 1e9:.2f} GB, "
                             f"{NBATCH} rotating batches",
                       "cuda_graphs": sorted(b.graphs) if b.graphs else (b.graph_note or "none"),
                       "per_T": per_T},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": b.launches(), "clocks": head_clocks}
    b.release()

    if args.workload == "all":
        blocks = {}
        for name in [n for n in WORKLOADS if n != head]:
            c = ClockSampler(uuid).__enter__()
            wb = Bench(name, args, dev, dist, world)
            rr = wb.measure(c)
            c.__exit__(None, None, None)
            wclocks = c.summary()
            rl, pt = wb.report(rr, wclocks)
            blk = {"workload": describe(name), "value": rr["value"], "unit": "tokens/s",
                   "ms_per_step": rr["elapsed_ms"] / args.steps,
                   "dtype": "fp8" if wb.fp8 else "bf16", "roofline": rl, "per_T": pt,
                   "cuda_graphs": sorted(wb.graphs) if wb.graphs else (wb.graph_note or "none"),
                   "gpu_launches": wb.launches(), "clocks": wclocks}
            if rank == 0 and world == 1 and not args.no_cpu_baseline and wb.lora is None:
                T, pool = ORACLE_SAMPLE[name]
                blk["cpu_baseline"] = cpu_baseline(wb.W, wb.dtype, T, args.cpu_seconds_other,
                                                   pool, single_thread=False)
            wb.release()
            del wb
            blocks[name] = blk
        if world == 1 and not args.no_split:
            # host cores are shared by the ranks of one node: one GPU only
            blocks["split"] = run_split(args, dev, uuid)
        line["workloads"] = blocks
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_split_calls(args):
    """Profiling mode of the split: N calls of the split layer at one T (the
    dynamic plan with the latency model measured at set-up), for a profiler."""
    import mixture_experts_expert_route_b200 as moe
    T = int(args.Ts.split(",")[0]) if args.Ts else 64
    dev = torch.device("cuda", 0)
    sb = SplitBench(args, dev, Ts=(T,))
    x, lg = sb.dev_in[T][0]
    for _ in range(args.calls):
        sb.layer(x, lg, out=sb.outs[T])
    torch.cuda.synchronize()
    if sb.layer.check() != 0:
        raise RuntimeError("device status word reports a fault")
    print(f"split T={T}: {args.calls} calls, plan {[int(v) for v in sb.layer.where]}", flush=True)


def run_calls(args):
    """Profiling mode: N forward calls of one workload at one T (no timing, no
    JSON), for a profiler to capture; the weights are drawn on the GPU."""
    import mixture_experts_expert_route_b200 as moe
    name = headline_name(args)
    if name == "split":
        run_split_calls(args)
        return
    wl = WORKLOADS[name]
    cfg = CONFIGS[wl["cfg"]]
    T = int(args.Ts.split(",")[0]) if args.Ts else max(cfg["T"])
    dev = torch.device("cuda", 0)
    W = make_weights(wl["cfg"], 0, "cuda", E=args.experts)
    layer = moe.MoELayer(W.Wg, W.Wu, W.Wd, k=cfg["k"], dtype=wl["dtype"])
    E = W.E
    del W
    torch.cuda.empty_cache()
    Wr = make_weights(wl["cfg"], 0, "cpu", E=args.experts, router_only=True)
    x, lg = (t.to(dev) for t in make_batch(Wr, T, 0, 0))
    out = torch.empty((T, cfg["H"]), dtype=torch.bfloat16, device=dev)
    call = lambda: layer(x, lg, out=out)
    if wl.get("lora"):
        # the adapter variant: the same adapters and token assignment as the bench
        from workloads import adapter_ids, make_lora
        n, r = wl["lora"]
        lw = make_lora(E, cfg["H"], cfg["I"], n_adapters=n, rank=r, seed=1)
        lora = moe.Lora(*(m.to(dev) for m in (lw.Ag, lw.Bg, lw.Au, lw.Bu, lw.Ad, lw.Bd)), lw.scale)
        ad = adapter_ids(T, n, seed=T).to(dev)
        call = lambda: moe.forward(wl["dtype"], x, lg, layer.packed, layer.scales, E, cfg["I"],
                                   cfg["k"], out=out, status=layer.status, ws=layer.workspace(T),
                                   lora=lora, adapter=ad)
    for _ in range(args.calls):
        call()
    torch.cuda.synchronize()
    if layer.check() != 0:
        raise RuntimeError("device status word reports a fault")
    print(f"{name} T={T} E={E}: {args.calls} calls", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-split", action="store_true",
                    help="leave the CPU/GPU split block out of --workload all")
    ap.add_argument("--workload", choices=["all", "split"] + sorted(WORKLOADS), default="all",
                    help="all: decode headline plus a block per other workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graphs", action="store_true",
                    help="run T <= 64 as CUDA graph replays (default: direct launches, which "
                         "measured faster on the device)")
    ap.add_argument("--no-graphs", action="store_true",
                    help="direct launches (the default; kept for older command lines)")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="oracle budget of the headline's CPU baseline (each of all-core "
                         "and single-thread)")
    ap.add_argument("--cpu-seconds-other", type=float, default=3.0,
                    help="oracle budget of each other workload's CPU baseline")
    ap.add_argument("--ref-step-seconds", type=float, default=5.0)
    ap.add_argument("--Ts", default="", help="comma-separated subset of the headline's "
                                            "token counts")
    ap.add_argument("--calls", type=int, default=0,
                    help="profiling mode: run this many forward calls of the workload (at the "
                         "first of --Ts, else its largest T) and exit")
    ap.add_argument("--experts", type=int, default=None,
                    help="profiling mode: override the workload's expert count")
    args = ap.parse_args()
    if args.calls > 0:
        run_calls(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
