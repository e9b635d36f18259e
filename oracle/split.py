"""Oracle of the CPU/GPU expert split's decisions -- TEST INFRASTRUCTURE.

Only the tests and the benchmark's CPU legs may import this module.  Plain
Python, written from FIDDLER as summarised on aibr.jp/archives/173321
("FIDDLER: CPU-GPU orchestration for fast inference of Mixture-of-Experts
models"), § "3.中核となる技術的要素":

- placement: the experts hit most often in offline profiling go to GPU
  memory first, up to the budget;
- plan: for each expert a batch uses that is not in GPU memory, compare the
  expected latency of running it on the CPU with that of bringing its
  weights to the GPU and running it there, from the batch's token count,
  and take the faster.

Readings where the page is silent (shared with the library's definition):
equal hit counts place the lower index first; a tie between the two
latencies keeps the expert on the CPU (no copy); when more experts would
gain from a copy than there are staging slots, the slots go to the largest
savings, equal savings to the lower index.

The layer output of the split is the layer of ``oracle.moe_layer``: the
split only decides where each expert runs.
"""
from __future__ import annotations

IDLE, RESIDENT, STAGED, CPU = 0, 1, 2, 3


def place(hits, budget: int) -> list[int]:
    """resident[e] = 1 for the `budget` experts with the most hits."""
    E = len(hits)
    if not 0 <= budget <= E:
        raise ValueError("budget outside [0, E]")
    ranked = sorted(range(E), key=lambda e: (-int(hits[e]), e))
    chosen = set(ranked[:budget])
    return [1 if e in chosen else 0 for e in range(E)]


def cpu_latency(costs: dict, n: int) -> float:
    return costs["cpu_us"] + costs["cpu_us_per_token"] * n


def gpu_latency(costs: dict, n: int) -> float:
    return costs["xfer_us"] + costs["gpu_us"] + costs["gpu_us_per_token"] * n


def plan(counts, resident, costs: dict, n_stage: int) -> list[int]:
    """where[e] in {IDLE, RESIDENT, STAGED, CPU} for one batch."""
    where = []
    savings = []
    for e, n in enumerate(counts):
        n = int(n)
        if n == 0:
            where.append(IDLE)
        elif resident[e]:
            where.append(RESIDENT)
        else:
            where.append(CPU)
            c, g = cpu_latency(costs, n), gpu_latency(costs, n)
            if g < c:
                savings.append((c - g, e))
    savings.sort(key=lambda item: (-item[0], item[1]))
    for _, e in savings[:n_stage]:
        where[e] = STAGED
    return where


def plan_balanced(counts, resident, costs: dict, n_stage: int) -> list[int]:
    """The balanced plan (an extension beyond the page, same latency model):
    the host and the host-to-GPU link work in parallel, so a batch's
    non-resident experts cost max(host time, link time), with host time the
    sum of cpu(n) of the experts left on the host and link time the sum of
    gpu(n) of the staged ones.  Candidates (active, not resident) are ranked
    by cpu(n) / gpu(n), largest first (gpu(n) <= 0 ranks first; equal ratios:
    lower index first); the plan stages the first j of them, j in
    0..min(n_stage, #candidates) minimising that maximum (equal maxima: the
    smaller j).  Sums run in rank order."""
    where = []
    cand = []
    for e, n in enumerate(counts):
        n = int(n)
        if n == 0:
            where.append(IDLE)
        elif resident[e]:
            where.append(RESIDENT)
        else:
            where.append(CPU)
            c, g = cpu_latency(costs, n), gpu_latency(costs, n)
            ratio = float("inf") if g <= 0 else c / g
            cand.append((ratio, e, c, g))
    cand.sort(key=lambda item: (-item[0], item[1]))
    best_j, best = 0, None
    for j in range(min(n_stage, len(cand)) + 1):
        host = 0.0
        for i in range(j, len(cand)):
            host += cand[i][2]
        link = 0.0
        for i in range(j):
            link += cand[i][3]
        cost = max(host, link)
        if best is None or cost < best:
            best_j, best = j, cost
    for i in range(best_j):
        where[cand[i][1]] = STAGED
    return where
