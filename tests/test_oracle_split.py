"""Pins of the split oracle's decisions (oracle/split.py) against definitions
other than its own code: brute force over every placement, the closed-form
token threshold of the latency comparison, and hand-derived cases."""
import itertools
import random

import pytest

from oracle import split as osplit


def brute_place(hits, budget):
    """Among all budget-sized expert sets, the one with the most hits; among
    equals, the lexicographically smallest set of indices."""
    best = None
    for combo in itertools.combinations(range(len(hits)), budget):
        key = (-sum(hits[e] for e in combo), combo)
        if best is None or key < best:
            best = key
    chosen = set(best[1])
    return [1 if e in chosen else 0 for e in range(len(hits))]


@pytest.mark.parametrize("seed", range(40))
def test_place_is_the_best_set(seed):
    rng = random.Random(seed)
    E = rng.randint(1, 9)
    hits = [rng.randint(0, 4) for _ in range(E)]     # small range: many ties
    for budget in range(E + 1):
        assert osplit.place(hits, budget) == brute_place(hits, budget)


def test_place_hand_cases():
    assert osplit.place([5, 9, 1, 9], 2) == [0, 1, 0, 1]
    assert osplit.place([3, 3, 3], 2) == [1, 1, 0]
    assert osplit.place([0, 0], 0) == [0, 0]
    assert osplit.place([7], 1) == [1]
    with pytest.raises(ValueError):
        osplit.place([1, 2], 3)


COSTS = dict(cpu_us=100.0, cpu_us_per_token=50.0, xfer_us=600.0, gpu_us=20.0,
             gpu_us_per_token=2.0)


def test_plan_threshold_closed_form():
    # staged iff xfer + gpu0 + g1 n < cpu0 + c1 n  <=>  n > (xfer + gpu0 - cpu0) / (c1 - g1)
    n_star = (600.0 + 20.0 - 100.0) / (50.0 - 2.0)          # 10.83...
    for n in range(1, 30):
        where = osplit.plan([n], [0], COSTS, n_stage=1)
        assert where == [osplit.STAGED if n > n_star else osplit.CPU], n


def test_plan_tie_stays_on_cpu():
    costs = dict(cpu_us=0.0, cpu_us_per_token=10.0, xfer_us=100.0, gpu_us=0.0,
                 gpu_us_per_token=0.0)
    assert osplit.plan([10], [0], costs, 1) == [osplit.CPU]      # 100 == 100
    assert osplit.plan([11], [0], costs, 1) == [osplit.STAGED]


def test_plan_hand_case():
    counts = [0, 3, 40, 12, 40, 25, 0, 11]
    resident = [1, 1, 0, 0, 0, 0, 0, 1]
    # savings (c1 - g1) n - 520: expert 2 and 4 -> 1400, 5 -> 680, 3 -> 56; 11 -> -- (resident)
    assert osplit.plan(counts, resident, COSTS, n_stage=2) == [
        osplit.IDLE, osplit.RESIDENT, osplit.STAGED, osplit.CPU, osplit.STAGED, osplit.CPU,
        osplit.IDLE, osplit.RESIDENT]
    assert osplit.plan(counts, resident, COSTS, n_stage=3)[5] == osplit.STAGED
    assert osplit.plan(counts, resident, COSTS, n_stage=8)[3] == osplit.STAGED
    assert osplit.plan(counts, resident, COSTS, n_stage=0) == [
        osplit.IDLE, osplit.RESIDENT, osplit.CPU, osplit.CPU, osplit.CPU, osplit.CPU,
        osplit.IDLE, osplit.RESIDENT]


@pytest.mark.parametrize("seed", range(30))
def test_plan_staged_set_by_brute_force(seed):
    """With per-token costs c1 > g1 the saving grows with n, so the staged set
    is the n_stage non-resident experts above the threshold with the most
    tokens (equal counts: lower index): checked against that selection done
    by enumerating every subset."""
    rng = random.Random(1000 + seed)
    E = rng.randint(1, 8)
    counts = [rng.choice([0, 1, 5, 11, 12, 20, 20, 30]) for _ in range(E)]
    resident = [rng.random() < 0.3 for _ in range(E)]
    n_stage = rng.randint(0, E)
    where = osplit.plan(counts, resident, COSTS, n_stage)
    n_star = (600.0 + 20.0 - 100.0) / 48.0
    cand = [e for e in range(E) if counts[e] > n_star and not resident[e]]
    m = min(n_stage, len(cand))
    best = None
    for combo in itertools.combinations(cand, m):
        key = (-sum(counts[e] for e in combo), combo)
        if best is None or key < best:
            best = key
    staged = set(best[1]) if best else set()
    for e in range(E):
        if counts[e] == 0:
            assert where[e] == osplit.IDLE
        elif resident[e]:
            assert where[e] == osplit.RESIDENT
        else:
            assert where[e] == (osplit.STAGED if e in staged else osplit.CPU), (e, where)


def makespan(where, counts, costs):
    host = sum(osplit.cpu_latency(costs, counts[e]) for e in range(len(counts))
               if where[e] == osplit.CPU)
    link = sum(osplit.gpu_latency(costs, counts[e]) for e in range(len(counts))
               if where[e] == osplit.STAGED)
    return max(host, link)


def test_balanced_hand_case():
    # four experts of 128 tokens: host 5.0 ms each, copy 6.4 ms each;
    # staging two gives max(10.0, 12.8) = 12.8 ms, the best prefix
    costs = dict(cpu_us=1700.0, cpu_us_per_token=25.78125, xfer_us=6400.0, gpu_us=0.0,
                 gpu_us_per_token=0.0)
    counts = [128, 0, 128, 128, 128]
    resident = [0, 1, 0, 0, 0]
    where = osplit.plan_balanced(counts, resident, costs, n_stage=4)
    assert where == [osplit.STAGED, osplit.IDLE, osplit.STAGED, osplit.CPU, osplit.CPU]
    assert makespan(where, counts, costs) == 12800.0
    # the per-expert rule keeps all four on the host (5.0 < 6.4): 20 ms
    assert osplit.plan(counts, resident, costs, 4) == [osplit.CPU, osplit.IDLE, osplit.CPU,
                                                       osplit.CPU, osplit.CPU]
    # with one slot: max(15.0, 6.4)
    assert osplit.plan_balanced(counts, resident, costs, 1).count(osplit.STAGED) == 1


@pytest.mark.parametrize("seed", range(40))
def test_balanced_with_equal_experts_is_optimal(seed):
    """When every candidate has the same token count the ranking is only the
    index order and the best prefix is the best subset: checked against all
    subsets; and in general the plan is never worse than staging nothing."""
    rng = random.Random(2000 + seed)
    E = rng.randint(1, 9)
    n = rng.choice([1, 16, 128, 512])
    counts = [n if rng.random() < 0.8 else 0 for _ in range(E)]
    resident = [rng.random() < 0.25 for _ in range(E)]
    costs = dict(cpu_us=rng.uniform(0, 3000), cpu_us_per_token=rng.uniform(0, 60),
                 xfer_us=rng.uniform(100, 8000), gpu_us=0.0, gpu_us_per_token=0.0)
    n_stage = rng.randint(0, E)
    where = osplit.plan_balanced(counts, resident, costs, n_stage)
    cand = [e for e in range(E) if counts[e] and not resident[e]]
    best = min(makespan([osplit.STAGED if e in set(sub) else
                         (osplit.CPU if e in cand else osplit.IDLE) for e in range(E)],
                        counts, costs)
               for m in range(min(n_stage, len(cand)) + 1)
               for sub in itertools.combinations(cand, m))
    assert makespan(where, counts, costs) == pytest.approx(best, rel=1e-12)
    for e in range(E):
        if counts[e] == 0:
            assert where[e] == osplit.IDLE
        elif resident[e]:
            assert where[e] == osplit.RESIDENT


@pytest.mark.parametrize("seed", range(40))
def test_balanced_never_worse_than_fixed_plans(seed):
    rng = random.Random(3000 + seed)
    E = rng.randint(1, 12)
    counts = [rng.choice([0, 1, 3, 16, 64, 128, 300, 700]) for _ in range(E)]
    resident = [rng.random() < 0.3 for _ in range(E)]
    costs = dict(cpu_us=rng.uniform(0, 3000), cpu_us_per_token=rng.uniform(0, 60),
                 xfer_us=rng.uniform(100, 8000), gpu_us=rng.uniform(0, 100),
                 gpu_us_per_token=rng.uniform(0, 1))
    n_stage = rng.randint(0, E)
    where = osplit.plan_balanced(counts, resident, costs, n_stage)
    assert where.count(osplit.STAGED) <= n_stage
    cand = [e for e in range(E) if counts[e] and not resident[e]]
    all_cpu = [osplit.CPU if e in cand else where[e] for e in range(E)]
    assert makespan(where, counts, costs) <= makespan(all_cpu, counts, costs)
