"""The CPU/GPU split layer (moe_split_forward) on the GPU against the oracle:
the plan it took equals the split oracle's for the batch's routing, and the
layer output equals the layer oracle's, whichever experts ran on the host,
from staging slots or from GPU memory."""
import numpy as np
import pytest
import torch

import oracle
from oracle import split as osplit
from tests.gpu_helpers import assert_close, lib

pytestmark = pytest.mark.gpu

BIG = 1e30


def make(T, E, k, H, I, seed, skew=0.0):
    g = torch.Generator().manual_seed(seed)
    Wg = (torch.randn(E, H, I, generator=g) / H ** 0.5).to(torch.bfloat16)
    Wu = (torch.randn(E, H, I, generator=g) / H ** 0.5).to(torch.bfloat16)
    Wd = (torch.randn(E, I, H, generator=g) / I ** 0.5).to(torch.bfloat16)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=g) + skew * torch.linspace(2, -2, E)
    return Wg, Wu, Wd, x, logits


def expected_plan(ids, E, resident, policy, costs, n_stage, moe):
    counts = np.bincount(ids.ravel(), minlength=E)
    if policy == moe.POLICY_ALL_CPU:
        c = dict(cpu_us=0.0, cpu_us_per_token=0.0, xfer_us=BIG, gpu_us=0.0, gpu_us_per_token=0.0)
    elif policy == moe.POLICY_ALL_STAGED:
        c = dict(cpu_us=BIG, cpu_us_per_token=0.0, xfer_us=0.0, gpu_us=0.0, gpu_us_per_token=0.0)
    elif policy == moe.POLICY_BALANCED:
        return osplit.plan_balanced(counts, resident, costs, n_stage)
    else:
        c = costs
    return osplit.plan(counts, resident, c, n_stage)


def run_case(T, E, k, H, I, resident, n_stage, policy, costs, seed, skew=0.0, calls=1):
    moe = lib()
    Wg, Wu, Wd, x, logits = make(T, E, k, H, I, seed, skew)
    layer = moe.SplitLayer(Wg, Wu, Wd, k, resident, n_stage=n_stage, policy=policy,
                           costs=moe.split_costs(**costs))
    for call in range(calls):
        if call:
            g = torch.Generator().manual_seed(seed + 100 * call)
            x = torch.randn(T, H, generator=g).to(torch.bfloat16)
            logits = torch.randn(T, E, generator=g) + skew * torch.linspace(2, -2, E)
        out = layer(x.cuda(), logits.cuda())
        torch.cuda.synchronize()
        assert layer.check() == 0
        ids, w = oracle.route_topk(logits, k)
        want = expected_plan(ids, E, resident, policy, costs, n_stage, moe)
        assert list(layer.where) == want
        ref = oracle.moe_layer(x, ids, w, Wg, Wu, Wd)
        assert_close(out, ref, 0, f"split T={T} call {call}")
    return layer


COSTS = dict(cpu_us=10.0, cpu_us_per_token=20.0, xfer_us=100.0, gpu_us=0.0,
             gpu_us_per_token=0.0)   # staged above 4.5 tokens


@pytest.mark.parametrize("policy", [1, 2])
def test_single_token(policy):
    run_case(1, 8, 2, 256, 512, [1, 0, 1, 0, 0, 0, 0, 0], 2, policy, COSTS, seed=1)


@pytest.mark.parametrize("T", [37, 200])
def test_dynamic_mix(T):
    # more experts would gain from a copy than there are slots: some go to the host
    run_case(T, 8, 2, 256, 512, [0, 1, 0, 0, 1, 0, 0, 1], 2, 0, COSTS, seed=T, skew=1.0)


@pytest.mark.parametrize("T", [40, 300])
def test_balanced_mix(T):
    # host and link both busy: the balanced plan stages a prefix of the ranked experts
    costs = dict(cpu_us=50.0, cpu_us_per_token=1.0, xfer_us=150.0, gpu_us=0.0,
                 gpu_us_per_token=0.0)
    layer = run_case(T, 8, 2, 256, 512, [0, 1, 0, 0, 0, 0, 0, 1], 3, 3, costs, seed=T + 1)
    assert 0 < list(layer.where).count(3) and 0 < list(layer.where).count(2)


def test_everything_on_host():
    run_case(64, 8, 2, 128, 256, [0] * 8, 0, 0, COSTS, seed=3)


def test_everything_resident():
    run_case(64, 8, 2, 128, 256, [1] * 8, 2, 0, COSTS, seed=4)


def test_everything_staged():
    run_case(48, 8, 2, 192, 320, [0] * 8, 8, 2, COSTS, seed=5)


def test_large_tiles_start_past_the_host_rows():
    # ~300 rows per resident expert: CTA-pair tiles, whose rows a gather kernel
    # lays out from the first row of their own segment
    run_case(600, 4, 2, 256, 256, [1, 0, 1, 0], 1, 0, COSTS, seed=6)


def test_many_experts_and_repeated_calls():
    resident = [1 if e % 3 == 0 else 0 for e in range(16)]
    run_case(300, 16, 4, 256, 384, resident, 3, 0, COSTS, seed=7, skew=0.5, calls=3)


def test_block_m_and_one_host_thread():
    moe = lib()
    Wg, Wu, Wd, x, logits = make(90, 8, 2, 128, 256, seed=10)
    layer = moe.SplitLayer(Wg, Wu, Wd, 2, [1, 0, 0, 1, 0, 0, 0, 0], n_stage=2, policy=0,
                           costs=moe.split_costs(**COSTS), block_m=64, host_threads=1)
    out = layer(x.cuda(), logits.cuda())
    torch.cuda.synchronize()
    assert layer.check() == 0
    ids, w = oracle.route_topk(logits, 2)
    assert list(layer.where) == expected_plan(ids, 8, [1, 0, 0, 1, 0, 0, 0, 0], 0, COSTS, 2, moe)
    assert_close(out, oracle.moe_layer(x, ids, w, Wg, Wu, Wd), 0, "split block_m=64")


def test_many_experts_top8():
    # E = 256, k = 8: 1 + 40 + 16 slots, several host experts per batch
    resident = [1 if e % 7 == 0 else 0 for e in range(256)]
    run_case(128, 256, 8, 128, 128, resident, 16, 0, COSTS, seed=11, skew=0.5)


def test_zero_tokens():
    moe = lib()
    Wg, Wu, Wd, x, logits = make(4, 4, 2, 64, 64, seed=12)
    layer = moe.SplitLayer(Wg, Wu, Wd, 2, [1, 0, 0, 0], n_stage=1,
                           costs=moe.split_costs(**COSTS))
    out = layer(x[:0].cuda(), logits[:0].cuda())
    torch.cuda.synchronize()
    assert out.shape == (0, 64) and layer.check() == 0


def test_calibrate():
    moe = lib()
    Wg, Wu, Wd, _, _ = make(1, 4, 2, 256, 512, seed=8)
    layer = moe.SplitLayer(Wg, Wu, Wd, 2, [1, 0, 0, 0], n_stage=1)
    c = layer.costs
    assert c.xfer_us > 0 and c.cpu_us >= 0 and c.cpu_us_per_token >= 0
    assert c.gpu_us == 0 and c.gpu_us_per_token == 0


@pytest.mark.slow
def test_full_size_mixtral_shape():
    """H=4096, I=14336, E=8, k=2, four experts resident, two staging slots,
    the latency model measured on this system; the oracle on a token sample."""
    moe = lib()
    T, E, k, H, I = 16, 8, 2, 4096, 14336
    Wg, Wu, Wd, x, logits = make(T, E, k, H, I, seed=9)
    resident = [1, 1, 1, 1, 0, 0, 0, 0]
    layer = moe.SplitLayer(Wg, Wu, Wd, k, resident, n_stage=2)
    out = layer(x.cuda(), logits.cuda())
    torch.cuda.synchronize()
    assert layer.check() == 0
    ids, w = oracle.route_topk(logits, k)
    counts = np.bincount(ids.ravel(), minlength=E)
    c = layer.costs
    costs = dict(cpu_us=c.cpu_us, cpu_us_per_token=c.cpu_us_per_token, xfer_us=c.xfer_us,
                 gpu_us=c.gpu_us, gpu_us_per_token=c.gpu_us_per_token)
    assert list(layer.where) == osplit.plan(counts, resident, costs, 2)
    sample = [0, 3, 7, 10, 15]
    ref = oracle.moe_layer(x, ids, w, Wg, Wu, Wd, tokens=sample)
    assert_close(out[sample], ref, 0, "split full size")
