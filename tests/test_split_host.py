"""The host side of the CPU/GPU expert split, through the C ABI, on the CPU:
placement and plan against the split oracle (exact), the host expert kernel
against the layer oracle (both instruction-set paths), its weight layout,
and argument errors."""
import random

import numpy as np
import pytest
import torch

import oracle
from oracle import split as osplit
from tests.conftest import rel_err


@pytest.fixture(scope="module")
def L():
    from mixture_experts_expert_route_b200 import _lib, build
    build.build(debug=_lib.DEBUG_CHECKS)
    import mixture_experts_expert_route_b200 as moe
    return moe


@pytest.mark.parametrize("seed", range(25))
def test_place_matches_oracle(L, seed):
    rng = random.Random(seed)
    E = rng.randint(1, 256)
    hits = [rng.randint(0, 6) * rng.choice([1, 1000, 10**9]) for _ in range(E)]
    budget = rng.randint(0, E)
    assert list(L.split_place(hits, budget)) == osplit.place(hits, budget)


@pytest.mark.parametrize("seed", range(25))
def test_plan_matches_oracle(L, seed):
    rng = random.Random(100 + seed)
    E = rng.randint(1, 256)
    counts = [rng.choice([0, 0, 1, 2, 3, 7, 16, 64, 500]) for _ in range(E)]
    resident = [int(rng.random() < 0.4) for _ in range(E)]
    costs = dict(cpu_us=rng.uniform(0, 200), cpu_us_per_token=rng.uniform(0, 100),
                 xfer_us=rng.uniform(0, 5000), gpu_us=rng.uniform(0, 50),
                 gpu_us_per_token=rng.uniform(0, 5))
    n_stage = rng.randint(0, 8)
    got = L.split_plan(counts, resident, L.split_costs(**costs), n_stage)
    assert list(got) == osplit.plan(counts, resident, costs, n_stage)


@pytest.mark.parametrize("seed", range(25))
def test_balanced_plan_matches_oracle(L, seed):
    rng = random.Random(500 + seed)
    E = rng.randint(1, 256)
    counts = [rng.choice([0, 0, 1, 2, 16, 64, 128, 128, 500]) for _ in range(E)]
    resident = [int(rng.random() < 0.4) for _ in range(E)]
    costs = dict(cpu_us=rng.uniform(0, 3000), cpu_us_per_token=rng.uniform(0, 60),
                 xfer_us=rng.uniform(0, 8000), gpu_us=rng.uniform(0, 50),
                 gpu_us_per_token=rng.uniform(0, 1))
    if seed % 5 == 0:
        costs.update(xfer_us=0.0, gpu_us=0.0, gpu_us_per_token=0.0)   # gpu(n) = 0: ranks first
    n_stage = rng.randint(0, 16)
    got = L.split_plan(counts, resident, L.split_costs(**costs), n_stage, balanced=True)
    assert list(got) == osplit.plan_balanced(counts, resident, costs, n_stage)


def test_plan_and_place_errors(L):
    lib = L.lib()
    c = L.split_costs()
    assert lib.moe_split_place(None, 4, 1, None) == 1
    with pytest.raises(L.MoEError):
        L.split_place([1, 2, 3], 4)
    with pytest.raises(L.MoEError):
        L.split_place([1, -2, 3], 1)
    with pytest.raises(L.MoEError):
        L.split_plan([1, -1], [0, 0], c, 1)
    with pytest.raises(L.MoEError):
        L.split_plan([1, 1], [0, 0], c, -1)


def master(E, H, I, seed):
    g = torch.Generator().manual_seed(seed)
    Wg = (torch.randn(E, H, I, generator=g) / H ** 0.5).to(torch.bfloat16)
    Wu = (torch.randn(E, H, I, generator=g) / H ** 0.5).to(torch.bfloat16)
    Wd = (torch.randn(E, I, H, generator=g) / I ** 0.5).to(torch.bfloat16)
    return Wg, Wu, Wd


def test_host_layout(L):
    """Section of a [K][N] matrix = [N/16][K/2][16][2]: element (r, c) of W at
    ((c//16 * K/2 + r//2) * 16 + c%16) * 2 + r%2, sections G, U, D in order."""
    E, H, I = 2, 64, 128
    vals = torch.arange(E * H * I, dtype=torch.int32)
    Wg = (vals % 32749).to(torch.int16).view(torch.bfloat16).reshape(E, H, I).clone()
    Wu = ((vals + 7) % 32749).to(torch.int16).view(torch.bfloat16).reshape(E, H, I).clone()
    Wd = ((vals + 13) % 32749).to(torch.int16).view(torch.bfloat16).reshape(E, I, H).clone()
    packed = L.host_pack_weights(Wg, Wu, Wd)
    assert packed.shape == (E, 3 * H * I * 2)
    p16 = packed.view(torch.int16).reshape(E, 3, H * I)
    rng = np.random.default_rng(0)
    for _ in range(300):
        e = int(rng.integers(E))
        which = int(rng.integers(3))
        W, K, N = [(Wg, H, I), (Wu, H, I), (Wd, I, H)][which]
        r, c = int(rng.integers(K)), int(rng.integers(N))
        pos = ((c // 16 * (K // 2) + r // 2) * 16 + c % 16) * 2 + r % 2
        assert int(p16[e, which, pos]) == int(W[e, r, c].view(torch.int16))


@pytest.mark.parametrize("H,I,n", [(64, 64, 1), (128, 256, 3), (256, 192, 8), (192, 320, 13),
                                   (512, 128, 33)])
@pytest.mark.parametrize("path", ["auto", "avx512_bf16", "portable"])
def test_host_expert_matches_oracle(L, H, I, n, path):
    need = {"auto": 0, "avx512_bf16": L.HOST_ISA_AVX512_BF16, "portable": 0}[path]
    if L.host_isa() < need:
        pytest.skip("this CPU has no AVX512_BF16")
    Wg, Wu, Wd = master(1, H, I, seed=H + I + n)
    g = torch.Generator().manual_seed(n)
    x = torch.randn(n, H, generator=g).to(torch.bfloat16)
    w = torch.rand(n, generator=g) + 0.25
    packed = L.host_pack_weights(Wg, Wu, Wd)
    h, y = L.host_expert_ffn(packed[0], x, w, path=path)
    ids = np.zeros((n, 1), np.int32)
    ref = oracle.moe_layer(x, ids, w.double().numpy()[:, None], Wg, Wu, Wd)
    err = rel_err(y.double().numpy(), ref)
    assert err <= 2e-2, err
    # h against its definition in fp64 (bf16 rounding of h on the host)
    xd = x.double()
    gd = xd @ Wg[0].double()
    ud = xd @ Wu[0].double()
    hd = gd / (1 + torch.exp(-gd)) * ud
    assert rel_err(h.double().numpy(), hd.numpy()) <= 1e-2


@pytest.mark.parametrize("n", [9, 16, 40])
def test_host_paths_agree(L, n):
    """Every instruction-set path this CPU has against the portable one: fp32
    sums in a different order, so a few bf16 ulps at most."""
    H, I = 256, 512
    Wg, Wu, Wd = master(1, H, I, seed=5)
    x = torch.randn(n, H, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    w = torch.ones(n)
    packed = L.host_pack_weights(Wg, Wu, Wd)
    _, y1 = L.host_expert_ffn(packed[0], x, w, path="portable")
    paths = ["auto"] + (["avx512_bf16"] if L.host_isa() >= L.HOST_ISA_AVX512_BF16 else [])
    for p in paths:
        _, y0 = L.host_expert_ffn(packed[0], x, w, path=p)
        assert rel_err(y0.double().numpy(), y1.double().numpy()) <= 4e-3, p


def test_host_threads_do_not_change_result(L):
    H, I, n = 128, 256, 5
    Wg, Wu, Wd = master(1, H, I, seed=9)
    x = torch.randn(n, H, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    w = torch.rand(n) + 0.5
    packed = L.host_pack_weights(Wg, Wu, Wd)
    ys = [L.host_expert_ffn(packed[0], x, w, threads=t)[1] for t in (1, 2, 0)]
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])


def test_host_expert_zero_rows_and_errors(L):
    H, I = 64, 64
    Wg, Wu, Wd = master(1, H, I, seed=1)
    packed = L.host_pack_weights(Wg, Wu, Wd)
    h, y = L.host_expert_ffn(packed[0], torch.zeros(0, H, dtype=torch.bfloat16), torch.zeros(0))
    assert y.shape == (0, H)
    lib = L.lib()
    a = L._lib.HostFfnArgs(H, 100, 1, None, None, None, None, None, 0, 0)   # I % 64 != 0
    import ctypes
    assert lib.moe_host_expert_ffn(ctypes.byref(a)) == 1
    assert lib.moe_host_packed_size(64, 100) == 0
    assert lib.moe_host_packed_size(4096, 14336) == 3 * 4096 * 14336 * 2
    assert lib.moe_split_workspace_size(64, 2, 8, 4, 2, 4096, 14336, 0) > 0
    assert lib.moe_split_workspace_size(64, 2, 8, 4, 252, 4096, 14336, 0) == 0   # > 256 slots
    assert lib.moe_split_host_workspace_size(64, 2, 4096, 14336) > 64 * 2 * 4096 * 2


def test_split_forward_argument_errors(L):
    import ctypes
    lib = L.lib()
    res = np.array([1, 0, 0, 1], np.int32)
    a = L._lib.SplitArgs(4, 2, 4, 64, 64, 0, None, None, None, res.ctypes.data, None, None, 0,
                         None, None, None, L.POLICY_DYNAMIC, None, None, None, None, 0)
    assert lib.moe_split_forward(ctypes.byref(a), None, 0, None, 0, None) == 1   # no costs
    a.policy = 7
    assert lib.moe_split_forward(ctypes.byref(a), None, 0, None, 0, None) == 1
    a.policy = L.POLICY_ALL_CPU
    a.k = 5                                                                     # k > E
    assert lib.moe_split_forward(ctypes.byref(a), None, 0, None, 0, None) == 1
    a.k = 2
    a.T = 0
    assert lib.moe_split_forward(ctypes.byref(a), None, 0, None, 0, None) == 0  # no-op
    a.T = 4
    a.n_stage = 254                                                             # 1 + 2 + 254
    assert lib.moe_split_forward(ctypes.byref(a), None, 0, None, 0, None) == 2


def test_host_kernel_in_a_forked_child(L):
    """A child made by fork() after the parent used the host kernel gets its
    own thread pool (the parent's threads do not exist in it)."""
    import os
    import signal
    import time
    import warnings
    H, I = 64, 128
    Wg, Wu, Wd = master(1, H, I, seed=2)
    packed = L.host_pack_weights(Wg, Wu, Wd)
    x = torch.randn(5, H, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    w = torch.ones(5)
    _, y0 = L.host_expert_ffn(packed[0], x, w)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore", DeprecationWarning)
        pid = os.fork()
    if pid == 0:
        try:
            _, y1 = L.host_expert_ffn(packed[0], x, w)
            os._exit(0 if torch.equal(y0, y1) else 3)
        except BaseException:
            os._exit(4)
    deadline = time.time() + 60
    while True:
        done, status = os.waitpid(pid, os.WNOHANG)
        if done:
            break
        if time.time() > deadline:
            os.kill(pid, signal.SIGKILL)
            os.waitpid(pid, 0)
            pytest.fail("the forked child did not finish")
        time.sleep(0.05)
    assert os.WIFEXITED(status) and os.WEXITSTATUS(status) == 0


def test_calibrate_and_sizes_argument_errors(L):
    import ctypes
    lib = L.lib()
    costs = L._lib.SplitCosts()
    fake = ctypes.c_void_p(0x1000)
    # bad sizes, missing buffers, a host workspace too small: nothing runs
    assert lib.moe_split_calibrate(64, 100, 4, fake, fake, fake, fake, 1 << 20, 0, None,
                                   ctypes.byref(costs)) == 1
    assert lib.moe_split_calibrate(64, 64, 0, fake, fake, fake, fake, 1 << 20, 0, None,
                                   ctypes.byref(costs)) == 1
    assert lib.moe_split_calibrate(64, 64, 4, None, fake, fake, fake, 1 << 20, 0, None,
                                   ctypes.byref(costs)) == 1
    need = lib.moe_split_host_workspace_size(4, 1, 64, 64)
    assert need > 0
    assert lib.moe_split_calibrate(64, 64, 4, fake, fake, fake, fake, need - 1, 0, None,
                                   ctypes.byref(costs)) == 3
    # workspace sizes: resident count above E, staging slots past 256 slots, bad dims
    assert lib.moe_split_workspace_size(8, 2, 8, 9, 1, 128, 128, 0) == 0
    assert lib.moe_split_workspace_size(8, 2, 8, 8, 247, 128, 128, 0) > 0      # 1 + 8 + 247
    assert lib.moe_split_workspace_size(8, 2, 8, 8, 248, 128, 128, 0) == 0
    assert lib.moe_split_workspace_size(8, 2, 8, 4, 2, 100, 128, 0) == 0
    assert lib.moe_split_host_workspace_size(8, 0, 128, 128) == 0
    # plans and placement past 256 experts
    big = np.zeros(257, np.int32)
    assert lib.moe_split_plan(big.ctypes.data, big.ctypes.data, 257, ctypes.byref(costs), 1,
                              big.ctypes.data) == 1
    assert lib.moe_split_plan_balanced(big.ctypes.data, big.ctypes.data, 257,
                                       ctypes.byref(costs), 1, big.ctypes.data) == 1
    hits = np.zeros(257, np.int64)
    assert lib.moe_split_place(hits.ctypes.data, 257, 1, big.ctypes.data) == 1
