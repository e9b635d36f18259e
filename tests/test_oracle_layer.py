"""Pins of the oracle's layer output against torch fp64 library routines and
the invariants the layer's definition implies."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import make_layer
from tests.conftest import rel_err
from tests.test_oracle_route import brute_route


def dense_forward(x, Wg, Wu, Wd, ids, w):
    """Every expert on every token (torch fp64 matmuls), then a routing mask."""
    X = x.double()
    G = torch.einsum("th,ehi->eti", X, Wg.double())
    U = torch.einsum("th,ehi->eti", X, Wu.double())
    Y = torch.einsum("eti,eih->eth", F.silu(G) * U, Wd.double())
    T, E = X.shape[0], Wg.shape[0]
    mask = torch.zeros(T, E, dtype=torch.float64)
    for t in range(T):
        for j in range(ids.shape[1]):
            mask[t, int(ids[t, j])] += float(w[t, j])
    return torch.einsum("te,eth->th", mask, Y).numpy()


def brute_routing(logits, k):
    lg = logits.numpy()
    ids, ws = [], []
    for t in range(lg.shape[0]):
        i, w = brute_route(lg[t].tolist(), k)
        ids.append(i)
        ws.append(w)
    return np.array(ids, np.int32), np.array(ws, np.float64)


def test_tiny_fp32_vs_dense():
    L = make_layer("tiny")
    assert L.Wg.dtype == torch.float32
    ids, w = brute_routing(L.logits, L.k)
    ref = dense_forward(L.x, L.Wg, L.Wu, L.Wd, ids, w)
    out = oracle.moe_layer(L.x, ids, w, L.Wg, L.Wu, L.Wd)
    assert rel_err(out, ref) < 1e-12
    # the bf16-rounded weights (what the GPU path computes with)
    g, u, d = L.weights_bf16()
    out = oracle.moe_layer(L.x, ids, w, g, u, d)
    assert rel_err(out, dense_forward(L.x, g, u, d, ids, w)) < 1e-12


def test_token_subset_matches_full():
    L = make_layer("tiny")
    ids, w = oracle.route_topk(L.logits, L.k)
    full = oracle.moe_layer(L.x, ids, w, L.Wg, L.Wu, L.Wd)
    sub = [15, 0, 7, 7]
    part = oracle.moe_layer(L.x, ids, w, L.Wg, L.Wu, L.Wd, tokens=sub)
    assert np.array_equal(part, full[sub])


def test_single_expert_is_dense_swiglu():
    L = make_layer("tiny", E=1, k=1, T=9)
    ids, w = oracle.route_topk(L.logits, 1)
    assert np.all(ids == 0) and np.all(w == 1.0)
    out = oracle.moe_layer(L.x, ids, w, L.Wg, L.Wu, L.Wd)
    X = L.x.double()
    ref = (F.silu(X @ L.Wg[0].double()) * (X @ L.Wu[0].double())) @ L.Wd[0].double()
    assert rel_err(out, ref.numpy()) < 1e-12


def test_all_experts_equal_logits_is_mean():
    L = make_layer("tiny", k=8, T=5, zero_router=True)
    ids, w = oracle.route_topk(L.logits, 8)
    np.testing.assert_allclose(w, 1 / 8, rtol=0, atol=1e-16)
    out = oracle.moe_layer(L.x, ids, w, L.Wg, L.Wu, L.Wd)
    X = L.x.double()
    ys = [(F.silu(X @ L.Wg[e].double()) * (X @ L.Wu[e].double())) @ L.Wd[e].double()
          for e in range(8)]
    ref = torch.stack(ys).mean(0).numpy()
    assert rel_err(out, ref) < 1e-12


def test_token_permutation_equivariance():
    L = make_layer("tiny")
    ids, w = oracle.route_topk(L.logits, L.k)
    out = oracle.moe_layer(L.x, ids, w, L.Wg, L.Wu, L.Wd)
    perm = torch.randperm(L.T, generator=torch.Generator().manual_seed(3))
    ids2, w2 = oracle.route_topk(L.logits[perm], L.k)
    out2 = oracle.moe_layer(L.x[perm], ids2, w2, L.Wg, L.Wu, L.Wd)
    assert np.array_equal(out2, out[perm.numpy()])


def test_linear_in_down_projection():
    L = make_layer("tiny")
    ids, w = oracle.route_topk(L.logits, L.k)
    out = oracle.moe_layer(L.x, ids, w, L.Wg, L.Wu, L.Wd)
    out2 = oracle.moe_layer(L.x, ids, w, L.Wg, L.Wu, L.Wd * 2)
    assert np.array_equal(out2, 2 * out)


def test_identical_experts_share_mass():
    """Two identical experts chosen together give that expert's output whatever
    the split: catches a missing renormalisation of the top-k weights."""
    L = make_layer("tiny", E=4, k=2, T=7)
    Wg = L.Wg.clone(); Wu = L.Wu.clone(); Wd = L.Wd.clone()
    Wg[1] = Wg[0]; Wu[1] = Wu[0]; Wd[1] = Wd[0]
    lg = L.logits.clone()
    lg[:, 0] = 5 + torch.arange(7, dtype=torch.float32) * 0.1
    lg[:, 1] = 4.5
    ids, w = oracle.route_topk(lg, 2)
    assert np.all(np.sort(ids, axis=1) == [0, 1])
    out = oracle.moe_layer(L.x, ids, w, Wg, Wu, Wd)
    X = L.x.double()
    ref = ((F.silu(X @ Wg[0].double()) * (X @ Wu[0].double())) @ Wd[0].double()).numpy()
    assert rel_err(out, ref) < 1e-12


@pytest.mark.parametrize("E,k,T", [(8, 2, 16), (6, 3, 11), (16, 8, 4)])
def test_random_routing_vs_dense(E, k, T):
    L = make_layer("tiny", E=E, k=k, T=T, H=128, I=192, seed=E + k)
    ids, w = oracle.route_topk(L.logits, k)
    g, u, d = L.weights_bf16()
    out = oracle.moe_layer(L.x, ids, w, g, u, d)
    assert rel_err(out, dense_forward(L.x, g, u, d, ids, w)) < 1e-12
