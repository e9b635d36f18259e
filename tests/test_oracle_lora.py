"""Pins of the multi-LoRA oracle (oracle_moe_layer_lora) against things it
must equal by the definition of a low-rank adapter:
  * tokens without an adapter (-1), or adapters with scale 0, give exactly the
    base layer's output (the base oracle, itself pinned);
  * a token of adapter a sees the merged weights W + s_a A B: the base oracle
    on merged weights (formed with torch fp64 matmuls) agrees;
  * a dense every-expert forward in torch fp64 with the adapters applied per
    token agrees to rounding, and exactly the tokens with an adapter change;
  * a subset of tokens gives those tokens' rows of the full output."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from tests.conftest import rel_err
from workloads import adapter_ids, make_layer, make_lora


def layer_case(T=12, E=4, k=2, H=128, I=64, n_a=3, r=8, seed=1):
    L = make_layer("tiny", T=T, E=E, k=k, H=H, I=I, seed=seed)
    lora = make_lora(E, H, I, n_adapters=n_a, rank=r, seed=seed)
    g, u, d = L.weights_bf16()
    ids, w = oracle.route_topk(L.logits, k)
    return L, lora, (g, u, d), ids, w


def test_no_adapter_is_base_layer():
    L, lora, (g, u, d), ids, w = layer_case()
    ad = torch.full((L.T,), -1, dtype=torch.int32)
    out = oracle.moe_layer_lora(L.x, ids, w, g, u, d, ad, lora.as_dict(), lora.scale)
    base = oracle.moe_layer(L.x, ids, w, g, u, d)
    assert np.array_equal(out, base)


def test_zero_scale_is_base_layer():
    L, lora, (g, u, d), ids, w = layer_case()
    ad = adapter_ids(L.T, 3, seed=2, base_share=0.0)
    out = oracle.moe_layer_lora(L.x, ids, w, g, u, d, ad, lora.as_dict(), torch.zeros(3))
    base = oracle.moe_layer(L.x, ids, w, g, u, d)
    assert np.array_equal(out, base)


@pytest.mark.parametrize("a", [0, 2])
def test_one_adapter_equals_merged_weights(a):
    L, lora, (g, u, d), ids, w = layer_case()
    ad = torch.full((L.T,), a, dtype=torch.int32)
    out = oracle.moe_layer_lora(L.x, ids, w, g, u, d, ad, lora.as_dict(), lora.scale)
    s = float(lora.scale[a])
    mg = g.double() + s * torch.matmul(lora.Ag[a].double(), lora.Bg[a].double())
    mu = u.double() + s * torch.matmul(lora.Au[a].double(), lora.Bu[a].double())
    md = d.double() + s * torch.matmul(lora.Ad[a].double(), lora.Bd[a].double())
    # the base oracle takes f32 weights: the merged matrices rounded to f32
    ref = oracle.moe_layer(L.x, ids, w, mg.float(), mu.float(), md.float())
    assert rel_err(out, ref) < 1e-5


def dense_lora_forward(x, Wg, Wu, Wd, ids, w, ad, lora, scale):
    """Every expert on every token in torch fp64, each token with its own
    adapter's deltas, then the routing mask."""
    X = x.double()
    T, E = X.shape[0], Wg.shape[0]
    G = torch.einsum("th,ehi->eti", X, Wg.double())
    U = torch.einsum("th,ehi->eti", X, Wu.double())
    for t in range(T):
        a = int(ad[t])
        if a < 0:
            continue
        s = float(scale[a])
        G[:, t] += s * torch.einsum("h,ehr,eri->ei", X[t], lora.Ag[a].double(), lora.Bg[a].double())
        U[:, t] += s * torch.einsum("h,ehr,eri->ei", X[t], lora.Au[a].double(), lora.Bu[a].double())
    Hh = F.silu(G) * U
    Y = torch.einsum("eti,eih->eth", Hh, Wd.double())
    for t in range(T):
        a = int(ad[t])
        if a < 0:
            continue
        s = float(scale[a])
        Y[:, t] += s * torch.einsum("ei,eir,erh->eh", Hh[:, t], lora.Ad[a].double(),
                                    lora.Bd[a].double())
    mask = torch.zeros(T, E, dtype=torch.float64)
    for t in range(T):
        for j in range(ids.shape[1]):
            mask[t, int(ids[t, j])] += float(w[t, j])
    return torch.einsum("te,eth->th", mask, Y).numpy()


def test_mixed_adapters_vs_dense_fp64():
    L, lora, (g, u, d), ids, w = layer_case(T=20)
    ad = adapter_ids(L.T, 3, seed=5)
    assert (ad < 0).any() and (ad >= 0).any()
    out = oracle.moe_layer_lora(L.x, ids, w, g, u, d, ad, lora.as_dict(), lora.scale)
    ref = dense_lora_forward(L.x, g, u, d, ids, w, ad, lora, lora.scale)
    assert rel_err(out, ref) < 1e-12
    # and the adapters change the tokens that have one
    base = oracle.moe_layer(L.x, ids, w, g, u, d)
    changed = np.abs(out - base).max(axis=1) > 1e-6
    assert changed.tolist() == (ad.numpy() >= 0).tolist()


def test_token_subset_and_adapter_order():
    L, lora, (g, u, d), ids, w = layer_case(T=16)
    ad = adapter_ids(L.T, 3, seed=9)
    full = oracle.moe_layer_lora(L.x, ids, w, g, u, d, ad, lora.as_dict(), lora.scale)
    sub = [3, 15, 0, 3]
    part = oracle.moe_layer_lora(L.x, ids, w, g, u, d, ad, lora.as_dict(), lora.scale,
                                 tokens=sub)
    assert np.array_equal(part, full[sub])
