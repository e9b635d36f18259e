"""Multi-LoRA layers on the GPU through the C ABI against the oracle
(oracle_moe_layer_lora): per-token adapters (-1 = base model), rank-r deltas
on every expert matrix, bf16.  Shapes cover one-CTA tiles (gathered rows),
CTA-pair tiles, ragged weight tiles, stream-K splits, several adapter counts
and ranks, and a prefill-sized layer on sampled tokens."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import assert_close, check_routing, lib
from workloads import adapter_ids, make_layer, make_lora

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def moe():
    return lib()


def run_lora(moe, L, lora, ad, max_ctas=0, combine=0, tokens=None):
    Wg, Wu, Wd = (W.to(DEV) for W in L.weights_bf16())
    packed, _ = moe.pack_weights(moe.BF16, Wg, Wu, Wd)
    dl = moe.Lora(*(m.to(DEV) for m in (lora.Ag, lora.Bg, lora.Au, lora.Bu, lora.Ad, lora.Bd)),
                  lora.scale)
    ids = torch.empty((L.T, L.k), dtype=torch.int32, device=DEV)
    w = torch.empty((L.T, L.k), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = moe.forward(moe.BF16, L.x.to(DEV), L.logits.to(DEV), packed, None, L.E, L.I, L.k,
                      ids=ids, w=w, status=st, max_ctas=max_ctas, combine=combine, lora=dl,
                      adapter=ad.to(DEV))
    assert moe.check_status(st) == 0
    ids_o, w_o = check_routing(ids, w, L.logits)
    g, u, d = L.weights_bf16()
    ref = oracle.moe_layer_lora(L.x, ids_o, w_o, g, u, d, ad, lora.as_dict(), lora.scale,
                                tokens=tokens)
    return out, ref


CASES = [
    # T, E, k, H, I, n_adapters, rank
    (16, 8, 2, 256, 512, 4, 16),     # one-CTA tiles
    (37, 8, 2, 256, 320, 3, 8),      # ragged weight tiles (5 gate/up tiles)
    (300, 4, 2, 320, 192, 4, 16),    # CTA pairs, ragged down tile
    (700, 2, 1, 192, 128, 2, 32),    # two token tiles per expert
    (5, 16, 16, 128, 128, 1, 64),    # k = E, one adapter of rank 64
]


@pytest.mark.parametrize("case", CASES)
def test_lora_layer_small(moe, case):
    T, E, k, H, I, n, r = case
    L = make_layer("tiny", T=T, E=E, k=k, H=H, I=I, seed=T + E)
    lora = make_lora(E, H, I, n_adapters=n, rank=r, seed=T)
    ad = adapter_ids(T, n, seed=T)
    out, ref = run_lora(moe, L, lora, ad)
    assert_close(out, ref, 0, f"lora {case}")
    # the adapters changed the output of the tokens that have one
    base = oracle.moe_layer(L.x, *oracle.route_topk(L.logits, k), *L.weights_bf16())
    moved = np.abs(ref - base).max(axis=1) > 1e-3 * np.abs(base).max()
    assert moved.any()


@pytest.mark.parametrize("max_ctas", [3, 14])
def test_lora_stream_k_splits(moe, max_ctas):
    L = make_layer("tiny", T=600, E=4, k=2, H=384, I=320, seed=6)
    lora = make_lora(4, 384, 320, n_adapters=4, rank=16, seed=6)
    ad = adapter_ids(600, 4, seed=6)
    out, ref = run_lora(moe, L, lora, ad, max_ctas=max_ctas)
    assert_close(out, ref, 0, f"lora max_ctas={max_ctas}")


def test_lora_all_base_tokens_equal_base_layer(moe):
    """Every token on the base model (-1): the masked shrink outputs are zero,
    so the expand adds exact zeros; the result matches the layer without
    adapters up to the fp32 summation grouping (the two extra k-blocks move
    the stream-K split points), and the base oracle."""
    L = make_layer("tiny", T=50, E=8, k=2, H=256, I=256, seed=3)
    lora = make_lora(8, 256, 256, n_adapters=4, rank=16, seed=3)
    ad = torch.full((50,), -1, dtype=torch.int32)
    out, _ = run_lora(moe, L, lora, ad)
    Wg, Wu, Wd = (W.to(DEV) for W in L.weights_bf16())
    packed, _ = moe.pack_weights(moe.BF16, Wg, Wu, Wd)
    plain = moe.forward(moe.BF16, L.x.to(DEV), L.logits.to(DEV), packed, None, 8, 256, 2)
    torch.cuda.synchronize()
    diff = (out.float() - plain.float()).abs().max().item()
    assert diff <= 2 ** -7 * plain.float().abs().max().item()
    ids_o, w_o = oracle.route_topk(L.logits, 2)
    assert_close(out, oracle.moe_layer(L.x, ids_o, w_o, *L.weights_bf16()), 0, "lora, no adapter")


def test_lora_prefill_shape(moe):
    """The prefill shape (H=2048, I=768, E=128, top-8, T=4096) with four rank-16
    adapters, checked on sampled tokens."""
    from workloads import CONFIGS
    c = CONFIGS["prefill"]
    L = make_layer("prefill", seed=0)
    lora = make_lora(c["E"], c["H"], c["I"], n_adapters=4, rank=16, seed=1)
    ad = adapter_ids(L.T, 4, seed=1)
    rng = np.random.default_rng(0)
    tok = sorted(rng.choice(L.T, size=96, replace=False).tolist())
    out, ref = run_lora(moe, L, lora, ad, tokens=tok)
    assert_close(out[tok], ref, 0, "lora prefill")
