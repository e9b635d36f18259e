"""Seeded synthetic inputs for the fused MoE layer.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark.  It only draws random numbers and forms the router logits; it holds
none of the layer's arithmetic (no routing, no permutation, no expert FFN).

Workloads (shapes from the five configurations this library is measured on):

  tiny     T=16,  H=256,  I=512,   E=8,   k=2   fp32 master weights
  decode   T in {1,4,16,64}, H=4096, I=14336, E=8, k=2   bf16, uniform routing
  prefill  T=4096, H=2048, I=768,  E=128, k=8   bf16, ~256 tokens per expert
  fp8      T in {1,32,256,2048}, H=I=2880, E=32, k=4   bf16 masters -> e4m3
  skewed   T=8192, H=7168, I=2048, E=256, k=8   bf16, Zipf(1.2) expert bias

Recipe (identical for every workload):
  * weights: one torch.Generator seeded with ``seed`` draws, in this order,
    W_r, the bias ranks (skewed only), W_g, W_u, W_d (one expert at a time);
  * inputs: batch b of T tokens is drawn by its own generator seeded
    batch_seed(seed, T, b), so any number of batches share one weight set;
  * x ~ N(0, 1); W_r ~ N(0, 1/sqrt(H)) (std); W_g, W_u ~ N(0, 1/sqrt(H));
    W_d ~ N(0, 1/sqrt(I)) -- "N(0, 1/sqrt(fan_in))" read as a standard
    deviation, which keeps activations O(1);
  * logits = float32(x_f64 @ W_r_f64) + bias, with bias = 0 except for the
    skewed workload, where experts get a seeded random popularity rank r_e
    (1 = most popular) and bias_e = -1.2 * ln(r_e);
  * the router projection is formed here because the layer starts from
    float32 logits; both the oracle and the GPU path read the same buffer.

Weights live in the layout the layer's callers hand over: W_g, W_u [E, H, I]
and W_d [E, I, H], row-major.  Large workloads may draw their weights on a
CUDA device (torch's Philox generator) to avoid minutes of host sampling; the
values then differ from the CPU draw of the same seed, and tests that need
them on the host copy them back.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

ZIPF_S = 1.2

CONFIGS = {
    "tiny": dict(H=256, I=512, E=8, k=2, T=(16,), master="fp32"),
    "decode": dict(H=4096, I=14336, E=8, k=2, T=(1, 4, 16, 64), master="bf16"),
    "prefill": dict(H=2048, I=768, E=128, k=8, T=(4096,), master="bf16"),
    "fp8": dict(H=2880, I=2880, E=32, k=4, T=(1, 32, 256, 2048), master="bf16"),
    "skewed": dict(H=7168, I=2048, E=256, k=8, T=(8192,), master="bf16", zipf=True),
}


@dataclass
class Layer:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    x: torch.Tensor            # [T, H] bf16
    logits: torch.Tensor       # [T, E] f32
    Wg: torch.Tensor           # [E, H, I] bf16 (fp32 for the tiny master copy)
    Wu: torch.Tensor           # [E, H, I]
    Wd: torch.Tensor           # [E, I, H]
    Wr: torch.Tensor           # [H, E] f32
    bias: torch.Tensor         # [E] f32
    meta: dict = field(default_factory=dict)

    def weights_bf16(self):
        """The expert weights rounded to bf16 (the GPU path's precision)."""
        return (self.Wg.to(torch.bfloat16), self.Wu.to(torch.bfloat16),
                self.Wd.to(torch.bfloat16))


def _normal(gen, shape, std, device, dtype):
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=gen)
    return t.to(dtype)


def zipf_bias(E: int, gen: torch.Generator, s: float = ZIPF_S) -> torch.Tensor:
    """Per-expert bias: a seeded random rank r_e in 1..E, bias_e = -s*ln(r_e)."""
    perm = torch.randperm(E, generator=gen)            # perm[rank-1] = expert
    rank = torch.empty(E, dtype=torch.float64)
    rank[perm] = torch.arange(1, E + 1, dtype=torch.float64)
    return (-s * torch.log(rank)).to(torch.float32)


def batch_seed(seed: int, T: int, batch: int) -> int:
    """Seed of input batch ``batch`` with T tokens (independent of the weights' draw)."""
    return seed * 1_000_003 + 7919 * (batch + 1) + T


@dataclass
class Weights:
    name: str
    H: int
    I: int
    E: int
    k: int
    Wg: torch.Tensor           # [E, H, I]
    Wu: torch.Tensor           # [E, H, I]
    Wd: torch.Tensor           # [E, I, H]
    Wr: torch.Tensor           # [H, E] f32 (CPU)
    bias: torch.Tensor         # [E] f32 (CPU)


def make_weights(name: str, seed: int = 0, device: str = "cpu", E: int | None = None,
                 k: int | None = None, H: int | None = None, I: int | None = None,
                 zero_router: bool = False, router_only: bool = False) -> Weights:
    """Router and expert weights of a workload.  Generator(seed) draws, in order,
    W_r, the Zipf ranks (skewed only), then W_g, W_u, W_d one expert at a time.
    On a CUDA ``device`` the expert weights come from a CUDA generator seeded
    seed + 1 (different values, same distribution).  ``router_only`` stops after
    the router (same W_r and bias; the expert tensors are left empty)."""
    cfg = dict(CONFIGS[name])
    H = H or cfg["H"]
    I = I or cfg["I"]
    E = E or cfg["E"]
    k = k or cfg["k"]
    wdtype = torch.float32 if cfg["master"] == "fp32" else torch.bfloat16
    gen = torch.Generator(device="cpu").manual_seed(seed)
    Wr = _normal(gen, (H, E), 1.0 / math.sqrt(H), "cpu", torch.float32)
    if zero_router:
        Wr.zero_()
    bias = zipf_bias(E, gen) if cfg.get("zipf") else torch.zeros(E, dtype=torch.float32)
    if router_only:
        empty = torch.empty(0, dtype=wdtype)
        return Weights(name, H, I, E, k, empty, empty, empty, Wr, bias)
    wgen = gen if device == "cpu" else torch.Generator(device=device).manual_seed(seed + 1)
    Wg = torch.empty((E, H, I), dtype=wdtype, device=device)
    Wu = torch.empty((E, H, I), dtype=wdtype, device=device)
    Wd = torch.empty((E, I, H), dtype=wdtype, device=device)
    # one expert at a time keeps the float32 staging buffer small
    for W, std in ((Wg, 1.0 / math.sqrt(H)), (Wu, 1.0 / math.sqrt(H)), (Wd, 1.0 / math.sqrt(I))):
        for e in range(E):
            W[e] = _normal(wgen, W.shape[1:], std, device, wdtype)
    return Weights(name, H, I, E, k, Wg, Wu, Wd, Wr, bias)


def make_batch(W: Weights, T: int, seed: int = 0, batch: int = 0):
    """x ~ N(0,1) bf16 [T, H] and logits = f32(x W_r in f64) + bias [T, E] (CPU)."""
    gen = torch.Generator(device="cpu").manual_seed(batch_seed(seed, T, batch))
    x = _normal(gen, (T, W.H), 1.0, "cpu", torch.bfloat16)
    logits = (x.to(torch.float64) @ W.Wr.to(torch.float64)).to(torch.float32) + W.bias
    return x, logits


def make_layer(name: str, T: int | None = None, seed: int = 0, device: str = "cpu",
               E: int | None = None, k: int | None = None, H: int | None = None,
               I: int | None = None, zero_router: bool = False) -> Layer:
    """One workload: its weights plus input batch 0.  Keyword overrides give the
    small variants the tests use; ``zero_router`` sets W_r = 0 (all logits
    equal), a special case the oracle is pinned on."""
    W = make_weights(name, seed, device, E=E, k=k, H=H, I=I, zero_router=zero_router)
    T = CONFIGS[name]["T"][0] if T is None else T
    x, logits = make_batch(W, T, seed, 0)
    return Layer(name, T, W.H, W.I, W.E, W.k, x, logits, W.Wg, W.Wu, W.Wd, W.Wr, W.bias,
                 meta=dict(seed=seed, weight_device=device))


@dataclass
class Lora:
    """Synthetic adapters for multi-LoRA layers (the pages give no adapter
    shapes): n_adapters rank-r pairs per expert and matrix, bf16.
    A_g, A_u [n,E,H,r], B_g, B_u [n,E,r,I], A_d [n,E,I,r], B_d [n,E,r,H];
    scale [n] float32."""
    Ag: torch.Tensor
    Bg: torch.Tensor
    Au: torch.Tensor
    Bu: torch.Tensor
    Ad: torch.Tensor
    Bd: torch.Tensor
    scale: torch.Tensor

    def as_dict(self):
        return dict(Ag=self.Ag, Bg=self.Bg, Au=self.Au, Bu=self.Bu, Ad=self.Ad, Bd=self.Bd)


def make_lora(E: int, H: int, I: int, n_adapters: int = 4, rank: int = 16, seed: int = 0,
              device: str = "cpu") -> Lora:
    """Adapters drawn by Generator(seed): A ~ N(0, 1/sqrt(fan_in)) (std), B ~
    N(0, 0.1/sqrt(rank)) so each delta is about a tenth of its base matrix's
    output; scale_a = 1 + a/4."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    n, r = n_adapters, rank
    mk = lambda shape, std: _normal(gen, shape, std, "cpu", torch.bfloat16).to(device)
    Ag = mk((n, E, H, r), 1.0 / math.sqrt(H))
    Bg = mk((n, E, r, I), 0.1 / math.sqrt(r))
    Au = mk((n, E, H, r), 1.0 / math.sqrt(H))
    Bu = mk((n, E, r, I), 0.1 / math.sqrt(r))
    Ad = mk((n, E, I, r), 1.0 / math.sqrt(I))
    Bd = mk((n, E, r, H), 0.1 / math.sqrt(r))
    scale = torch.tensor([1.0 + a / 4.0 for a in range(n)], dtype=torch.float32)
    return Lora(Ag, Bg, Au, Bu, Ad, Bd, scale)


def adapter_ids(T: int, n_adapters: int, seed: int = 0, base_share: float = 0.25) -> torch.Tensor:
    """Adapter of each token, int32 [T]: -1 (base model only) with probability
    base_share, else uniform over the adapters."""
    gen = torch.Generator().manual_seed(seed * 7 + 3)
    u = torch.rand(T, generator=gen)
    a = torch.randint(0, max(n_adapters, 1), (T,), generator=gen, dtype=torch.int32)
    return torch.where(u < base_share, torch.full_like(a, -1), a)


def random_ids(T: int, E: int, k: int, seed: int = 0, skew: float = 0.0) -> torch.Tensor:
    """Distinct expert ids per token, [T, k] int32: a seeded routing stand-in for
    tests of the permutation alone.  ``skew`` > 0 biases towards low ids."""
    gen = torch.Generator().manual_seed(seed)
    if T == 0:
        return torch.empty((0, k), dtype=torch.int32)
    p = torch.arange(1, E + 1, dtype=torch.float64) ** (-skew)
    p = p.expand(T, E).contiguous()
    return torch.multinomial(p, k, replacement=False, generator=gen).to(torch.int32)
