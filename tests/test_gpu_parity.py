"""GPU parity: every entry point through the C ABI against the CPU oracle.

Routing ids, permutation, offsets and tiles bit-exact; routing weights within
1e-6 relative; layer outputs within 2e-2 (bf16) / 6e-2 (FP8) max-normalised.
Shapes span several tiles with ragged tails (token tiles, weight tiles, K
blocks), stream-K splits (capped grids), padding variants and edge cases."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import (TOL, assert_close, check_permutation, check_routing, lib,
                               oracle_layer, to_host)
from workloads import make_layer, random_ids

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def moe():
    return lib()


def test_wait_timeout_reports_status(moe):
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.selftest_wait_timeout(st, 20000)
    assert moe.check_status(st) == 5          # MOE_ERR_TIMEOUT
    # the context is still usable afterwards
    st.zero_()
    assert moe.check_status(st) == 0
    assert torch.ones(4, device=DEV).sum().item() == 4


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (16, 8, 2), (33, 4, 4), (100, 32, 4),
                                   (257, 128, 8), (64, 256, 8), (40, 64, 64), (5, 256, 256),
                                   (4096, 128, 8), (3, 1, 1), (50, 33, 5)])
def test_route_topk_bit_exact(moe, T, E, k):
    g = torch.Generator().manual_seed(T * 1000 + E)
    lg = torch.randn(T, E, generator=g)
    lg[::3] = torch.round(lg[::3] * 2) / 2           # ties
    if T > 2 and E > 2:
        lg[1, 0] = -0.0
        lg[1, 1] = 0.0
        lg[2, E // 2] = float("nan")
    ids, w = moe.route_topk(lg.to(DEV), k)
    torch.cuda.synchronize()
    check_routing(ids, w, lg)


@pytest.mark.parametrize("T,E,k,bm,skew", [(0, 8, 2, 16, 0.0), (1, 8, 2, 16, 0.0),
                                           (64, 8, 2, 16, 0.0), (300, 32, 4, 64, 1.0),
                                           (1024, 128, 8, 16, 0.0), (4096, 128, 8, 128, 0.0),
                                           (8192, 256, 8, 16, 1.2), (5000, 7, 3, 32, 2.0),
                                           (100, 256, 8, 16, 0.0),
                                           # chunk edges of the multi-CTA path (512 per chunk):
                                           # one past the single-CTA limit, exact multiples,
                                           # a last chunk of one assignment, E = 256 skewed
                                           (2049, 8, 1, 16, 0.0), (1024, 64, 4, 16, 0.5),
                                           (3073, 5, 1, 16, 0.0), (16384, 256, 2, 64, 1.5),
                                           # small batches: E above 32, every expert, E = 1
                                           (16, 8, 2, 16, 0.0), (3, 256, 8, 16, 0.0),
                                           (4, 8, 8, 32, 0.0), (31, 1, 1, 16, 0.0)])
def test_align_permute_bit_exact(moe, T, E, k, bm, skew):
    ids = random_ids(T, E, k, seed=T + k, skew=skew)
    perm = moe.align_permute(ids.to(DEV), E, bm)
    torch.cuda.synchronize()
    check_permutation(perm, ids.numpy(), E, bm)


def expected_packed_rows(Wg, Wu, Wd):
    """Packed row order: gate/up rows interleaved by 16, W_d transposed (K-major)."""
    E, H, I = Wg.shape
    gt = Wg.transpose(1, 2).reshape(E, I // 16, 16, H)
    ut = Wu.transpose(1, 2).reshape(E, I // 16, 16, H)
    gu = torch.stack([gt, ut], dim=2).reshape(E, 2 * I, H)
    dn = Wd.transpose(1, 2).contiguous()
    return gu.contiguous(), dn


def tile_image(M, bk):
    """[E, R, K] -> bytes of 16 KB tiles (128 rows x 128 B), zero-padded, each
    in the 128-byte-swizzle layout: 16-byte chunk c of row r at c ^ (r % 8)."""
    E, R, K = M.shape
    MT, KB = -(-R // 128), -(-K // bk)
    pad = torch.zeros((E, MT * 128, KB * bk), dtype=M.dtype)
    pad[:, :R, :K] = M
    t = pad.view(E, MT, 128, KB, bk).permute(0, 1, 3, 2, 4).contiguous()
    b = t.view(torch.uint8).view(E, MT, KB, 128, 8, 16)
    r = torch.arange(128).view(128, 1)
    c = torch.arange(8).view(1, 8)
    idx = (c ^ (r % 8)).view(1, 1, 1, 128, 8, 1).expand_as(b)
    return torch.gather(b, 4, idx).reshape(-1)


@pytest.mark.parametrize("E,H,I", [(3, 128, 192), (2, 320, 64)])
def test_pack_weights_layout(moe, E, H, I):
    L = make_layer("decode", T=1, E=E, H=H, I=I, k=1)
    Wg, Wu, Wd = (W.to(DEV) for W in (L.Wg, L.Wu, L.Wd))
    packed, _ = moe.pack_weights(moe.BF16, Wg, Wu, Wd)
    torch.cuda.synchronize()
    gu, dn = expected_packed_rows(L.Wg, L.Wu, L.Wd)
    ref = torch.cat([tile_image(gu, 64), tile_image(dn, 64)])
    assert torch.equal(to_host(packed), ref)


def test_pack_weights_fp8_codes(moe):
    E, H, I = 3, 320, 192                       # ragged tiles in both directions
    L = make_layer("fp8", T=1, E=E, H=H, I=I, k=1)
    Wg, Wu, Wd = (W.to(DEV) for W in (L.Wg, L.Wu, L.Wd))
    packed, scales = moe.pack_weights(moe.FP8_E4M3, Wg, Wu, Wd)
    torch.cuda.synchronize()
    codes = {}
    for m, W in enumerate((L.Wg, L.Wu, L.Wd)):
        for e in range(E):
            s, q = oracle.fp8_quantize(W[e])
            assert to_host(scales)[e, m].item() == s
            codes[(m, e)] = torch.from_numpy(q)
    qg, qu, qd = (torch.stack([codes[(m, e)] for e in range(E)]) for m in range(3))
    gu, dn = expected_packed_rows(qg, qu, qd)
    ref = torch.cat([tile_image(gu, 128), tile_image(dn, 128)])
    assert torch.equal(to_host(packed), ref)


def run_forward(moe, dtype, L, block_m=0, max_ctas=0, ws=None, combine=0):
    Wg, Wu, Wd = (W.to(DEV) for W in L.weights_bf16())
    packed, scales = moe.pack_weights(dtype, Wg, Wu, Wd)
    x = L.x.to(DEV)
    logits = L.logits.to(DEV)
    ids = torch.empty((L.T, L.k), dtype=torch.int32, device=DEV)
    w = torch.empty((L.T, L.k), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = moe.forward(dtype, x, logits, packed, scales, L.E, L.I, L.k, ids=ids, w=w, status=st,
                      block_m=block_m, max_ctas=max_ctas, ws=ws, combine=combine)
    assert moe.check_status(st) == 0
    return out, ids, w


LAYER_CASES = [
    # name, T, E, k, H, I
    ("tiny", 16, 8, 2, 256, 512),        # the tiny workload (bf16-rounded weights)
    ("tiny", 37, 8, 2, 256, 320),        # 5 gate/up weight tiles, ragged token counts
    ("tiny", 300, 4, 2, 320, 192),       # ragged down weight tile (320 rows), N up to 256
    ("tiny", 1, 8, 2, 512, 256),         # decode-shaped, 1 token
    ("tiny", 5, 16, 16, 128, 128),       # k = E: every expert
    ("tiny", 700, 2, 1, 192, 128),       # two token tiles per expert (256 + ragged)
    ("tiny", 9, 1, 1, 256, 256),         # E = 1: dense SwiGLU
    ("tiny", 40, 2, 2, 256, 256),        # pair tiles, token cap 2*mean = 80 (not a multiple of 32)
    ("tiny", 56, 2, 2, 192, 128),        # pair tiles, 2*mean = 112
    # small batches: 32 assignments, and E above 32 with k = 8
    ("tiny", 16, 8, 2, 256, 256),
    ("tiny", 3, 64, 8, 128, 128),
    # past the single-CTA permutation (T*k > 2048): route, count, scan+scatter
    ("tiny", 1100, 8, 2, 256, 256),      # 5 chunks, pair tiles (gather kernel between)
    ("tiny", 300, 128, 8, 128, 128),     # 5 chunks, one-CTA tiles: the GEMM follows scan+scatter
    ("tiny", 520, 64, 8, 128, 192),      # 9 chunks, pair tiles
    ("tiny", 800, 16, 3, 128, 192),      # k = 3, pair tiles
    ("tiny", 1000, 96, 3, 128, 128),     # k = 3, one-CTA tiles
]


# the two forms of the combine: y_perm rows summed in j order, and the
# down GEMM's epilogue reducing into an fp32 token-order accumulator
COMBINES = [1, 2]


@pytest.mark.parametrize("combine", COMBINES)
@pytest.mark.parametrize("dtype", [0, 1])
@pytest.mark.parametrize("case", LAYER_CASES)
def test_forward_small(moe, dtype, case, combine):
    name, T, E, k, H, I = case
    L = make_layer(name, T=T, E=E, k=k, H=H, I=I, seed=T + E)
    out, ids, w = run_forward(moe, dtype, L, combine=combine)
    ids_o, w_o = check_routing(ids, w, L.logits)
    g, u, d = L.weights_bf16()
    ref = oracle_layer(dtype, L.x, ids_o, w_o, g, u, d)
    assert_close(out, ref, dtype, f"{case} dtype={dtype}")


@pytest.mark.parametrize("combine", COMBINES)
@pytest.mark.parametrize("max_ctas", [1, 3, 7, 13, 64])
@pytest.mark.parametrize("dtype", [0, 1])
def test_forward_stream_k_splits(moe, dtype, max_ctas, combine):
    """Capped grids cut units mid-K: the fixed-order partial reduction must
    give the same result as the oracle and as the uncapped grid."""
    L = make_layer("tiny", T=45, E=6, k=2, H=384, I=256, seed=5)
    out, ids, w = run_forward(moe, dtype, L, max_ctas=max_ctas, combine=combine)
    ids_o, w_o = check_routing(ids, w, L.logits)
    g, u, d = L.weights_bf16()
    ref = oracle_layer(dtype, L.x, ids_o, w_o, g, u, d)
    assert_close(out, ref, dtype, f"max_ctas={max_ctas}")


@pytest.mark.parametrize("combine", COMBINES)
@pytest.mark.parametrize("max_ctas", [2, 7, 14, 0])
@pytest.mark.parametrize("dtype", [0, 1])
def test_forward_cta_pair_splits(moe, dtype, max_ctas, combine):
    """Large token tiles run on CTA pairs (M = 256 per MMA): odd weight-tile
    counts (5 gate/up, 3 down tiles), ragged token tiles and capped grids that
    split pair units stream-K style."""
    L = make_layer("tiny", T=600, E=4, k=2, H=384, I=320, seed=6)
    out, ids, w = run_forward(moe, dtype, L, max_ctas=max_ctas, combine=combine)
    ids_o, w_o = check_routing(ids, w, L.logits)
    g, u, d = L.weights_bf16()
    ref = oracle_layer(dtype, L.x, ids_o, w_o, g, u, d)
    assert_close(out, ref, dtype, f"pair max_ctas={max_ctas}")


@pytest.mark.parametrize("block_m", [16, 32, 64, 128])
def test_forward_block_m_variants(moe, block_m):
    L = make_layer("tiny", T=50, E=8, k=2, H=256, I=256, seed=9)
    out, ids, w = run_forward(moe, 0, L, block_m=block_m)
    ids_o, w_o = check_routing(ids, w, L.logits)
    g, u, d = L.weights_bf16()
    assert_close(out, oracle.moe_layer(L.x, ids_o, w_o, g, u, d), 0, f"block_m={block_m}")


@pytest.mark.parametrize("dtype", [0, 1])
def test_forward_deterministic(moe, dtype):
    """The deterministic combine (and the fixed-order stream-K reduction) give
    bit-identical outputs run after run."""
    L = make_layer("tiny", T=200, E=8, k=2, H=256, I=256, seed=2)
    outs = [run_forward(moe, dtype, L, max_ctas=11, combine=1)[0] for _ in range(10)]
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_combine_auto_is_deterministic(moe):
    """Auto takes the deterministic combine at every size: bit-identical to the
    explicit mode; the fused reduction matches up to rounding."""
    for T, k, expect in ((100, 2, 1), (1100, 4, 1), (1100, 4, 2)):
        L = make_layer("tiny", T=T, E=8, k=k, H=256, I=256, seed=T)
        auto = run_forward(moe, 0, L, combine=0)[0]
        ref = run_forward(moe, 0, L, combine=expect)[0]
        ids_o, w_o = oracle.route_topk(L.logits, k)
        g, u, d = L.weights_bf16()
        assert_close(auto, oracle.moe_layer(L.x, ids_o, w_o, g, u, d), 0, f"auto T={T}")
        if expect == 1:
            assert torch.equal(auto, ref)
        else:
            assert_close(ref, oracle.moe_layer(L.x, ids_o, w_o, g, u, d), 0, f"fused T={T}")
            # fused sums follow the schedule's order: equal up to rounding
            diff = (auto.float() - ref.float()).abs().max().item()
            assert diff <= 1e-2 * ref.float().abs().max().item()


# FP8 paths of amax(x) and the codes of x: the single-CTA route kernel
# (T = 24 / 48), and the amax and quantisation passes feeding one-CTA tiles
# (T = 200, 64 experts) or the gather of CTA-pair tiles (T = 600, 4 experts)
X_PATHS = [(24, 8), (200, 64), (600, 4)]


@pytest.mark.parametrize("combine", COMBINES)
@pytest.mark.parametrize("T,E", X_PATHS)
def test_fp8_zero_input(moe, combine, T, E):
    """x = 0: amax = 0 gives s_x = 1 (and then h = 0, s_h = 1); the output is
    exactly zero, as the oracle's."""
    L = make_layer("tiny", T=T, E=E, k=2, H=256, I=256, seed=3)
    L.x = torch.zeros_like(L.x)
    out, ids, w = run_forward(moe, 1, L, combine=combine)
    ids_o, w_o = check_routing(ids, w, L.logits)
    g, u, d = L.weights_bf16()
    ref, _, (sx, sh) = oracle.moe_layer_fp8(L.x, ids_o, w_o, g, u, d)
    assert sx == 1.0 and sh == 1.0 and not ref.any()
    assert torch.count_nonzero(out).item() == 0


# bf16 values a for which the fp32 product a * (1 / (a / 448)) rounds above
# 448: the element equal to amax(x) must still get the largest code (448).
@pytest.mark.parametrize("T,E", [(48, 8), (200, 64), (600, 4)])
@pytest.mark.parametrize("amax", [8.1875, 11.25, 15.9375])
def test_fp8_amax_element_saturates(moe, amax, T, E):
    L = make_layer("tiny", T=T, E=E, k=2, H=256, I=256, seed=4)
    x = L.x.clone()
    x[3, 17] = amax
    x[20, 200] = -amax
    x[41, 5] = amax
    L.x = x
    out, ids, w = run_forward(moe, 1, L)
    ids_o, w_o = check_routing(ids, w, L.logits)
    g, u, d = L.weights_bf16()
    ref, _, (sx, _) = oracle.moe_layer_fp8(L.x, ids_o, w_o, g, u, d)
    assert sx == np.float32(np.float32(amax) / np.float32(448.0))
    assert torch.isfinite(out).all()
    assert_close(out, ref, 1, f"planted amax {amax}")


@pytest.mark.parametrize("combine", COMBINES)
@pytest.mark.parametrize("dtype", [0, 1])
def test_nonfinite_logits(moe, dtype, combine):
    """Tokens with NaN, -inf and +inf logits: routing stays bit-exact (NaN
    ranks last, -inf below every number); a +inf selection makes that token's
    weights NaN (exp(inf - inf)) on both sides, and only that token's output;
    every other token matches the oracle."""
    L = make_layer("tiny", T=40, E=8, k=2, H=256, I=256, seed=8)
    lg = L.logits.clone()
    lg[5, 3] = float("nan")
    lg[6, 0] = float("nan")
    lg[6, 7] = float("nan")
    lg[7, 2] = float("-inf")
    lg[8, :6] = float("-inf")            # two finite logits left: they are chosen
    lg[9, 4] = float("inf")
    L.logits = lg
    out, ids, w = run_forward(moe, dtype, L, combine=combine)
    ids_o, w_o = check_routing(ids, w, lg)
    bad = ~np.isfinite(w_o).all(axis=1)
    assert bad.tolist() == [t == 9 for t in range(L.T)]
    assert torch.isnan(w[9]).all()
    good = [t for t in range(L.T) if not bad[t]]
    g, u, d = L.weights_bf16()
    # the oracle on the other tokens (token 9's NaN weights zeroed: they do not
    # enter any other token's output, nor the FP8 scale of h)
    w_fin = np.where(np.isfinite(w_o), w_o, 0.0)
    ref = oracle_layer(dtype, L.x, ids_o, w_fin, g, u, d, tokens=good)
    assert_close(out[good], ref, dtype, f"non-finite logits dtype={dtype}")
    assert not torch.isfinite(out[9]).any()


@pytest.mark.parametrize("T,E", X_PATHS)
def test_fp8_nan_in_x(moe, T, E):
    """A NaN element of x (reading R19): amax(x) skips it on both sides (a
    maximum ignores NaN), it codes as NaN, and only its token's output is NaN;
    every other token matches the oracle."""
    L = make_layer("tiny", T=T, E=E, k=2, H=256, I=256, seed=12)
    x = L.x.clone()
    x[5, 10] = float("nan")
    L.x = x
    out, ids, w = run_forward(moe, 1, L)
    ids_o, w_o = check_routing(ids, w, L.logits)
    g, u, d = L.weights_bf16()
    ref, _, (sx, _) = oracle.moe_layer_fp8(L.x, ids_o, w_o, g, u, d)
    assert np.isfinite(sx)
    assert np.isnan(ref).any(axis=1).tolist() == [t == 5 for t in range(T)]
    assert np.isnan(ref[5]).all()
    o = to_host(out).float()
    assert torch.isnan(o[5]).all()
    good = [t for t in range(T) if t != 5]
    assert torch.isfinite(o[good]).all()
    assert_close(out[good], ref[good], 1, f"NaN in x, T={T}")


@pytest.mark.parametrize("T,E", X_PATHS)
@pytest.mark.parametrize("val", [float("inf"), float("-inf")])
def test_fp8_inf_in_x(moe, T, E, val):
    """An infinite element of x (reading R19) makes amax(x) and s_x = amax/448
    infinite; every finite element then codes as 0 and dequantises to
    0 * inf = NaN, so the whole output is NaN, on both sides."""
    L = make_layer("tiny", T=T, E=E, k=2, H=256, I=256, seed=13)
    x = L.x.clone()
    x[7, 3] = val
    L.x = x
    out, ids, w = run_forward(moe, 1, L)
    ids_o, w_o = check_routing(ids, w, L.logits)
    g, u, d = L.weights_bf16()
    ref, _, (sx, _) = oracle.moe_layer_fp8(L.x, ids_o, w_o, g, u, d)
    assert np.isinf(sx)
    assert np.isnan(ref).all()
    assert torch.isnan(to_host(out).float()).all()


def test_forward_empty_batch(moe):
    L = make_layer("tiny", T=4, E=8, k=2, H=256, I=256)
    Wg, Wu, Wd = (W.to(DEV) for W in L.weights_bf16())
    packed, _ = moe.pack_weights(0, Wg, Wu, Wd)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    lg = torch.empty((0, 8), dtype=torch.float32, device=DEV)
    out = moe.forward(0, x, lg, packed, None, 8, 256, 2)
    assert out.shape == (0, 256)


def test_components_compose_to_forward(moe):
    """route -> align_permute -> grouped_ffn -> combine equals moe_forward."""
    L = make_layer("tiny", T=70, E=8, k=2, H=256, I=320, seed=4)
    Wg, Wu, Wd = (W.to(DEV) for W in L.weights_bf16())
    packed, scales = moe.pack_weights(0, Wg, Wu, Wd)
    x, lg = L.x.to(DEV), L.logits.to(DEV)
    ids, w = moe.route_topk(lg, L.k)
    perm = moe.align_permute(ids, L.E, 16)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    y, _ = moe.grouped_ffn(0, x, w.view(-1), perm, packed, scales, L.E, L.I, L.k, status=st)
    out = moe.combine(y, perm["inv_perm"], L.T, L.k, L.H)
    assert moe.check_status(st) == 0
    ref = moe.forward(0, x, lg, packed, scales, L.E, L.I, L.k, combine=moe.COMBINE_DETERMINISTIC)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
