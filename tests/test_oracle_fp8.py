"""Pins of the oracle's e4m3 codec and FP8 layer against torch.float8_e4m3fn."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import make_layer
from tests.conftest import rel_err
from tests.test_oracle_layer import dense_forward


def torch_decode(codes):
    return torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()


def torch_encode_sat(v):
    """Saturating RNE through torch's (non-saturating) cast: clamp first."""
    t = torch.tensor(v, dtype=torch.float32)
    t = torch.where(torch.isnan(t), t, t.clamp(-448.0, 448.0))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_exhaustive():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_decode(codes)
    ref = torch_decode(codes)
    same = (mine == ref) | (np.isnan(mine) & np.isnan(ref))
    assert same.all()
    assert np.isnan(mine[[0x7F, 0xFF]]).all() and np.isfinite(np.delete(mine, [0x7F, 0xFF])).all()
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6


def test_encode_sweep():
    vals = torch_decode(np.arange(256, dtype=np.uint8))
    fin = np.sort(np.unique(vals[np.isfinite(vals)]))
    mids = (fin[:-1].astype(np.float64) + fin[1:]) / 2          # exact ties
    mids = mids.astype(np.float32)
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(-np.inf))
    rng = np.random.default_rng(0)
    rnd = (rng.standard_normal(20000) * np.exp(rng.uniform(-14, 7, 20000))).astype(np.float32)
    edge = np.array([0.0, -0.0, 448.0, -448.0, 449.0, 464.0, 465.0, -500.0, 1e30, np.inf,
                     -np.inf, 2.0 ** -10, 2.0 ** -9, 3 * 2.0 ** -11, 2.0 ** -7, np.nan],
                    np.float32)
    v = np.concatenate([fin, mids, up, dn, rnd, edge])
    mine = oracle.e4m3_encode(v)
    ref = torch_encode_sat(v)
    assert np.array_equal(mine, ref)


def test_quantize_scale():
    t = torch.tensor([[0.5, -3.5], [1.75, 0.0]], dtype=torch.bfloat16)
    s, q = oracle.fp8_quantize(t)
    assert s == np.float32(3.5) / np.float32(448)
    assert q[0, 1] == 0xFE  # -448
    s0, q0 = oracle.fp8_quantize(torch.zeros(3, 3))
    assert s0 == 1.0 and np.all(q0 == 0)


def qdq_torch(t, s=None):
    """Quantise-dequantise with torch's cast: s = amax/448 (float), RNE, saturate."""
    t32 = t.float()
    if s is None:
        amax = t32.abs().max()
        s = (amax / 448.0) if amax > 0 else torch.tensor(1.0)
    s = torch.as_tensor(s, dtype=torch.float32)
    q = (t32 / s).clamp(-448, 448).to(torch.float8_e4m3fn)
    return q.to(torch.float64) * s.double(), float(s)


def test_fp8_layer_vs_torch():
    L = make_layer("fp8", T=6, H=128, I=192, E=4, k=2)
    ids, w = oracle.route_topk(L.logits, L.k)
    out, wsc, (sx, sh) = oracle.moe_layer_fp8(L.x, ids, w, L.Wg, L.Wu, L.Wd)
    # independent: torch casts + fp64 einsums
    qd = [[qdq_torch(W[e]) for e in range(L.E)] for W in (L.Wg, L.Wu, L.Wd)]
    np.testing.assert_array_equal(wsc, np.array([[qd[m][e][1] for m in range(3)]
                                                 for e in range(L.E)], np.float32))
    Wg = torch.stack([qd[0][e][0] for e in range(L.E)])
    Wu = torch.stack([qd[1][e][0] for e in range(L.E)])
    Wd = torch.stack([qd[2][e][0] for e in range(L.E)])
    X, sx_ref = qdq_torch(L.x)
    assert sx == sx_ref
    Hh = []
    for t in range(L.T):
        for j in range(L.k):
            e = int(ids[t, j])
            Hh.append(F.silu(X[t] @ Wg[e]) * (X[t] @ Wu[e]))
    Hh = torch.stack(Hh)
    amax = Hh.abs().max()
    sh_ref = np.float32(np.float32(amax.item()) / np.float32(448))
    assert sh == sh_ref
    Hq = (Hh.float() / torch.tensor(sh_ref)).clamp(-448, 448).to(torch.float8_e4m3fn)
    Hq = Hq.double() * float(sh_ref)
    ref = np.zeros((L.T, L.H))
    for t in range(L.T):
        for j in range(L.k):
            e = int(ids[t, j])
            ref[t] += w[t, j] * (Hq[t * L.k + j] @ Wd[e]).numpy()
    assert rel_err(out, ref) < 1e-12


def test_fp8_layer_near_unquantised_layer():
    """Sanity: e4m3 keeps 3 mantissa bits, so the FP8 layer sits within a few
    percent (max-normalised, here ~7%) of the unquantised layer; a wrong scale
    direction or a dropped scale would be off by orders of magnitude."""
    L = make_layer("fp8", T=8, H=256, I=256, E=4, k=2)
    ids, w = oracle.route_topk(L.logits, L.k)
    out8, _, _ = oracle.moe_layer_fp8(L.x, ids, w, L.Wg, L.Wu, L.Wd)
    ref = oracle.moe_layer(L.x, ids, w, L.Wg, L.Wu, L.Wd)
    assert rel_err(out8, ref) < 0.15
