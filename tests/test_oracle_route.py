"""Pins of the oracle's router: hand-derived cases, brute force, closed forms."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f(v):
    return float("nan") if v == "nan" else float(v)


def _beats(a, ia, b, ib):
    na, nb = math.isnan(a), math.isnan(b)
    if na and nb:
        return ia < ib
    if na:
        return False
    if nb:
        return True
    if a != b:
        return a > b
    return ia < ib


def brute_route(row, k):
    """The unique k-subset whose members all beat all non-members, by enumeration."""
    E = len(row)
    winners = []
    for S in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in S]
        if all(_beats(row[s], s, row[r], r) for s in S for r in rest):
            winners.append(S)
    assert len(winners) == 1
    S = list(winners[0])
    # order the subset: selection sort by the same total order
    out = []
    while S:
        best = S[0]
        for s in S[1:]:
            if _beats(row[s], s, row[best], best):
                best = s
        out.append(best)
        S.remove(best)
    sel = np.array([row[s] for s in out], np.float64)
    e = np.exp(sel - sel.max())
    return out, e / e.sum()


def test_golden_cases():
    with open(os.path.join(GOLDEN, "route_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        lg = np.array([[_f(v) for v in c["logits"]]], np.float32)
        ids, w = oracle.route_topk(lg, c["k"])
        assert ids[0].tolist() == c["ids"], c["why"]
        if c["w"] is not None:
            np.testing.assert_allclose(w[0], c["w"], rtol=1e-15, atol=0)


@pytest.mark.parametrize("E,k", [(2, 1), (4, 2), (8, 2), (8, 3), (8, 8), (6, 4), (1, 1)])
def test_brute_force(E, k):
    rng = np.random.default_rng(E * 100 + k)
    T = 64
    lg = rng.standard_normal((T, E)).astype(np.float32)
    # plant ties, signed zeros and NaNs
    lg[::7, :] = np.round(lg[::7, :])
    lg[3, 0] = -0.0
    if E > 1:
        lg[3, 1] = 0.0
        lg[5, E - 1] = np.nan
        lg[9, :2] = np.nan
    ids, w = oracle.route_topk(lg, k)
    for t in range(T):
        bi, bw = brute_route(lg[t].tolist(), k)
        assert ids[t].tolist() == bi
        if not np.isnan(bw).any():
            np.testing.assert_allclose(w[t], bw, rtol=1e-14, atol=1e-300)


def test_closed_forms():
    rng = np.random.default_rng(1)
    lg = rng.standard_normal((32, 16)).astype(np.float32)
    ids, w = oracle.route_topk(lg, 1)
    assert np.all(w == 1.0)
    assert np.array_equal(ids[:, 0], np.argmax(lg, axis=1))
    ids, w = oracle.route_topk(np.zeros((4, 8), np.float32), 8)
    assert np.all(ids == np.arange(8)) and np.allclose(w, 1 / 8, rtol=0, atol=1e-16)
    ids, w = oracle.route_topk(lg, 5)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    # weights are a softmax of the selected logits: ratios are exp of differences
    sel = np.take_along_axis(lg, ids, axis=1).astype(np.float64)
    np.testing.assert_allclose(w[:, 1] / w[:, 0], np.exp(sel[:, 1] - sel[:, 0]), rtol=1e-13)
    assert np.all(np.diff(sel, axis=1) <= 0)


def test_selection_invariant_to_softmax():
    """Selecting on logits equals selecting on the full softmax (R1)."""
    rng = np.random.default_rng(2)
    lg = (rng.standard_normal((64, 32)) * 3).astype(np.float32)
    ids, _ = oracle.route_topk(lg, 4)
    p = np.exp(lg.astype(np.float64) - lg.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ref = np.argsort(-p, axis=1, kind="stable")[:, :4]
    assert np.array_equal(ids, ref)
