"""Pins of the oracle's permutation: a hand-derived case, invariants, stable sort."""
import json
import os

import numpy as np
import pytest

import oracle
from workloads import random_ids

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_case():
    with open(os.path.join(GOLDEN, "permute_case.json")) as f:
        g = json.load(f)
    out = oracle.align_permute(np.array(g["ids"], np.int32), g["E"], g["block_m"])
    assert out["capacity"] == g["capacity"]
    for key in ("counts", "offsets", "sorted_ids", "inv_perm", "tiles"):
        assert out[key].tolist() == g[key], key
    assert out["num_tiles"] == g["num_tiles"]


def check_invariants(ids, E, bm, out):
    T, k = ids.shape
    A = T * k
    c, o, s, inv = out["counts"], out["offsets"], out["sorted_ids"], out["inv_perm"]
    assert c.sum() == A
    assert o[0] == 0 and np.all(np.diff(o) >= 0) and np.all(o % bm == 0)
    assert np.all(np.diff(o) == (c + bm - 1) // bm * bm)
    valid = s[s >= 0]
    assert sorted(valid.tolist()) == list(range(A))
    assert np.all(s[s < 0] == -1)
    if A:
        assert np.array_equal(s[inv], np.arange(A))
    tiles = out["tiles"]
    nt = out["num_tiles"]
    assert nt * bm == o[E]
    for e in range(E):
        assert np.all(tiles[o[e] // bm:o[e + 1] // bm] == e)
    assert np.all(tiles[nt:] == -1)


def stable_sort_reference(ids, E, bm):
    """Brute force: stable sort of (expert, flat index) pairs, then pad."""
    flat = ids.reshape(-1)
    pairs = sorted(range(len(flat)), key=lambda f: (int(flat[f]), f))
    rows = []
    for e in range(E):
        seg = [f for f in pairs if flat[f] == e]
        if seg:
            seg = seg + [-1] * ((-len(seg)) % bm)
        rows += seg
    return rows


@pytest.mark.parametrize("T,E,k,bm,skew", [
    (0, 8, 2, 16, 0.0), (1, 8, 2, 16, 0.0), (3, 3, 3, 1, 0.0), (17, 8, 2, 64, 0.0),
    (64, 8, 2, 16, 0.0), (200, 32, 4, 16, 1.5), (300, 128, 8, 128, 0.0), (50, 256, 8, 16, 1.2),
    (33, 1, 1, 16, 0.0),
])
def test_invariants_and_stable_sort(T, E, k, bm, skew):
    ids = random_ids(T, E, k, seed=T + E, skew=skew).numpy()
    out = oracle.align_permute(ids, E, bm)
    check_invariants(ids, E, bm, out)
    ref = stable_sort_reference(ids, E, bm)
    assert out["sorted_ids"][: len(ref)].tolist() == ref
    assert np.all(out["sorted_ids"][len(ref):] == -1)
