"""The synthetic workloads have the structure their descriptions promise:
uniform routing spreads tokens over (nearly) all experts, and the Zipf(1.2)
bias of the skewed workload leaves some experts empty while a few take more
than 5% of the tokens each.  Checked on the exact inputs the bench and the
full-size parity tests use (seed 0, batch 0), routed by the oracle."""
import numpy as np
import pytest

import oracle
from workloads import CONFIGS, make_batch, make_weights


def _hist(name, T):
    W = make_weights(name, 0, router_only=True)
    _, logits = make_batch(W, T, 0, 0)
    ids, w = oracle.route_topk(logits, W.k)
    return np.bincount(ids.reshape(-1), minlength=W.E), W


def test_skewed_workload_load_imbalance():
    T = CONFIGS["skewed"]["T"][0]
    counts, W = _hist("skewed", T)
    assert counts.sum() == T * W.k
    assert (counts == 0).sum() >= 1                       # some experts empty
    assert (counts > 0.05 * T).sum() >= 3                 # a few take >5% of the tokens
    assert counts.max() <= T                              # an expert appears once per token


@pytest.mark.parametrize("name", ["prefill", "fp8"])
def test_uniform_workloads_spread(name):
    T = max(CONFIGS[name]["T"])
    counts, W = _hist(name, T)
    mean = T * W.k / W.E
    assert (counts > 0).all()
    assert counts.max() < 2 * mean and counts.min() > 0.5 * mean
