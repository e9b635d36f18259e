"""Shared helpers of the GPU parity tests (test infrastructure)."""
import numpy as np
import torch

import oracle
from tests.conftest import rel_err

TOL = {0: 2e-2, 1: 6e-2}          # layer output, max-normalised: bf16, FP8
W_RTOL = 1e-6                      # routing weights


def lib():
    from mixture_experts_expert_route_b200 import _lib, build
    build.build(debug=_lib.DEBUG_CHECKS)
    import mixture_experts_expert_route_b200 as moe
    return moe


def to_host(t):
    return t.detach().cpu()


def check_routing(ids_gpu, w_gpu, logits):
    ids_o, w_o = oracle.route_topk(to_host(logits), ids_gpu.shape[1])
    ids_g = to_host(ids_gpu).numpy()
    assert np.array_equal(ids_g, ids_o), "routing ids differ from the oracle"
    w_g = to_host(w_gpu).numpy().astype(np.float64)
    fin = np.isfinite(w_o)
    np.testing.assert_allclose(w_g[fin], w_o[fin], rtol=W_RTOL, atol=1e-12)
    return ids_o, w_o


def check_permutation(perm, ids_np, E, block_m):
    ref = oracle.align_permute(ids_np, E, block_m, capacity=perm["capacity"])
    for key in ("counts", "offsets", "inv_perm"):
        g = to_host(perm[key]).numpy()[: len(ref[key])]
        assert np.array_equal(g, ref[key]), key
    cap = perm["capacity"]
    assert np.array_equal(to_host(perm["sorted_ids"]).numpy()[:cap], ref["sorted_ids"][:cap])
    nt = cap // block_m
    assert np.array_equal(to_host(perm["tiles"]).numpy()[:nt], ref["tiles"][:nt])
    assert int(to_host(perm["num_tiles"])[0]) == ref["num_tiles"]
    return ref


def oracle_layer(dtype, x, ids, w, Wg, Wu, Wd, tokens=None):
    if dtype == 0:
        return oracle.moe_layer(x, ids, w, Wg, Wu, Wd, tokens=tokens)
    out, _, _ = oracle.moe_layer_fp8(x, ids, w, Wg, Wu, Wd, tokens=tokens)
    return out


def assert_close(out_gpu, ref, dtype, what=""):
    y = to_host(out_gpu).to(torch.float64).numpy()
    err = rel_err(y, ref)
    assert err <= TOL[dtype], f"{what}: max rel err {err:.3e} > {TOL[dtype]}"
    return err
