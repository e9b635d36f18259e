"""moe_align_permute_noalloc, the permutation for callers that cannot allocate
device memory or pass a workspace (e.g. a runtime plugin given no workspace).

Calls run back to back through the C ABI; each result must equal the CPU
oracle's permutation bit for bit, and what moe_align_permute (with its
caller-provided workspace) gives.  The cases cover the single-CTA path
(T*k <= 2048, no scratch used), the chunked path that uses the library's
built-in scratch array, and a problem exactly at that array's bound
(ceil(T*k/512) * E == 65536).  The scratch is shared by all calls, so each
later call also checks that nothing left behind by an earlier one leaks into
its results.  Collected last on purpose."""
import numpy as np
import pytest
import torch

from tests.gpu_helpers import check_permutation, lib
from workloads import random_ids

pytestmark = pytest.mark.gpu
DEV = "cuda"

KEYS = ("counts", "offsets", "sorted_ids", "inv_perm", "tiles", "num_tiles")
SCRATCH_INTS = 65536

CASES = [(8192, 256, 8, 16, 1.2),    # 128 chunks x 256 experts of built-in scratch
         (3000, 32, 4, 64, 0.5),     # fewer experts: stale counters must not leak
         (200, 64, 8, 16, 0.0),      # T*k = 1600 <= 2048: one CTA, no scratch
         (16384, 256, 8, 16, 0.3)]   # exactly at the bound: 256 chunks x 256 experts


def test_bound_case_is_at_the_limit():
    T, E, k = CASES[-1][:3]
    assert -(-T * k // 512) * E == SCRATCH_INTS


def test_noalloc_matches_oracle_and_workspace_entry():
    moe = lib()
    results = []
    for T, E, k, bm, skew in CASES:
        ids = random_ids(T, E, k, seed=T, skew=skew).to(DEV)
        got = moe._lib.align_permute_noalloc(ids, E, bm)   # the calls run back to back
        results.append((ids, E, bm, got))
    torch.cuda.synchronize()
    for ids, E, bm, got in results:
        check_permutation(got, ids.cpu().numpy(), E, bm)
        ref = moe.align_permute(ids, E, bm)
        torch.cuda.synchronize()
        for key in KEYS:
            assert torch.equal(got[key], ref[key]), key


def test_noalloc_twice_same_inputs():
    """Two identical calls in a row give identical results (the second reads
    scratch the first left behind)."""
    moe = lib()
    ids = random_ids(5000, 128, 8, seed=11, skew=0.8).to(DEV)
    a = moe._lib.align_permute_noalloc(ids, 128, 32)
    b = moe._lib.align_permute_noalloc(ids, 128, 32)
    torch.cuda.synchronize()
    check_permutation(b, ids.cpu().numpy(), 128, 32)
    for key in KEYS:
        assert np.array_equal(a[key].cpu().numpy(), b[key].cpu().numpy()), key


def test_noalloc_rejects_problems_beyond_its_scratch():
    moe = lib()
    # ceil(T*k/512) * E > 65536 counters: refused before any launch
    T, k, E = 16385, 8, 256
    assert -(-T * k // 512) * E > SCRATCH_INTS
    ids = torch.zeros((1, 1), dtype=torch.int32, device=DEV)   # never read
    lib_ = moe.lib()
    cap = moe.permute_capacity(T, k, E, 16)
    buf = torch.empty(16, dtype=torch.int32, device=DEV)
    p = buf.data_ptr()
    rc = lib_.moe_align_permute_noalloc(ids.data_ptr(), T, k, E, 16, p, p, p, p, p, p, cap,
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == 3   # MOE_ERR_WORKSPACE
