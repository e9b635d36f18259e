"""moe_align_permute_noalloc, the permutation for callers that cannot allocate
device memory or pass a workspace (e.g. a runtime plugin given no workspace):
two calls in a row through the C ABI must give exactly what moe_align_permute
(with its caller-provided workspace) gives.  Its scratch is a fixed array in
the library shared by all calls, so the second call also checks that nothing
left behind by the first leaks into its results.  Collected last on purpose."""
import pytest
import torch

from tests.gpu_helpers import lib
from workloads import random_ids

pytestmark = pytest.mark.gpu
DEV = "cuda"

KEYS = ("counts", "offsets", "sorted_ids", "inv_perm", "tiles", "num_tiles")


def test_noalloc_matches_workspace_entry_twice():
    moe = lib()
    cases = [(8192, 256, 8, 16, 1.2),   # 128 chunks x 256 experts of built-in scratch
             (3000, 32, 4, 64, 0.5)]    # fewer experts: stale counters must not leak
    results = []
    for T, E, k, bm, skew in cases:
        ids = random_ids(T, E, k, seed=T, skew=skew).to(DEV)
        got = moe._lib.align_permute_noalloc(ids, E, bm)   # the two calls run back to back
        results.append((ids, E, bm, got))
    for ids, E, bm, got in results:
        ref = moe.align_permute(ids, E, bm)
        torch.cuda.synchronize()
        for key in KEYS:
            assert torch.equal(got[key], ref[key]), key


def test_noalloc_rejects_problems_beyond_its_scratch():
    moe = lib()
    # ceil(T*k/512) * E > 65536 counters: refused before any launch
    T, k, E = 70000, 8, 256
    ids = torch.zeros((1, 1), dtype=torch.int32, device=DEV)   # never read
    lib_ = moe.lib()
    cap = moe.permute_capacity(T, k, E, 16)
    buf = torch.empty(16, dtype=torch.int32, device=DEV)
    p = buf.data_ptr()
    rc = lib_.moe_align_permute_noalloc(ids.data_ptr(), T, k, E, 16, p, p, p, p, p, p, cap,
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == 3   # MOE_ERR_WORKSPACE
