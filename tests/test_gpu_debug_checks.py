"""The MOE_DEBUG_CHECKS build (libmoe_b200_debug.so): a permutation with a flat
index past T*k, or an expert block past the capacity, is reported as
MOE_ERR_DEVICE in the status word and skipped -- no trap, the context stays
usable.  Runs in a child process that selects the debug library.

The corrupt entries are chosen so that even an unchecked access would stay
inside allocated memory (x and w are allocated with spare rows): a missing
check shows up as a failed assertion, not as a fault."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, torch
sys.path.insert(0, ROOT)
from tests.gpu_helpers import lib
moe = lib()
assert moe._lib.DEBUG_CHECKS and moe.LIB_PATH.endswith("libmoe_b200_debug.so")
from workloads import make_layer
DEV = "cuda"
T, E, k, H, I = 24, 4, 2, 256, 256
L = make_layer("tiny", T=T, E=E, k=k, H=H, I=I, seed=1)
Wg, Wu, Wd = (W.to(DEV) for W in L.weights_bf16())
packed, scales = moe.pack_weights(0, Wg, Wu, Wd)
x_big = torch.zeros((T + 8, H), dtype=torch.bfloat16, device=DEV)
x_big[:T] = L.x.to(DEV)
ids, w = moe.route_topk(L.logits.to(DEV), k)
w_big = torch.zeros(T * k + 64, dtype=torch.float32, device=DEV)
w_big[:T * k] = w.view(-1)
perm = moe.align_permute(ids, E, 16)
torch.cuda.synchronize()
# 1) clean call: status 0
st = torch.zeros(1, dtype=torch.int32, device=DEV)
moe.grouped_ffn(0, x_big[:T], w_big, perm, packed, scales, E, I, k, status=st)
assert moe.check_status(st) == 0, "clean permutation reported a fault"
# 2) a flat index T*k + 1 (token T: a spare row of x_big, never a fault)
bad = dict(perm)
bad["sorted_ids"] = perm["sorted_ids"].clone()
bad["sorted_ids"][0] = T * k + 1
st.zero_()
moe.grouped_ffn(0, x_big[:T], w_big, bad, packed, scales, E, I, k, status=st)
assert moe.check_status(st) == 6, "flat index past T*k not reported"
# 3) counts that push an expert's block past the capacity (the GEMM skips it)
bad = dict(perm)
bad["counts"] = perm["counts"].clone()
bad["counts"][E - 1] = perm["capacity"]
st.zero_()
moe.grouped_ffn(0, x_big[:T], w_big, bad, packed, scales, E, I, k, status=st)
assert moe.check_status(st) == 6, "expert block past the capacity not reported"
# the context is still usable
assert torch.ones(4, device=DEV).sum().item() == 4
print("debug checks ok")
'''


def test_debug_build_reports_bad_permutation():
    env = dict(os.environ, MOE_B200_DEBUG_CHECKS="1")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug checks ok" in r.stdout
