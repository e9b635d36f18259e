"""Two devices driven from one process: the GEMM kernels' shared-memory opt-in
is per device, so a layer on the second GPU must run as on the first.  Skipped
where fewer than two GPUs are visible."""
import pytest
import torch

from tests.gpu_helpers import assert_close, check_routing, lib, oracle_layer
from workloads import make_layer

pytestmark = pytest.mark.gpu


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs two visible GPUs")
@pytest.mark.parametrize("dtype", [0, 1])
def test_forward_on_two_devices(dtype):
    moe = lib()
    L = make_layer("tiny", T=40, E=8, k=2, H=256, I=256, seed=11)
    g, u, d = L.weights_bf16()
    outs = []
    for dev in ("cuda:0", "cuda:1"):
        with torch.cuda.device(dev):
            packed, scales = moe.pack_weights(dtype, g.to(dev), u.to(dev), d.to(dev))
            ids = torch.empty((L.T, L.k), dtype=torch.int32, device=dev)
            w = torch.empty((L.T, L.k), dtype=torch.float32, device=dev)
            out = moe.forward(dtype, L.x.to(dev), L.logits.to(dev), packed, scales, L.E, L.I,
                              L.k, ids=ids, w=w)
            torch.cuda.synchronize(dev)
            ids_o, w_o = check_routing(ids, w, L.logits)
            assert_close(out, oracle_layer(dtype, L.x, ids_o, w_o, g, u, d), dtype, dev)
            outs.append(out.cpu())
    # the same kernels on the same inputs: the same result on both devices
    assert torch.equal(outs[0], outs[1])
