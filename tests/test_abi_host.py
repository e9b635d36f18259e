"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/*.h declares, and rejects bad arguments
synchronously (nothing is launched, so no device is touched)."""
import ctypes
import os
import re

import pytest
import torch

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from mixture_experts_expert_route_b200 import _lib, build
    build.build(debug=_lib.DEBUG_CHECKS)
    import mixture_experts_expert_route_b200 as moe
    return moe


def declared_functions():
    src = ""
    inc = os.path.join(ROOT, "include")
    for name in sorted(os.listdir(inc)):
        if name.endswith(".h"):
            with open(os.path.join(inc, name)) as f:
                src += f.read()
    return sorted(set(re.findall(r"MOE_API [^;(]*?\b(moe_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 24
    lib = ctypes.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    # the binding wires the same names
    from mixture_experts_expert_route_b200._lib import _SIGS
    assert sorted(_SIGS) == names


def test_status_strings(L):
    for code, name in L._lib.STATUS.items():
        assert L.status_string(code) == name
    assert L.status_string(99) == "MOE_ERR_UNKNOWN"
    assert "sm_100a" in L.version()


@pytest.mark.parametrize("T,k,E,bm", [(0, 2, 8, 16), (1, 2, 8, 16), (64, 2, 8, 16), (17, 8, 128, 64),
                                      (8192, 8, 256, 16), (4096, 8, 128, 128), (3, 3, 3, 1)])
def test_capacity_matches_oracle(L, T, k, E, bm):
    assert L.permute_capacity(T, k, E, bm) == oracle.permute_capacity(T, k, E, bm)


def test_workspace_sizes(L):
    lib = L.lib()
    assert lib.moe_align_permute_workspace_size(64, 2, 8) == 0       # single chunk
    assert lib.moe_align_permute_workspace_size(4096, 8, 128) == 64 * 128 * 4   # 512 per chunk
    assert lib.moe_align_permute_workspace_size(256, 8, 128) == 0                # one CTA up to 2048
    # 16 KB tiles of 128 rows x 128 bytes, padded per expert matrix
    assert lib.moe_packed_weights_size(0, 8, 4096, 14336) == 3 * 8 * 4096 * 14336 * 2
    tiles = 32 * ((2 * 2880 // 128) * 23 + 23 * 23)
    assert lib.moe_packed_weights_size(1, 32, 2880, 2880) == tiles * 16384
    a = lib.moe_forward_workspace_size(0, 64, 2, 8, 4096, 14336, 0)
    b = lib.moe_forward_workspace_size(0, 64, 2, 8, 4096, 14336, 16)
    assert a == b > 0
    assert lib.moe_forward_workspace_size(1, 64, 2, 8, 4096, 14336, 16) > 0
    # unsupported shapes report size 0
    assert lib.moe_forward_workspace_size(0, 64, 2, 8, 4000, 14336, 16) == 0
    assert lib.moe_grouped_ffn_workspace_size(0, 64, 2, 8, 4096, 14336, 8) == 0


def test_argument_errors_return_synchronously(L):
    lib = L.lib()
    INVALID, UNSUP, WS = 1, 2, 3
    fake = ctypes.c_void_p(0x1000)
    assert lib.moe_route_topk(fake, 4, 8, 9, fake, fake, None) == INVALID      # k > E
    assert lib.moe_route_topk(fake, 4, 8, 0, fake, fake, None) == INVALID      # k < 1
    assert lib.moe_route_topk(fake, -1, 8, 2, fake, fake, None) == INVALID
    assert lib.moe_route_topk(fake, 4, 300, 2, fake, fake, None) == UNSUP      # E > 256
    assert lib.moe_route_topk(None, 4, 8, 2, fake, fake, None) == INVALID
    assert lib.moe_route_topk(None, 0, 8, 2, None, None, None) == 0            # T = 0 no-op
    cap = lib.moe_permute_capacity(64, 2, 8, 16)
    assert lib.moe_align_permute(fake, 64, 2, 8, 16, fake, fake, fake, fake, fake, fake,
                                 cap - 1, None, 0, None) == WS
    assert lib.moe_align_permute(fake, 8192, 8, 256, 16, fake, fake, fake, fake, fake, fake,
                                 lib.moe_permute_capacity(8192, 8, 256, 16), None, 0, None) == WS
    assert lib.moe_pack_weights(0, 8, 4000, 512, fake, fake, fake, fake, None, None) == UNSUP
    assert lib.moe_pack_weights(1, 8, 256, 512, fake, fake, fake, fake, None, None) == INVALID
    assert lib.moe_pack_weights(0, 8, 256, 512, ctypes.c_void_p(0x1001), fake, fake, fake,
                                None, None) == INVALID                            # misaligned
    assert lib.moe_combine(fake, fake, 4, 2, 100, fake, None) == INVALID          # H % 8
    assert lib.moe_check_status(None, None) == INVALID
    assert lib.moe_selftest_wait_timeout(fake, 0, None) == INVALID
    assert lib.moe_selftest_wait_timeout(fake, 2000000, None) == INVALID


def _fwd(L, **kw):
    base = dict(dtype=0, T=4, k=2, E=8, H=256, I=512, block_m=16, x=0x1000, logits=0x1000,
                packed=0x1000, scales=None, out=0x1000, ids=None, w=None, status=None,
                max_ctas=0, events=None, n_events=0, combine=0, lora=None)
    base.update(kw)
    a = L._lib.ForwardArgs(*[base[f] for f, _ in L._lib.ForwardArgs._fields_])
    return a


def test_forward_argument_errors(L):
    lib = L.lib()
    INVALID, UNSUP, WS = 1, 2, 3
    ws = ctypes.c_void_p(0x1000)
    big = 1 << 40
    call = lambda a, n=big: lib.moe_forward(ctypes.byref(a), ws, n, None)
    assert call(_fwd(L, k=9)) == INVALID
    assert call(_fwd(L, H=200)) == INVALID or call(_fwd(L, H=200)) == UNSUP
    assert call(_fwd(L, H=320 - 32)) == UNSUP                 # not a multiple of 64
    assert call(_fwd(L, block_m=8)) == INVALID
    assert call(_fwd(L, block_m=24)) == UNSUP
    assert call(_fwd(L, dtype=7)) == INVALID
    assert call(_fwd(L, dtype=1)) == INVALID                  # FP8 needs scales
    assert call(_fwd(L, x=0x1004)) == INVALID                 # misaligned
    assert call(_fwd(L, logits=None)) == INVALID
    assert call(_fwd(L, max_ctas=-1)) == INVALID
    assert call(_fwd(L, events=0x1000, n_events=3)) == INVALID
    assert call(_fwd(L, combine=3)) == INVALID                # unknown combine mode
    assert call(_fwd(L, combine=-1)) == INVALID
    # adapters: bf16 only, n * r <= 64, pointers required
    la = L._lib.LoraArgs(4, 16, 0x1000, 0x1000, 0x1000)
    assert call(_fwd(L, lora=ctypes.pointer(la), dtype=1, scales=0x1000)) == UNSUP
    assert call(_fwd(L, lora=ctypes.pointer(L._lib.LoraArgs(5, 16, 0x1000, 0x1000, 0x1000)))) == UNSUP
    assert call(_fwd(L, lora=ctypes.pointer(L._lib.LoraArgs(0, 16, 0x1000, 0x1000, 0x1000)))) == INVALID
    assert call(_fwd(L, lora=ctypes.pointer(L._lib.LoraArgs(4, 16, None, 0x1000, 0x1000)))) == INVALID
    assert lib.moe_packed_lora_size(8, 256, 512, 4, 16) > 0
    assert lib.moe_packed_lora_size(8, 256, 512, 4, 17) == 0
    assert call(_fwd(L), 64) == WS                            # workspace too small
    assert call(_fwd(L, T=0, x=None, logits=None)) == 0       # T = 0 no-op
    assert lib.moe_forward(None, ws, big, None) == INVALID


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No silent fallback: without the built library the binding raises."""
    import mixture_experts_expert_route_b200._lib as binding
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(ImportError):
        binding.lib()
    # and a CUDA tensor argument is required: host tensors are refused, not copied
    with pytest.raises(ValueError):
        binding._ptr(torch.zeros(1))
