"""ctypes binding of libmoe_b200.so (the C ABI of include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  There is no
CPU fallback: if the library is missing, importing this module's functions
raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_B200_DEBUG_CHECKS=1 selects the build whose kernels validate the
# permutation they are handed (see build.py --debug-checks)
DEBUG_CHECKS = os.environ.get("MOE_B200_DEBUG_CHECKS", "0") == "1"
LIB_PATH = os.path.join(_HERE, "libmoe_b200_debug.so" if DEBUG_CHECKS else "libmoe_b200.so")

BF16, FP8_E4M3 = 0, 1
COMBINE_AUTO, COMBINE_DETERMINISTIC, COMBINE_FUSED = 0, 1, 2
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
          3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT",
          6: "MOE_ERR_DEVICE"}

P = ctypes.c_void_p
I32 = ctypes.c_int
SZ = ctypes.c_size_t


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


class FfnArgs(ctypes.Structure):
    _fields_ = [("dtype", I32), ("T", I32), ("k", I32), ("E", I32), ("H", I32), ("I", I32),
                ("block_m", I32), ("capacity", I32), ("x", P), ("w", P), ("counts", P),
                ("offsets", P), ("sorted_ids", P), ("packed", P), ("scales", P),
                ("y_perm", P), ("status", P), ("max_ctas", I32)]


class LoraArgs(ctypes.Structure):
    _fields_ = [("n_adapters", I32), ("rank", I32), ("adapter", P), ("packed", P),
                ("scale", P)]


class ForwardArgs(ctypes.Structure):
    _fields_ = [("dtype", I32), ("T", I32), ("k", I32), ("E", I32), ("H", I32), ("I", I32),
                ("block_m", I32), ("x", P), ("logits", P), ("packed", P), ("scales", P),
                ("out", P), ("ids", P), ("w", P), ("status", P), ("max_ctas", I32),
                ("events", P), ("n_events", I32), ("combine", I32),
                ("lora", ctypes.POINTER(LoraArgs))]


class SplitCosts(ctypes.Structure):
    _fields_ = [("cpu_us", ctypes.c_double), ("cpu_us_per_token", ctypes.c_double),
                ("xfer_us", ctypes.c_double), ("gpu_us", ctypes.c_double),
                ("gpu_us_per_token", ctypes.c_double)]


class HostFfnArgs(ctypes.Structure):
    _fields_ = [("H", I32), ("I", I32), ("n", I32), ("weights", P), ("x", P), ("w", P),
                ("h", P), ("y", P), ("threads", I32), ("flags", I32)]


class SplitArgs(ctypes.Structure):
    _fields_ = [("T", I32), ("k", I32), ("E", I32), ("H", I32), ("I", I32), ("block_m", I32),
                ("x", P), ("logits", P), ("out", P), ("resident", P), ("resident_packed", P),
                ("stage_packed", P), ("n_stage", I32), ("host_packed", P), ("host_weights", P),
                ("costs", ctypes.POINTER(SplitCosts)), ("policy", I32), ("where", P),
                ("status", P), ("copy_stream", P), ("copy_event", P), ("host_threads", I32)]


_SIGS = {
    "moe_status_string": ([I32], ctypes.c_char_p),
    "moe_version": ([], ctypes.c_char_p),
    "moe_route_topk": ([P, I32, I32, I32, P, P, P], I32),
    "moe_permute_capacity": ([I32, I32, I32, I32], I32),
    "moe_align_permute_workspace_size": ([I32, I32, I32], SZ),
    "moe_align_permute": ([P, I32, I32, I32, I32, P, P, P, P, P, P, I32, P, SZ, P], I32),
    "moe_align_permute_noalloc": ([P, I32, I32, I32, I32, P, P, P, P, P, P, I32, P], I32),
    "moe_packed_weights_size": ([I32, I32, I32, I32], SZ),
    "moe_pack_weights": ([I32, I32, I32, I32, P, P, P, P, P, P], I32),
    "moe_packed_lora_size": ([I32, I32, I32, I32, I32], SZ),
    "moe_pack_lora": ([I32, I32, I32, I32, I32, P, P, P, P, P, P, P, P], I32),
    "moe_grouped_ffn_workspace_size": ([I32, I32, I32, I32, I32, I32, I32], SZ),
    "moe_grouped_ffn": ([ctypes.POINTER(FfnArgs), P, SZ, P], I32),
    "moe_combine": ([P, P, I32, I32, I32, P, P], I32),
    "moe_forward_workspace_size": ([I32, I32, I32, I32, I32, I32, I32], SZ),
    "moe_forward": ([ctypes.POINTER(ForwardArgs), P, SZ, P], I32),
    "moe_check_status": ([P, P], I32),
    "moe_selftest_wait_timeout": ([P, I32, P], I32),
    # CPU/GPU split (include/moe_split.h)
    "moe_split_place": ([P, I32, I32, P], I32),
    "moe_split_plan": ([P, P, I32, ctypes.POINTER(SplitCosts), I32, P], I32),
    "moe_split_plan_balanced": ([P, P, I32, ctypes.POINTER(SplitCosts), I32, P], I32),
    "moe_host_packed_size": ([I32, I32], SZ),
    "moe_host_pack_weights": ([I32, I32, I32, P, P, P, P], I32),
    "moe_host_isa": ([], I32),
    "moe_host_expert_ffn": ([ctypes.POINTER(HostFfnArgs)], I32),
    "moe_split_calibrate": ([I32, I32, I32, P, P, P, P, SZ, I32, P, ctypes.POINTER(SplitCosts)],
                            I32),
    "moe_split_workspace_size": ([I32, I32, I32, I32, I32, I32, I32, I32], SZ),
    "moe_split_host_workspace_size": ([I32, I32, I32, I32], SZ),
    "moe_split_forward": ([ctypes.POINTER(SplitArgs), P, SZ, P, SZ, P], I32),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mixture_experts_expert_route_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(code: int, where: str) -> None:
    if code != 0:
        raise MoEError(code, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def version() -> str:
    return lib().moe_version().decode()


def permute_capacity(T: int, k: int, E: int, block_m: int) -> int:
    return lib().moe_permute_capacity(T, k, E, block_m)


def route_topk(logits: torch.Tensor, k: int, ids=None, w=None, stream=None):
    T, E = logits.shape
    dev = logits.device
    ids = torch.empty((T, k), dtype=torch.int32, device=dev) if ids is None else ids
    w = torch.empty((T, k), dtype=torch.float32, device=dev) if w is None else w
    _check(lib().moe_route_topk(_ptr(logits), T, E, k, _ptr(ids), _ptr(w), _stream(stream)),
           "moe_route_topk")
    return ids, w


def align_permute(ids: torch.Tensor, E: int, block_m: int, capacity: int | None = None,
                  stream=None):
    T, k = ids.shape
    dev = ids.device
    cap = permute_capacity(T, k, E, block_m) if capacity is None else capacity
    out = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               sorted_ids=torch.empty(max(cap, 1), dtype=torch.int32, device=dev),
               inv_perm=torch.empty(max(T * k, 1), dtype=torch.int32, device=dev),
               tiles=torch.empty(max(cap // block_m, 1), dtype=torch.int32, device=dev),
               num_tiles=torch.empty(1, dtype=torch.int32, device=dev))
    nws = lib().moe_align_permute_workspace_size(T, k, E)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    _check(lib().moe_align_permute(_ptr(ids), T, k, E, block_m, _ptr(out["counts"]),
                                   _ptr(out["offsets"]), _ptr(out["sorted_ids"]),
                                   _ptr(out["inv_perm"]), _ptr(out["tiles"]),
                                   _ptr(out["num_tiles"]), cap, _ptr(ws), nws, _stream(stream)),
           "moe_align_permute")
    out["capacity"] = cap
    out["block_m"] = block_m
    return out


def align_permute_noalloc(ids: torch.Tensor, E: int, block_m: int, capacity: int | None = None,
                          stream=None):
    """align_permute without a workspace (the library's built-in scratch)."""
    T, k = ids.shape
    dev = ids.device
    cap = permute_capacity(T, k, E, block_m) if capacity is None else capacity
    out = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               sorted_ids=torch.empty(max(cap, 1), dtype=torch.int32, device=dev),
               inv_perm=torch.empty(max(T * k, 1), dtype=torch.int32, device=dev),
               tiles=torch.empty(max(cap // block_m, 1), dtype=torch.int32, device=dev),
               num_tiles=torch.empty(1, dtype=torch.int32, device=dev))
    _check(lib().moe_align_permute_noalloc(_ptr(ids), T, k, E, block_m, _ptr(out["counts"]),
                                           _ptr(out["offsets"]), _ptr(out["sorted_ids"]),
                                           _ptr(out["inv_perm"]), _ptr(out["tiles"]),
                                           _ptr(out["num_tiles"]), cap, _stream(stream)),
           "moe_align_permute_noalloc")
    out["capacity"] = cap
    out["block_m"] = block_m
    return out


def pack_weights(dtype: int, Wg: torch.Tensor, Wu: torch.Tensor, Wd: torch.Tensor, stream=None):
    """Packs bf16 master weights once.  Returns (packed uint8 tensor, scales or None)."""
    E, H, I = Wg.shape
    for W in (Wg, Wu, Wd):
        if W.dtype != torch.bfloat16 or not W.is_contiguous():
            raise ValueError("master weights must be contiguous bf16")
    n = lib().moe_packed_weights_size(dtype, E, H, I)
    packed = torch.empty(n, dtype=torch.uint8, device=Wg.device)
    scales = torch.empty((E, 3), dtype=torch.float32, device=Wg.device) \
        if dtype == FP8_E4M3 else None
    _check(lib().moe_pack_weights(dtype, E, H, I, _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(packed),
                                  _ptr(scales), _stream(stream)), "moe_pack_weights")
    return packed, scales


class Lora:
    """Packed multi-LoRA adapters on the device (see moe_pack_lora)."""

    def __init__(self, Ag, Bg, Au, Bu, Ad, Bd, scale, stream=None):
        n, E, H, r = Ag.shape
        I = Bg.shape[3]
        for M in (Ag, Bg, Au, Bu, Ad, Bd):
            if M.dtype != torch.bfloat16 or not M.is_contiguous() or not M.is_cuda:
                raise ValueError("adapter matrices must be contiguous bf16 CUDA tensors")
        self.n_adapters, self.rank, self.E, self.H, self.I = n, r, E, H, I
        size = lib().moe_packed_lora_size(E, H, I, n, r)
        if size == 0:
            raise MoEError(2, "moe_packed_lora_size")
        self.packed = torch.empty(size, dtype=torch.uint8, device=Ag.device)
        _check(lib().moe_pack_lora(E, H, I, n, r, _ptr(Ag), _ptr(Bg), _ptr(Au), _ptr(Bu),
                                   _ptr(Ad), _ptr(Bd), _ptr(self.packed), _stream(stream)),
               "moe_pack_lora")
        self.scale = scale.to(device=Ag.device, dtype=torch.float32).contiguous()

    def args(self, adapter):
        """The C struct for tokens whose adapters are `adapter` (device int32 [T])."""
        if adapter.dtype != torch.int32 or not adapter.is_cuda:
            raise ValueError("adapter must be a CUDA int32 tensor")
        return LoraArgs(self.n_adapters, self.rank, _ptr(adapter), _ptr(self.packed),
                        _ptr(self.scale))


def grouped_ffn_workspace_size(dtype, T, k, E, H, I, block_m) -> int:
    return lib().moe_grouped_ffn_workspace_size(dtype, T, k, E, H, I, block_m)


def grouped_ffn(dtype: int, x: torch.Tensor, w: torch.Tensor, perm: dict, packed, scales,
                E: int, I: int, k: int, y_perm=None, status=None, ws=None, max_ctas: int = 0,
                stream=None):
    T, H = x.shape
    bm, cap = perm["block_m"], perm["capacity"]
    y_perm = torch.empty((max(cap, 1), H), dtype=torch.bfloat16, device=x.device) \
        if y_perm is None else y_perm
    n = grouped_ffn_workspace_size(dtype, T, k, E, H, I, bm)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device=x.device) if ws is None else ws
    a = FfnArgs(dtype, T, k, E, H, I, bm, cap, _ptr(x), _ptr(w), _ptr(perm["counts"]),
                _ptr(perm["offsets"]), _ptr(perm["sorted_ids"]), _ptr(packed), _ptr(scales),
                _ptr(y_perm), _ptr(status), max_ctas)
    _check(lib().moe_grouped_ffn(ctypes.byref(a), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_grouped_ffn")
    return y_perm, ws


def combine(y_perm, inv_perm, T: int, k: int, H: int, out=None, stream=None):
    out = torch.empty((T, H), dtype=torch.bfloat16, device=y_perm.device) if out is None else out
    _check(lib().moe_combine(_ptr(y_perm), _ptr(inv_perm), T, k, H, _ptr(out), _stream(stream)),
           "moe_combine")
    return out


def forward_workspace_size(dtype, T, k, E, H, I, block_m=0) -> int:
    return lib().moe_forward_workspace_size(dtype, T, k, E, H, I, block_m)


def forward(dtype: int, x, logits, packed, scales, E: int, I: int, k: int, out=None, ids=None,
            w=None, status=None, ws=None, block_m: int = 0, max_ctas: int = 0, events=None,
            combine: int = COMBINE_AUTO, lora=None, adapter=None, stream=None):
    """The whole layer.  ``events`` (7 torch.cuda.Event, optional) are recorded after
    each stage: entry, route+permute, FP8 x quantisation, gate/up, h quant, down,
    combine.  ``combine``: COMBINE_AUTO, COMBINE_DETERMINISTIC or COMBINE_FUSED.
    ``lora`` (a Lora) with ``adapter`` (CUDA int32 [T], -1 = none) applies
    multi-LoRA adapters (bf16 layers)."""
    T, H = x.shape
    out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device) if out is None else out
    n = forward_workspace_size(dtype, T, k, E, H, I, block_m)
    if ws is None:
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device=x.device)
    ev_arr = None
    if events is not None:
        if len(events) != 7:
            raise ValueError("events must hold 7 torch.cuda.Event")
        for e in events:
            if e.cuda_event == 0:  # create lazily-initialised events
                e.record()
        ev_arr = (ctypes.c_void_p * 7)(*[e.cuda_event for e in events])
    largs = lora.args(adapter) if lora is not None else None
    a = ForwardArgs(dtype, T, k, E, H, I, block_m, _ptr(x), _ptr(logits), _ptr(packed),
                    _ptr(scales), _ptr(out), _ptr(ids), _ptr(w), _ptr(status), max_ctas,
                    ctypes.cast(ev_arr, ctypes.c_void_p) if ev_arr is not None else None,
                    7 if ev_arr is not None else 0, combine,
                    ctypes.pointer(largs) if largs is not None else None)
    _check(lib().moe_forward(ctypes.byref(a), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_forward")
    return out


def check_status(status: torch.Tensor, stream=None) -> int:
    return lib().moe_check_status(_ptr(status), _stream(stream))


def selftest_wait_timeout(status: torch.Tensor, timeout_us: int, stream=None) -> None:
    _check(lib().moe_selftest_wait_timeout(_ptr(status), timeout_us, _stream(stream)),
           "moe_selftest_wait_timeout")


class MoELayer:
    """A fused MoE layer with packed weights and a reusable workspace.

    >>> layer = MoELayer(Wg, Wu, Wd, k=2, dtype=BF16)   # bf16 [E,H,I], [E,I,H] on cuda
    >>> out = layer(x, logits)                            # x bf16 [T,H], logits f32 [T,E]
    """

    def __init__(self, Wg, Wu, Wd, k: int, dtype: int = BF16, block_m: int = 0,
                 max_ctas: int = 0, combine: int = COMBINE_AUTO):
        self.E, self.H, self.I = Wg.shape
        self.k, self.dtype, self.block_m, self.max_ctas = k, dtype, block_m, max_ctas
        self.combine = combine
        self.packed, self.scales = pack_weights(dtype, Wg, Wu, Wd)
        self.device = Wg.device
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self._ws = {}

    def workspace(self, T: int) -> torch.Tensor:
        if T not in self._ws:
            n = forward_workspace_size(self.dtype, T, self.k, self.E, self.H, self.I,
                                       self.block_m)
            self._ws[T] = torch.empty(max(n, 16), dtype=torch.uint8, device=self.device)
        return self._ws[T]

    def __call__(self, x, logits, out=None, events=None, stream=None):
        T = x.shape[0]
        return forward(self.dtype, x, logits, self.packed, self.scales, self.E, self.I,
                       self.k, out=out, status=self.status, ws=self.workspace(T),
                       block_m=self.block_m, max_ctas=self.max_ctas, events=events,
                       combine=self.combine, stream=stream)

    def check(self) -> int:
        return check_status(self.status)


# ---- CPU/GPU expert split (include/moe_split.h) ----------------------------

SPLIT_IDLE, SPLIT_RESIDENT, SPLIT_STAGED, SPLIT_CPU = 0, 1, 2, 3
POLICY_DYNAMIC, POLICY_ALL_CPU, POLICY_ALL_STAGED, POLICY_BALANCED = 0, 1, 2, 3
HOST_ISA_PORTABLE, HOST_ISA_AVX512_BF16, HOST_ISA_AMX_BF16 = 0, 1, 2
HOST_PATHS = {"auto": 0, "portable": 1, "avx512_bf16": 2}   # moe_host_ffn_args.flags


def _hptr(t):
    """Address of a host (CPU) tensor or numpy array."""
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if t.is_cuda:
            raise ValueError("expected a host tensor")
        return t.data_ptr()
    return t.ctypes.data


def _i32(a):
    import numpy as np
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def split_place(hits, budget: int):
    """resident int32 [E]: 1 for the `budget` experts with the most hits."""
    import numpy as np
    h = np.ascontiguousarray(np.asarray(hits, dtype=np.int64))
    resident = np.zeros(len(h), np.int32)
    _check(lib().moe_split_place(_hptr(h), len(h), budget, _hptr(resident)), "moe_split_place")
    return resident


def split_costs(cpu_us=0.0, cpu_us_per_token=0.0, xfer_us=0.0, gpu_us=0.0,
                gpu_us_per_token=0.0) -> SplitCosts:
    return SplitCosts(cpu_us, cpu_us_per_token, xfer_us, gpu_us, gpu_us_per_token)


def split_plan(counts, resident, costs: SplitCosts, n_stage: int, balanced: bool = False):
    """where int32 [E] (SPLIT_IDLE / RESIDENT / STAGED / CPU) for one batch:
    the per-expert rule, or with ``balanced`` the host/link balanced plan."""
    import numpy as np
    c, r = _i32(counts), _i32(resident)
    where = np.zeros(len(c), np.int32)
    fn = lib().moe_split_plan_balanced if balanced else lib().moe_split_plan
    _check(fn(_hptr(c), _hptr(r), len(c), ctypes.byref(costs), n_stage, _hptr(where)),
           "moe_split_plan")
    return where


def host_isa() -> int:
    return lib().moe_host_isa()


def host_packed_size(H: int, I: int) -> int:
    return lib().moe_host_packed_size(H, I)


def host_pack_weights(Wg, Wu, Wd):
    """Host layout of bf16 master weights (CPU tensors) -> uint8 CPU tensor [E, bytes]."""
    E, H, I = Wg.shape
    for W in (Wg, Wu, Wd):
        if W.dtype != torch.bfloat16 or W.is_cuda or not W.is_contiguous():
            raise ValueError("host master weights must be contiguous bf16 CPU tensors")
    out = torch.empty((E, host_packed_size(H, I)), dtype=torch.uint8)
    _check(lib().moe_host_pack_weights(E, H, I, _hptr(Wg), _hptr(Wu), _hptr(Wd), _hptr(out)),
           "moe_host_pack_weights")
    return out


def host_expert_ffn(weights, x, w, threads: int = 0, path: str = "auto"):
    """One expert on the host: (h bf16 [n,I], y bf16 [n,H]).  weights: one row of
    host_pack_weights' output; x bf16 [n,H]; w f32 [n] (CPU tensors).  path:
    "auto" (the fastest this CPU has), "avx512_bf16" (no AMX) or "portable"."""
    n, H = x.shape
    I = weights.numel() // (3 * H * 2)
    x = x.contiguous()
    w = w.to(torch.float32).contiguous()
    h = torch.empty((n, I), dtype=torch.bfloat16)
    y = torch.empty((n, H), dtype=torch.bfloat16)
    a = HostFfnArgs(H, I, n, _hptr(weights), _hptr(x), _hptr(w), _hptr(h), _hptr(y), threads,
                    HOST_PATHS[path])
    _check(lib().moe_host_expert_ffn(ctypes.byref(a)), "moe_host_expert_ffn")
    return h, y


class SplitLayer:
    """The CPU/GPU split layer (moe_split_forward): `resident` experts' weights
    live on the GPU, the rest in host memory; each batch runs every other
    expert it routes to either on the host or after copying its weights to
    one of `n_stage` staging slots, as `policy` and `costs` decide.

    Wg, Wu [E,H,I], Wd [E,I,H]: bf16 master weights on the host."""

    def __init__(self, Wg, Wu, Wd, k: int, resident, n_stage: int = 2,
                 policy: int = POLICY_DYNAMIC, costs: SplitCosts | None = None,
                 host_threads: int = 0, block_m: int = 0, device="cuda"):
        self.E, self.H, self.I = Wg.shape
        self.k, self.n_stage, self.policy = k, n_stage, policy
        self.host_threads, self.block_m = host_threads, block_m
        self.device = torch.device(device)
        self.resident = _i32(resident)
        self.S = int(self.resident.sum())
        E, H, I = self.E, self.H, self.I
        self.host_weights = host_pack_weights(Wg, Wu, Wd)
        # the GPU layout of each expert, made on the device one expert at a
        # time and kept in page-locked host memory as the source of the
        # staging copies (the GPU never holds more than one expert's copy)
        per = lib().moe_packed_weights_size(BF16, 1, H, I)
        self.host_packed = torch.empty((E, per), dtype=torch.uint8, pin_memory=True)
        for e in range(E):
            pk, _ = pack_weights(BF16, Wg[e:e + 1].to(self.device), Wu[e:e + 1].to(self.device),
                                 Wd[e:e + 1].to(self.device))
            self.host_packed[e].copy_(pk)
        del pk
        idx = [e for e in range(E) if self.resident[e]]
        self.resident_packed = None
        if idx:
            self.resident_packed, _ = pack_weights(BF16, Wg[idx].to(self.device),
                                                   Wu[idx].to(self.device),
                                                   Wd[idx].to(self.device))
        self.stage_packed = torch.empty(
            max(lib().moe_packed_weights_size(BF16, max(n_stage, 1), H, I), 16),
            dtype=torch.uint8, device=self.device)
        self.copy_stream = torch.cuda.Stream(device=self.device)
        self.copy_event = torch.cuda.Event()
        self.copy_event.record(self.copy_stream)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.where = _i32([0] * E)
        self._ws, self._hws = {}, {}
        self.costs = costs if costs is not None else self.calibrate()

    def calibrate(self, n_max: int = 128) -> SplitCosts:
        """The latency model measured here: the host kernel on 1 and n_max
        tokens (a line through both: flat while the host streams weights,
        steeper once its tile products bound it, so n_max sits where a copy
        starts to compete) and one expert's copy to the GPU."""
        c = SplitCosts()
        hws = torch.empty(lib().moe_split_host_workspace_size(n_max, 1, self.H, self.I),
                          dtype=torch.uint8, pin_memory=True)
        dst = self.stage_packed if self.n_stage > 0 else torch.empty(
            3 * self.H * self.I * 2, dtype=torch.uint8, device=self.device)
        _check(lib().moe_split_calibrate(self.H, self.I, n_max, _hptr(self.host_weights[0]),
                                         _hptr(self.host_packed), _ptr(dst), _hptr(hws),
                                         hws.numel(), self.host_threads, _stream(None),
                                         ctypes.byref(c)), "moe_split_calibrate")
        return c

    def workspaces(self, T: int):
        if T not in self._ws:
            n = lib().moe_split_workspace_size(T, self.k, self.E, self.S, self.n_stage, self.H,
                                               self.I, self.block_m)
            if n == 0:
                raise MoEError(1, "moe_split_workspace_size")
            self._ws[T] = torch.empty(n, dtype=torch.uint8, device=self.device)
            m = lib().moe_split_host_workspace_size(T, self.k, self.H, self.I)
            self._hws[T] = torch.empty(max(m, 16), dtype=torch.uint8, pin_memory=True)
        return self._ws[T], self._hws[T]

    def __call__(self, x, logits, out=None, stream=None, policy: int | None = None):
        T = x.shape[0]
        out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device) \
            if out is None else out
        ws, hws = self.workspaces(T)
        a = SplitArgs(T, self.k, self.E, self.H, self.I, self.block_m, _ptr(x), _ptr(logits),
                      _ptr(out), _hptr(self.resident), _ptr(self.resident_packed),
                      _ptr(self.stage_packed) if self.n_stage > 0 else None, self.n_stage,
                      _hptr(self.host_packed), _hptr(self.host_weights),
                      ctypes.pointer(self.costs), self.policy if policy is None else policy,
                      _hptr(self.where), _ptr(self.status), self.copy_stream.cuda_stream,
                      self.copy_event.cuda_event, self.host_threads)
        _check(lib().moe_split_forward(ctypes.byref(a), _ptr(ws), ws.numel(), _hptr(hws),
                                       hws.numel(), _stream(stream)), "moe_split_forward")
        return out

    def check(self) -> int:
        return check_status(self.status)
