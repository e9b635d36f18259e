"""CPU oracle of the fused MoE layer -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The library never does: it has no CPU fallback.

The arithmetic lives in ``moe_oracle.c`` (plain loops, double precision); this
file only builds it with gcc and marshals numpy/torch arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compiles the oracle (gcc, -O2, OpenMP, no fp contraction, no fast-math)."""
    with _lock:
        if force or not os.path.exists(_LIB_PATH) or \
                os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
            tmp = _LIB_PATH + f".{os.getpid()}.tmp"
            subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC",
                                   "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"])
            os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32 = ctypes.c_int
        L.oracle_route_topk.argtypes = [P, i32, i32, i32, P, P]
        L.oracle_permute_capacity.argtypes = [i32, i32, i32, i32]
        L.oracle_align_permute.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P, P, P]
        L.oracle_moe_layer.argtypes = [i32, i32, i32, i32, i32, P, i32, P, P, P, P, P, i32,
                                       P, i32, P]
        L.oracle_moe_layer_fp8.argtypes = [i32, i32, i32, i32, i32, P, i32, P, P, P, P, P, i32,
                                           P, i32, P, P, P]
        L.oracle_moe_layer_lora.argtypes = [i32, i32, i32, i32, i32, P, i32, P, P, P, P, P, i32,
                                            i32, i32, P, P, P, P, P, P, P, i32, P, P, i32, P]
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_float
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_fp8_quantize.argtypes = [P, i32, ctypes.c_size_t, P]
        L.oracle_fp8_quantize.restype = ctypes.c_float
        L.oracle_set_num_threads.argtypes = [i32]
        _lib = L
    return _lib


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def _arr(a, dtype=None):
    """numpy view of a CPU tensor/array; bf16 tensors become uint16 bit patterns."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                return np.ascontiguousarray(a.view(torch.int16).numpy().view(np.uint16)), BF16
            a = a.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a if dtype is None else np.asarray(a, dtype=dtype))
    if a.dtype == np.uint16:
        return a, BF16
    return a, F32


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def route_topk(logits, k: int):
    lg, _ = _arr(logits, np.float32)
    lg = lg.astype(np.float32, copy=False)
    T, E = lg.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    rc = lib().oracle_route_topk(_p(lg), T, E, k, _p(ids), _p(w))
    if rc != 0:
        raise ValueError(f"oracle_route_topk: {rc}")
    return ids, w


def permute_capacity(T: int, k: int, E: int, block_m: int) -> int:
    return lib().oracle_permute_capacity(T, k, E, block_m)


def align_permute(ids, E: int, block_m: int, capacity: int | None = None):
    ids = np.ascontiguousarray(np.asarray(ids, np.int32))
    T, k = ids.shape
    cap = permute_capacity(T, k, E, block_m) if capacity is None else capacity
    out = dict(counts=np.zeros(E, np.int32), offsets=np.zeros(E + 1, np.int32),
               sorted_ids=np.zeros(cap, np.int32), inv_perm=np.zeros(T * k, np.int32),
               tiles=np.zeros(max(cap // block_m, 1), np.int32),
               num_tiles=np.zeros(1, np.int32))
    rc = lib().oracle_align_permute(_p(ids), T, k, E, block_m, cap, _p(out["counts"]),
                                    _p(out["offsets"]), _p(out["sorted_ids"]),
                                    _p(out["inv_perm"]), _p(out["tiles"]),
                                    _p(out["num_tiles"]))
    if rc != 0:
        raise ValueError(f"oracle_align_permute: {rc}")
    out["tiles"] = out["tiles"][: cap // block_m]
    out["num_tiles"] = int(out["num_tiles"][0])
    out["capacity"] = cap
    return out


def _layer_args(x, ids, w, Wg, Wu, Wd, tokens):
    xa, xdt = _arr(x)
    if xdt == F32:
        xa = xa.astype(np.float32, copy=False)
    ga, gdt = _arr(Wg)
    ua, udt = _arr(Wu)
    da, ddt = _arr(Wd)
    if not (gdt == udt == ddt):
        raise TypeError("W_g, W_u, W_d must share a dtype")
    if gdt == F32:
        ga, ua, da = (a.astype(np.float32, copy=False) for a in (ga, ua, da))
    ids = np.ascontiguousarray(np.asarray(ids, np.int32))
    w = np.ascontiguousarray(np.asarray(w, np.float64))
    T, H = xa.shape
    E, H2, I = ga.shape
    assert H2 == H and da.shape == (E, I, H) and ua.shape == ga.shape
    k = ids.shape[1]
    if tokens is None:
        tok = None
        n = T
    else:
        tok = np.ascontiguousarray(np.asarray(tokens, np.int32))
        n = len(tok)
    return xa, xdt, ga, ua, da, gdt, ids, w, T, H, I, E, k, tok, n


def moe_layer(x, ids, w, Wg, Wu, Wd, tokens=None):
    """out [n, H] float64 for the listed tokens (all tokens if None)."""
    xa, xdt, ga, ua, da, gdt, ids, w, T, H, I, E, k, tok, n = _layer_args(x, ids, w, Wg, Wu, Wd,
                                                                          tokens)
    out = np.zeros((n, H), np.float64)
    rc = lib().oracle_moe_layer(T, H, I, E, k, _p(xa), xdt, _p(ids), _p(w), _p(ga), _p(ua),
                                _p(da), gdt, None if tok is None else _p(tok), n, _p(out))
    if rc != 0:
        raise ValueError(f"oracle_moe_layer: {rc}")
    return out


def moe_layer_fp8(x, ids, w, Wg, Wu, Wd, tokens=None):
    """FP8 e4m3 layer.  Returns (out [n,H] f64, w_scales [E,3] f32, (s_x, s_h))."""
    xa, xdt, ga, ua, da, gdt, ids, w, T, H, I, E, k, tok, n = _layer_args(x, ids, w, Wg, Wu, Wd,
                                                                          tokens)
    out = np.zeros((n, H), np.float64)
    ws = np.zeros((E, 3), np.float32)
    acts = np.zeros(2, np.float32)
    rc = lib().oracle_moe_layer_fp8(T, H, I, E, k, _p(xa), xdt, _p(ids), _p(w), _p(ga), _p(ua),
                                    _p(da), gdt, None if tok is None else _p(tok), n, _p(out),
                                    _p(ws), _p(acts))
    if rc != 0:
        raise ValueError(f"oracle_moe_layer_fp8: {rc}")
    return out, ws, (float(acts[0]), float(acts[1]))


def moe_layer_lora(x, ids, w, Wg, Wu, Wd, adapter, lora, scale, tokens=None):
    """Multi-LoRA layer.  adapter: int [T] (-1 = base model); lora: dict of
    Ag, Au [n_a,E,H,r], Bg, Bu [n_a,E,r,I], Ad [n_a,E,I,r], Bd [n_a,E,r,H]
    (one dtype); scale: [n_a].  Returns out [n,H] float64."""
    xa, xdt, ga, ua, da, gdt, ids, w, T, H, I, E, k, tok, n = _layer_args(x, ids, w, Wg, Wu, Wd,
                                                                          tokens)
    mats = [_arr(lora[key]) for key in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")]
    ldt = mats[0][1]
    if any(m[1] != ldt for m in mats):
        raise TypeError("adapter matrices must share a dtype")
    mats = [m[0] if ldt == BF16 else m[0].astype(np.float32, copy=False) for m in mats]
    n_a, E2, H2, r = mats[0].shape
    assert E2 == E and H2 == H
    assert mats[1].shape == (n_a, E, r, I) and mats[4].shape == (n_a, E, I, r)
    assert mats[5].shape == (n_a, E, r, H)
    ad = np.ascontiguousarray(np.asarray(adapter, np.int32))
    assert ad.shape == (T,)
    sc = np.ascontiguousarray(np.asarray(scale, np.float64))
    assert sc.shape == (n_a,)
    out = np.zeros((n, H), np.float64)
    rc = lib().oracle_moe_layer_lora(T, H, I, E, k, _p(xa), xdt, _p(ids), _p(w), _p(ga), _p(ua),
                                     _p(da), gdt, n_a, r, _p(ad), *[_p(m) for m in mats], ldt,
                                     _p(sc), None if tok is None else _p(tok), n, _p(out))
    if rc != 0:
        raise ValueError(f"oracle_moe_layer_lora: {rc}")
    return out


def e4m3_decode(codes) -> np.ndarray:
    c = np.asarray(codes, np.uint8).ravel()
    L = lib()
    return np.array([L.oracle_e4m3_decode(int(v)) for v in c], np.float32).reshape(
        np.shape(codes))


def e4m3_encode(values) -> np.ndarray:
    v = np.asarray(values, np.float32).ravel()
    L = lib()
    return np.array([L.oracle_e4m3_encode(float(f)) for f in v], np.uint8).reshape(
        np.shape(values))


def fp8_quantize(t):
    """(scale, codes) of one tensor: s = amax/448, codes = RNE_sat(t / s)."""
    a, dt = _arr(t)
    if dt == F32:
        a = a.astype(np.float32, copy=False)
    q = np.zeros(a.shape, np.uint8)
    s = lib().oracle_fp8_quantize(_p(a), dt, a.size, _p(q))
    return float(s), q
