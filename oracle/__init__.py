"""CPU oracle for the MoE layer (TEST INFRASTRUCTURE ONLY).

Only tests, the smoke check and the benchmark's CPU-baseline leg may import
this package. The product path (the CUDA library and its binding) never does,
and shares no code with it. The arithmetic lives in ``oracle.c`` (plain C,
fp32 with fp64 router sums); this module builds it with gcc and wraps it with
ctypes and numpy. ``lru.py`` simulates the expert cache policy.

The pages print no layer-level values, so the tests pin every function to
hand-worked fixtures, library routines, closed forms, invariants and brute
force instead, and check that planted mistakes are caught.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional

import numpy as np

from .lru import CacheFull, LruSim  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "_oracle.so")
_lib = None

FMT = {"bf16": 0, "fp8": 1, "mxfp4": 2, "nvfp4": 3}
ACT = {"a16": 0, "a4": 1}


def build(force: bool = False) -> str:
    """Compile oracle.c into _oracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _bind(path: str):
    """Load a build of oracle.c and declare its entry points."""
    L = C.CDLL(path)
    P = C.c_void_p
    i = C.c_int
    f = C.c_float
    L.oracle_e2m1.restype = C.c_double
    L.oracle_e2m1.argtypes = [i]
    L.oracle_e8m0.restype = C.c_double
    L.oracle_e8m0.argtypes = [i]
    L.oracle_e4m3.restype = C.c_double
    L.oracle_e4m3.argtypes = [i]
    L.oracle_bf16_round.restype = C.c_double
    L.oracle_bf16_round.argtypes = [C.c_double]
    L.oracle_dequant.restype = i
    L.oracle_dequant.argtypes = [i, i, i, P, P, f, P]
    L.oracle_route.restype = None
    L.oracle_route.argtypes = [P, i, i, P, i, P, i, i, P, P, P]
    L.oracle_permute.restype = None
    L.oracle_permute.argtypes = [P, i, i, i, P, P, P]
    L.oracle_ffn.restype = i
    L.oracle_ffn.argtypes = [P, i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, P, i]
    L.oracle_combine.restype = None
    L.oracle_combine.argtypes = [P, P, P, i, i, i, P]
    L.oracle_layer.restype = i
    L.oracle_layer.argtypes = [P, i, i, P, i, P, i, i, i, i, P, P, P, P, P, P, P, P, P, P, P, P, P, i]
    L.oracle_token_rows.restype = i
    L.oracle_token_rows.argtypes = [P, i, i, i, i, P, P, P, P, P, P, P, P, P, i, P, i, i]
    L.oracle_e4m3_encode.restype = i
    L.oracle_e4m3_encode.argtypes = [f]
    L.oracle_e2m1_encode.restype = i
    L.oracle_e2m1_encode.argtypes = [f]
    L.oracle_a4_tensor_scale.restype = f
    L.oracle_a4_tensor_scale.argtypes = [P, C.c_size_t]
    L.oracle_a4_quant.restype = None
    L.oracle_a4_quant.argtypes = [P, i, f, P, P, P]
    L.oracle_threads.restype = i
    L.oracle_threads.argtypes = []
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _np(t, dtype=None):
    """numpy view of a CPU tensor/array (bf16 tensors become uint16 bit patterns)."""
    if t is None:
        return None
    try:
        import torch

        if isinstance(t, torch.Tensor):
            t = t.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16:
                t = t.view(torch.uint16) if hasattr(torch, "uint16") else t.view(torch.int16)
            a = t.numpy()
            if a.dtype == np.int16:
                a = a.view(np.uint16)
            return np.ascontiguousarray(a if dtype is None else a.astype(dtype))
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(t)
    return a if dtype is None else a.astype(dtype)


def e2m1(code: int) -> float:
    return lib().oracle_e2m1(code)


def e8m0(code: int) -> float:
    return lib().oracle_e8m0(code)


def e4m3(code: int) -> float:
    return lib().oracle_e4m3(code)


def bf16_round(v: float) -> float:
    return lib().oracle_bf16_round(v)


def e4m3_encode(v: float) -> int:
    """Nearest E4M3 code of a magnitude (ties to the even code, saturating at 448)."""
    return lib().oracle_e4m3_encode(float(v))


def e2m1_encode(v: float) -> int:
    """Nearest E2M1 code (ties to the even code, saturating at 6; bit 3 = sign)."""
    return lib().oracle_e2m1_encode(float(v))


def a4_tensor_scale(x) -> float:
    """Per-tensor scale of activations x in the A4 form: amax / (6 * 448) (1 if all zero)."""
    xn = _np(x)
    return float(lib().oracle_a4_tensor_scale(_p(xn), xn.size))


def a4_quant(v, s_g: float):
    """A4 form of rows v[n, K] (fp32, K % 16 == 0) with tensor scale s_g.
    Returns (values, E2M1 codes [n, K], E4M3 scale codes [n, K/16])."""
    v = np.ascontiguousarray(v, np.float32)
    n, K = v.shape
    out = np.empty_like(v)
    codes = np.empty((n, K), np.uint8)
    scales = np.empty((n, K // 16), np.uint8)
    for r in range(n):
        lib().oracle_a4_quant(_p(v[r]), K, float(s_g), _p(out[r]), _p(codes[r]), _p(scales[r]))
    return out, codes, scales


def threads() -> int:
    return lib().oracle_threads()


def dequant(fmt: str, w, scale=None, tscale: float = 1.0, rows: Optional[int] = None, K: Optional[int] = None):
    """Dequantise one expert tensor to fp32 [rows, K]."""
    wn = _np(w)
    sn = _np(scale)
    if rows is None:
        rows = wn.shape[-2]
    if K is None:
        K = wn.shape[-1] * (2 if fmt in ("mxfp4", "nvfp4") else 1)
    out = np.empty((rows, K), np.float32)
    rc = lib().oracle_dequant(FMT[fmt], rows, K, _p(wn), _p(sn), float(tscale), _p(out))
    if rc:
        raise ValueError("bad format/shape")
    return out


def route(x, wr, k: int, bias=None, with_logits: bool = True):
    xn = _np(x)
    T, H = xn.shape
    wrn = _np(wr)
    E = wrn.shape[1]
    wr_is_fp32 = int(wrn.dtype == np.float32)
    bn = None if bias is None else _np(bias, np.float32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    logits = np.empty((T, E), np.float32) if with_logits else None
    lib().oracle_route(_p(xn), T, H, _p(wrn), wr_is_fp32, _p(bn), E, k, _p(idx), _p(w), _p(logits))
    return idx, w, logits


def permute(idx: np.ndarray, E: int):
    idx = np.ascontiguousarray(idx, np.int32)
    T, k = idx.shape
    off = np.empty(E + 1, np.int32)
    sp = np.empty(T * k, np.int32)
    pr = np.empty(T * k, np.int32)
    lib().oracle_permute(_p(idx), T, k, E, _p(off), _p(sp), _p(pr))
    return off, sp, pr


def _layer_arrays(layer):
    return (FMT[layer.fmt], _np(layer.w13), _np(layer.w13_scale), _np(layer.w13_tscale, np.float32),
            _np(layer.w2), _np(layer.w2_scale), _np(layer.w2_tscale, np.float32))


def ffn(x, layer, offsets, sorted_pair, k: int, want_h: bool = False, act: str = "a16"):
    xn = _np(x)
    T, H = xn.shape
    f, w13, s13, t13, w2, s2, t2 = _layer_arrays(layer)
    P = T * k
    y = np.empty((P, H), np.float32)
    h = np.empty((P, layer.I), np.float32) if want_h else None
    rc = lib().oracle_ffn(_p(xn), T, H, layer.I, layer.E, k, f, _p(w13), _p(s13), _p(t13), _p(w2), _p(s2), _p(t2),
                          _p(np.ascontiguousarray(offsets, np.int32)), _p(np.ascontiguousarray(sorted_pair, np.int32)),
                          _p(y), _p(h), ACT[act])
    if rc:
        raise ValueError("bad format")
    return (y, h) if want_h else y


def combine(y_perm: np.ndarray, pair_row: np.ndarray, w: np.ndarray, T: int, k: int):
    y_perm = np.ascontiguousarray(y_perm, np.float32)
    H = y_perm.shape[1]
    out = np.empty((T, H), np.float32)
    lib().oracle_combine(_p(y_perm), _p(np.ascontiguousarray(pair_row, np.int32)),
                         _p(np.ascontiguousarray(w, np.float32)), T, k, H, _p(out))
    return out


def layer_forward(x, layer, bias="layer", act: str = "a16"):
    """Whole layer. Returns dict(idx, w, offsets, sorted_pair, pair_row, y_perm, out)."""
    xn = _np(x)
    T, H = xn.shape
    k = layer.k
    wrn = _np(layer.wr)
    b = layer.bias if isinstance(bias, str) else bias
    bn = None if b is None else _np(b, np.float32)
    f, w13, s13, t13, w2, s2, t2 = _layer_arrays(layer)
    P = T * k
    r = dict(idx=np.empty((T, k), np.int32), w=np.empty((T, k), np.float32),
             offsets=np.empty(layer.E + 1, np.int32), sorted_pair=np.empty(P, np.int32),
             pair_row=np.empty(P, np.int32), y_perm=np.empty((P, H), np.float32), out=np.empty((T, H), np.float32))
    rc = lib().oracle_layer(_p(xn), T, H, _p(wrn), int(wrn.dtype == np.float32), _p(bn), layer.E, k, layer.I, f,
                            _p(w13), _p(s13), _p(t13), _p(w2), _p(s2), _p(t2), _p(r["idx"]), _p(r["w"]),
                            _p(r["offsets"]), _p(r["sorted_pair"]), _p(r["pair_row"]), _p(r["y_perm"]), _p(r["out"]),
                            ACT[act])
    if rc:
        raise ValueError("bad format")
    return r


def token_rows(x, layer, idx, w, tokens, act: str = "a16"):
    """out rows for the listed tokens given the batch routing (idx, w); x is the whole batch."""
    xn = _np(x)
    T, H = xn.shape
    f, w13, s13, t13, w2, s2, t2 = _layer_arrays(layer)
    toks = np.ascontiguousarray(tokens, np.int32)
    out = np.empty((len(toks), H), np.float32)
    rc = lib().oracle_token_rows(_p(xn), H, layer.I, layer.k, f, _p(w13), _p(s13), _p(t13), _p(w2), _p(s2), _p(t2),
                                 _p(np.ascontiguousarray(idx, np.int32)), _p(np.ascontiguousarray(w, np.float32)),
                                 _p(toks), len(toks), _p(out), T, ACT[act])
    if rc:
        raise ValueError("bad format")
    return out
