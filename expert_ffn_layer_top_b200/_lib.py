"""ctypes binding of libmoe.so. Argument marshalling only (see include/moe.h)."""
from __future__ import annotations

import ctypes as C
import os
import threading
from typing import List, Optional, Sequence

import torch

from . import build as _build

FMT = {"bf16": 0, "fp8": 1, "mxfp4": 2, "nvfp4": 3}
ACT = {"a16": 0, "a4": 1}
_STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "OOM", 5: "TIMEOUT", 6: "CACHE_FULL"}

_P = C.c_void_p
_I = C.c_int
_lock = threading.Lock()
_lib_handle = None


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status
        self.name = _STATUS.get(status, str(status))


class _Experts(C.Structure):
    _fields_ = [
        ("fmt", C.c_int), ("E", C.c_int), ("H", C.c_int), ("I", C.c_int),
        ("w13", _P), ("w13_scale", _P), ("w13_tscale", _P),
        ("w2", _P), ("w2_scale", _P), ("w2_tscale", _P),
        ("w13_estride", C.c_int64), ("w13s_estride", C.c_int64),
        ("w2_estride", C.c_int64), ("w2s_estride", C.c_int64),
        ("expert_map", _P), ("n_entries", C.c_int), ("layout", C.c_int),
    ]


class _CacheReport(C.Structure):
    _fields_ = [
        ("table_s", C.c_double), ("host_wait_s", C.c_double), ("issue_s", C.c_double), ("copy_s", C.c_double),
        ("compute_s", C.c_double), ("overlap_s", C.c_double), ("h2d_gbs", C.c_double),
        ("calls", C.c_uint64), ("prefetched", C.c_uint64), ("moved", C.c_uint64),
        ("n_slots", C.c_int), ("last_depth", C.c_int),
    ]


PREFETCH = {"none": 0, "predicted": 1, "full_layer": 2, "adaptive": 3}


def lib():
    """Load (building first if missing or stale) libmoe.so; raises if that fails."""
    global _lib_handle
    with _lock:
        if _lib_handle is None:
            path = _build.LIB
            if _build.needs_build():
                try:
                    _build.build()
                except Exception as e:  # no silent fallback
                    if not os.path.exists(path):
                        raise RuntimeError(f"libmoe.so is not built and the build failed: {e}") from e
            L = C.CDLL(path)
            st = _I
            L.moe_route_topk.restype = st
            L.moe_route_topk.argtypes = [_P, _I, _I, _P, _I, _P, _I, _I, _P, _P, _P, _P, C.c_size_t, _P]
            L.moe_permute.restype = st
            L.moe_permute.argtypes = [_P, _I, _I, _I, _P, _I, _I, _P, _P, _P, _P, _P, C.c_size_t, _P]
            L.moe_permute_static.restype = st
            L.moe_permute_static.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P]
            L.moe_grouped_ffn.restype = st
            L.moe_grouped_ffn.argtypes = [_P, _I, _P, C.POINTER(_Experts), _I, _P, _I, _P, C.c_size_t, _P]
            L.moe_combine.restype = st
            L.moe_combine.argtypes = [_P, _I, _P, _P, _I, _I, _I, _P, _P]
            L.moe_dequantize.restype = st
            L.moe_dequantize.argtypes = [_I, _P, _P, C.c_float, _I, _I, _P, _P]
            L.moe_layer_forward.restype = st
            L.moe_layer_forward.argtypes = [_P, _I, _P, _I, _P, _I, C.POINTER(_Experts), _I, _P, _I, _I, _P, _P,
                                            _P, _P, C.c_size_t, _P]
            L.moe_prepacked_expert_bytes.restype = C.c_size_t
            L.moe_prepacked_expert_bytes.argtypes = [_I, _I, _I, _I]
            L.moe_prepack.restype = st
            L.moe_prepack.argtypes = [C.POINTER(_Experts), _P, _P, _P]
            L.moe_workspace_size.restype = C.c_size_t
            L.moe_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I, _I]
            L.expert_cache_init.restype = st
            L.expert_cache_init.argtypes = [C.POINTER(_P), C.c_size_t, _I, C.POINTER(_Experts), _I]
            L.expert_cache_prefetch.restype = st
            L.expert_cache_prefetch.argtypes = [_P, _I, _P, _I, _P]
            L.expert_cache_evict.restype = st
            L.expert_cache_evict.argtypes = [_P, _I, _P, _I]
            L.expert_cache_stats.restype = st
            L.expert_cache_stats.argtypes = [_P, C.POINTER(C.c_uint64), C.POINTER(C.c_uint64),
                                             C.POINTER(C.c_uint64), C.POINTER(C.c_double)]
            L.expert_cache_set_prefetch.restype = st
            L.expert_cache_set_prefetch.argtypes = [_P, _I, _I]
            L.expert_cache_resize.restype = st
            L.expert_cache_resize.argtypes = [_P, C.c_size_t]
            L.expert_cache_report.restype = st
            L.expert_cache_report.argtypes = [_P, C.POINTER(_CacheReport)]
            L.moe_set_wait_limit_ns.restype = st
            L.moe_set_wait_limit_ns.argtypes = [C.c_uint64]
            L.moe_tensor_peak.restype = st
            L.moe_tensor_peak.argtypes = [_I, _I, C.POINTER(C.c_double)]
            L.moe_selftest_wait.restype = st
            L.moe_selftest_wait.argtypes = [_P]
            L.expert_cache_slot_of.restype = st
            L.expert_cache_slot_of.argtypes = [_P, _I, _I, C.POINTER(C.c_int32)]
            L.expert_cache_destroy.restype = st
            L.expert_cache_destroy.argtypes = [_P]
            L.moe_last_error_string.restype = C.c_char_p
            L.moe_last_error_string.argtypes = []
            L.moe_device_error.restype = st
            L.moe_device_error.argtypes = [C.POINTER(C.c_int)]
            L.moe_version.restype = C.c_char_p
            L.moe_version.argtypes = []
            L.moe_kernel_launch_count.restype = C.c_uint64
            L.moe_kernel_launch_count.argtypes = []
            _lib_handle = L
    return _lib_handle


def _check(status: int):
    if status != 0:
        raise MoeError(status, lib().moe_last_error_string().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("device tensors expected")


def moe_version() -> str:
    return lib().moe_version().decode()


def moe_kernel_launch_count() -> int:
    """Kernels the library has enqueued in this process so far."""
    return int(lib().moe_kernel_launch_count())


def moe_device_error() -> int:
    code = C.c_int(0)
    _check(lib().moe_device_error(C.byref(code)))
    return code.value


def moe_set_wait_limit_ns(ns: int) -> None:
    """Limit of the bounded device waits in ns (0 = the 2 s default); a test hook."""
    _check(lib().moe_set_wait_limit_ns(int(ns)))


def moe_selftest_wait(stream=None) -> None:
    """Enqueue the kernel whose bounded wait must give up (sets device error 1)."""
    _check(lib().moe_selftest_wait(_stream(stream)))


_PEAK_KIND = {"bf16": 0, "fp8": 1, "mxfp4": 2, "nvfp4": 3}


def moe_tensor_peak_tflops(kind: str, iters: int = 4000) -> float:
    """Dense tensor-core TFLOP/s of the current device for one MMA kind (library MMA loop)."""
    v = C.c_double()
    _check(lib().moe_tensor_peak(_PEAK_KIND[kind], int(iters), C.byref(v)))
    return v.value


def moe_workspace_size(T: int, H: int, I: int, E: int, k: int, y_fp32: bool = False, act: str = "a16") -> int:
    return int(lib().moe_workspace_size(T, H, I, E, k, int(y_fp32), ACT[act]))


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


class Experts:
    """A layer's experts (a moe_experts descriptor plus the tensors it points at)."""

    def __init__(self, fmt: str, E: int, H: int, I: int, w13, w2, w13_scale=None, w2_scale=None,
                 w13_tscale=None, w2_tscale=None, strides=(0, 0, 0, 0), expert_map=None, n_entries=0,
                 layout: int = 0):
        self.fmt, self.E, self.H, self.I, self.layout = fmt, E, H, I, layout
        self.w13, self.w2, self.w13_scale, self.w2_scale = w13, w2, w13_scale, w2_scale
        self.w13_tscale, self.w2_tscale = w13_tscale, w2_tscale
        self._keep = [w13, w2, w13_scale, w2_scale, w13_tscale, w2_tscale, expert_map]
        self.c = _Experts(FMT[fmt], E, H, I, _ptr(w13), _ptr(w13_scale), _ptr(w13_tscale), _ptr(w2), _ptr(w2_scale),
                          _ptr(w2_tscale), strides[0], strides[1], strides[2], strides[3], _ptr(expert_map),
                          n_entries, layout)

    @classmethod
    def from_layer(cls, layer) -> "Experts":
        """From an object with fmt/E/H/I/w13/w2/*_scale/*_tscale tensor attributes."""
        return cls(layer.fmt, layer.E, layer.H, layer.I, layer.w13, layer.w2, layer.w13_scale, layer.w2_scale,
                   layer.w13_tscale, layer.w2_tscale)


LAYOUT_STANDARD, LAYOUT_TILED = 0, 1


def moe_prepacked_expert_bytes(fmt: str, H: int, I: int, which: int) -> int:
    return int(lib().moe_prepacked_expert_bytes(FMT[fmt], H, I, which))


def moe_prepack(experts: Experts) -> Experts:
    """Tiled (prepacked) copy of standard-layout device experts (see moe_prepack in moe.h)."""
    _need_cuda(experts.w13, experts.w2)
    dev = experts.w13.device
    b13 = moe_prepacked_expert_bytes(experts.fmt, experts.H, experts.I, 0)
    b2 = moe_prepacked_expert_bytes(experts.fmt, experts.H, experts.I, 1)
    o13 = torch.empty(experts.E * b13, dtype=torch.uint8, device=dev)
    o2 = torch.empty(experts.E * b2, dtype=torch.uint8, device=dev)
    _check(lib().moe_prepack(C.byref(experts.c), _ptr(o13), _ptr(o2), _stream()))
    return Experts(experts.fmt, experts.E, experts.H, experts.I, o13, o2, None, None, experts.w13_tscale,
                   experts.w2_tscale, layout=LAYOUT_TILED)


def moe_route_topk(x: torch.Tensor, wr: torch.Tensor, k: int, bias: Optional[torch.Tensor] = None,
                   want_logits: bool = False, ws: Optional[torch.Tensor] = None):
    _need_cuda(x, wr, bias)
    T, H = x.shape
    E = wr.shape[1]
    idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    logits = torch.empty(T, E, dtype=torch.float32, device=x.device) if want_logits else None
    if ws is None:
        ws = _ws(moe_workspace_size(T, H, 128, E, k), x.device)
    _check(lib().moe_route_topk(_ptr(x), T, H, _ptr(wr), int(wr.dtype == torch.float32), _ptr(bias), E, k,
                                _ptr(idx), _ptr(w), _ptr(logits), _ptr(ws), ws.numel(), _stream()))
    return (idx, w, logits) if want_logits else (idx, w)


def moe_permute(idx: torch.Tensor, E: int, x: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                act: str = "a16"):
    _need_cuda(idx, x)
    T, k = idx.shape
    dev = idx.device
    P = T * k
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sp = torch.empty(max(P, 1), dtype=torch.int32, device=dev)
    pr = torch.empty(max(P, 1), dtype=torch.int32, device=dev)
    H = x.shape[1] if x is not None else 0
    x_perm = torch.empty(max(P, 1), H, dtype=torch.bfloat16, device=dev) if x is not None else None
    if ws is None:
        ws = _ws(moe_workspace_size(T, max(H, 8), 128, E, k, act=act), dev)
    _check(lib().moe_permute(_ptr(idx), T, k, E, _ptr(x), H, ACT[act], _ptr(offsets), _ptr(sp), _ptr(pr),
                             _ptr(x_perm), _ptr(ws), ws.numel(), _stream()))
    return offsets, sp[:P], pr[:P], (x_perm[:P] if x_perm is not None else None)


def moe_permute_static(idx: torch.Tensor, E: int, x: Optional[torch.Tensor] = None):
    """moe_permute with the library's fixed device scratch instead of a workspace."""
    _need_cuda(idx, x)
    T, k = idx.shape
    dev = idx.device
    P = T * k
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sp = torch.empty(max(P, 1), dtype=torch.int32, device=dev)
    pr = torch.empty(max(P, 1), dtype=torch.int32, device=dev)
    H = x.shape[1] if x is not None else 0
    x_perm = torch.empty(max(P, 1), H, dtype=torch.bfloat16, device=dev) if x is not None else None
    _check(lib().moe_permute_static(_ptr(idx), T, k, E, _ptr(x), H, _ptr(offsets), _ptr(sp), _ptr(pr),
                                    _ptr(x_perm), _stream()))
    return offsets, sp[:P], pr[:P], (x_perm[:P] if x_perm is not None else None)


def moe_grouped_ffn(x_perm: torch.Tensor, offsets: torch.Tensor, experts: Experts, y_fp32: bool = False,
                    ws: Optional[torch.Tensor] = None, act: str = "a16") -> torch.Tensor:
    _need_cuda(x_perm, offsets)
    n = x_perm.shape[0]
    y = torch.empty(max(n, 1), experts.H, dtype=torch.float32 if y_fp32 else torch.bfloat16, device=x_perm.device)
    if ws is None:
        ws = _ws(moe_workspace_size(max(n, 1), experts.H, experts.I, experts.E, 1, y_fp32, act), x_perm.device)
    _check(lib().moe_grouped_ffn(_ptr(x_perm), n, _ptr(offsets), C.byref(experts.c), ACT[act], _ptr(y), int(y_fp32),
                                 _ptr(ws), ws.numel(), _stream()))
    return y[:n]


def moe_combine(y_perm: torch.Tensor, pair_row: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
    _need_cuda(y_perm, pair_row, w)
    T, k = w.shape
    H = y_perm.shape[1]
    out = torch.empty(T, H, dtype=torch.bfloat16, device=w.device)
    _check(lib().moe_combine(_ptr(y_perm), int(y_perm.dtype == torch.float32), _ptr(pair_row), _ptr(w), T, k, H,
                             _ptr(out), _stream()))
    return out


def moe_dequantize(fmt: str, w: torch.Tensor, scale: Optional[torch.Tensor], tscale: float, rows: int,
                   K: int) -> torch.Tensor:
    _need_cuda(w, scale)
    out = torch.empty(rows, K, dtype=torch.bfloat16, device=w.device)
    _check(lib().moe_dequantize(FMT[fmt], _ptr(w), _ptr(scale), float(tscale), rows, K, _ptr(out), _stream()))
    return out


def moe_layer_forward(x: torch.Tensor, wr: torch.Tensor, k: int, experts: Experts,
                      bias: Optional[torch.Tensor] = None, cache: Optional["ExpertCache"] = None, layer: int = 0,
                      y_fp32: bool = False, ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                      idx_out: Optional[torch.Tensor] = None, w_out: Optional[torch.Tensor] = None,
                      act: str = "a16") -> torch.Tensor:
    _need_cuda(x, wr, bias, ws, out, idx_out, w_out)
    T, H = x.shape
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = _ws(moe_workspace_size(T, H, experts.I, experts.E, k, y_fp32, act), x.device)
    _check(lib().moe_layer_forward(_ptr(x), T, _ptr(wr), int(wr.dtype == torch.float32), _ptr(bias), k,
                                   C.byref(experts.c), ACT[act], cache.handle if cache is not None else None, layer,
                                   int(y_fp32), _ptr(out), _ptr(idx_out), _ptr(w_out), _ptr(ws), ws.numel(),
                                   _stream()))
    return out


class ExpertCache:
    """Device LRU expert cache over a pinned host pool (expert_cache_* in moe.h)."""

    def __init__(self, capacity_bytes: int, host_layers: Sequence[Experts], device: int = 0):
        self._layers = list(host_layers)   # keep the host tensors alive
        arr = (_Experts * len(self._layers))(*[l.c for l in self._layers])
        h = C.c_void_p(None)
        _check(lib().expert_cache_init(C.byref(h), capacity_bytes, len(self._layers), arr, device))
        self.handle = h

    def prefetch(self, layer: int, ids: Sequence[int]):
        a = (C.c_int32 * max(len(ids), 1))(*[int(i) for i in ids])
        _check(lib().expert_cache_prefetch(self.handle, layer, a, len(ids), _stream()))

    def evict(self, layer: int = -1, ids: Optional[Sequence[int]] = None):
        if ids is None:
            _check(lib().expert_cache_evict(self.handle, layer, None, -1))
        else:
            a = (C.c_int32 * max(len(ids), 1))(*[int(i) for i in ids])
            _check(lib().expert_cache_evict(self.handle, layer, a, len(ids)))

    def stats(self) -> dict:
        h, m, b = C.c_uint64(), C.c_uint64(), C.c_uint64()
        s = C.c_double()
        _check(lib().expert_cache_stats(self.handle, C.byref(h), C.byref(m), C.byref(b), C.byref(s)))
        return dict(hits=h.value, misses=m.value, bytes_h2d=b.value, copy_s=s.value)

    def set_prefetch(self, policy: str, depth: int = -1):
        """Next-layer prefetch: 'none', 'predicted' (first `depth`, -1 all), 'full_layer', 'adaptive'."""
        _check(lib().expert_cache_set_prefetch(self.handle, PREFETCH[policy], int(depth)))

    def resize(self, capacity_bytes: int):
        _check(lib().expert_cache_resize(self.handle, int(capacity_bytes)))

    def report(self) -> dict:
        r = _CacheReport()
        _check(lib().expert_cache_report(self.handle, C.byref(r)))
        return {name: getattr(r, name) for name, _ in _CacheReport._fields_}

    def slot_of(self, layer: int, e: int) -> int:
        v = C.c_int32()
        _check(lib().expert_cache_slot_of(self.handle, layer, e, C.byref(v)))
        return v.value

    def close(self):
        if self.handle:
            _check(lib().expert_cache_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
