"""B200-native (sm_100a) Mixture-of-Experts layer forward.

Python binding of the C ABI in ``include/moe.h`` (``libmoe.so``, built in-tree by
``mixture_experts_layer_logits_b200/build.py``).  The functions here only marshal
arguments -- device pointers, the shape struct and the current CUDA stream --
into the library; every step of the layer runs in its CUDA kernels.  There is no
fallback: if the library is missing or a call fails, an exception is raised.

torch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MoeError", "Shape", "moe_workspace_size", "moe_route", "moe_permute", "moe_grouped_ffn",
    "moe_combine", "moe_forward", "moe_forward_timed", "moe_forward_kernel_count",
    "moe_forward_fused", "moe_forward_w8", "moe_forward_w8_supported", "moe_selftest_wait_timeout",
    "moe_device_status", "library_path", "load_library",
    "MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED_SHAPE", "MOE_ERR_MISALIGNED",
    "MOE_ERR_WORKSPACE_TOO_SMALL", "MOE_ERR_CUDA", "MOE_ERR_DEVICE_TIMEOUT",
    "MOE_ERR_DEVICE_BOUNDS", "debug_library_path",
]

(MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_MISALIGNED,
 MOE_ERR_WORKSPACE_TOO_SMALL, MOE_ERR_CUDA, MOE_ERR_DEVICE_TIMEOUT,
 MOE_ERR_DEVICE_BOUNDS) = range(8)

_HERE = os.path.dirname(os.path.abspath(__file__))
# libmoe_debug.so: the same library with the kernels' input-index checks compiled
# in (moe_device_status then reports MOE_ERR_DEVICE_BOUNDS); MOE_LIBRARY=debug in
# the environment selects it at import.
debug_library_path = os.path.join(_HERE, "libmoe_debug.so")
library_path = (debug_library_path if os.environ.get("MOE_LIBRARY", "") == "debug"
                else os.path.join(_HERE, "libmoe.so"))


class Shape(ctypes.Structure):
    """moe_shape_t: T tokens, E experts, top_k, H hidden, I intermediate."""

    _fields_ = [("T", ctypes.c_int32), ("E", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("H", ctypes.c_int32), ("I", ctypes.c_int32)]

    def __repr__(self):
        return f"Shape(T={self.T}, E={self.E}, top_k={self.top_k}, H={self.H}, I={self.I})"


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load_library()
        msg = lib.moe_status_string(status).decode()
        if status == MOE_ERR_CUDA:
            msg += f" (cudaError {lib.moe_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")
        self.status = status


_lib = None
_vp = ctypes.c_void_p


def load_library():
    """Load the library at library_path (raises OSError if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise OSError(f"{library_path} is missing: run mixture_experts_layer_logits_b200/build.py")
    lib = ctypes.CDLL(library_path)
    lib.moe_workspace_size.argtypes = [Shape]
    lib.moe_workspace_size.restype = ctypes.c_size_t
    lib.moe_route.argtypes = [_vp, Shape, _vp, _vp, _vp]
    lib.moe_permute.argtypes = [_vp, Shape, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.moe_grouped_ffn.argtypes = [_vp, _vp, _vp, _vp, _vp, Shape, _vp, _vp, ctypes.c_size_t, _vp]
    lib.moe_combine.argtypes = [_vp, _vp, Shape, _vp, _vp]
    lib.moe_forward.argtypes = [_vp, _vp, _vp, _vp, Shape, _vp, _vp, _vp, _vp, _vp, _vp,
                                ctypes.c_size_t, _vp]
    lib.moe_forward_timed.argtypes = [_vp, _vp, _vp, _vp, Shape, _vp, _vp, _vp, _vp, _vp, _vp,
                                      ctypes.c_size_t, _vp, ctypes.POINTER(_vp), ctypes.c_int]
    lib.moe_forward_w8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, Shape, _vp, _vp, _vp, _vp, _vp,
                                   _vp, ctypes.c_size_t, _vp]
    lib.moe_forward_w8_timed.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, Shape, _vp, _vp, _vp, _vp,
                                         _vp, _vp, ctypes.c_size_t, _vp, ctypes.POINTER(_vp),
                                         ctypes.c_int]
    lib.moe_forward_w8_supported.argtypes = [Shape]
    lib.moe_forward_w8_supported.restype = ctypes.c_int
    lib.moe_forward_kernel_count.argtypes = [Shape]
    lib.moe_forward_kernel_count.restype = ctypes.c_int
    lib.moe_forward_fused.argtypes = [Shape]
    lib.moe_forward_fused.restype = ctypes.c_int
    lib.moe_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint,
                                              ctypes.c_void_p]
    lib.moe_selftest_wait_timeout.restype = ctypes.c_int
    lib.moe_device_status.argtypes = [_vp, ctypes.c_size_t, _vp]
    for fn in (lib.moe_route, lib.moe_permute, lib.moe_grouped_ffn, lib.moe_combine,
               lib.moe_forward, lib.moe_forward_timed, lib.moe_forward_w8,
               lib.moe_forward_w8_timed, lib.moe_device_status):
        fn.restype = ctypes.c_int
    lib.moe_status_string.argtypes = [ctypes.c_int]
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_last_cuda_error.argtypes = []
    lib.moe_last_cuda_error.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def _need(t: torch.Tensor, name: str, dtype, shape):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def moe_workspace_size(T: int, E: int, top_k: int, H: int = 0, I: int = 0) -> int:
    return int(load_library().moe_workspace_size(Shape(T, E, top_k, H, I)))


def workspace(T: int, E: int, top_k: int, H: int = 0, I: int = 0, device="cuda") -> torch.Tensor:
    """A device workspace big enough for the shape (uint8)."""
    n = moe_workspace_size(T, E, top_k, H, I)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_route(logits: torch.Tensor, top_k: int, topk_ids=None, topk_weights=None):
    T, E = logits.shape
    _need(logits, "logits", torch.float32, (T, E))
    ids = topk_ids if topk_ids is not None else torch.empty(T, top_k, dtype=torch.int32,
                                                            device=logits.device)
    w = topk_weights if topk_weights is not None else torch.empty(T, top_k, dtype=torch.float32,
                                                                  device=logits.device)
    _need(ids, "topk_ids", torch.int32, (T, top_k))
    _need(w, "topk_weights", torch.float32, (T, top_k))
    _check(load_library().moe_route(_ptr(logits), Shape(T, E, top_k, 0, 0), _ptr(ids), _ptr(w),
                                    _stream(logits)), "moe_route")
    return ids, w


def moe_permute(topk_ids: torch.Tensor, E: int, ws: torch.Tensor = None, expert_offsets=None,
                permuted_rows=None):
    T, k = topk_ids.shape
    _need(topk_ids, "topk_ids", torch.int32, (T, k))
    dev = topk_ids.device
    if ws is None:
        ws = workspace(T, E, k, device=dev)
    off = expert_offsets if expert_offsets is not None else torch.empty(E + 1, dtype=torch.int32,
                                                                        device=dev)
    rows = permuted_rows if permuted_rows is not None else torch.empty(T * k, dtype=torch.int32,
                                                                       device=dev)
    _need(off, "expert_offsets", torch.int32, (E + 1,))
    _need(rows, "permuted_rows", torch.int32, (T * k,))
    _check(load_library().moe_permute(_ptr(topk_ids), Shape(T, E, k, 0, 0), _ptr(off), _ptr(rows),
                                      _ptr(ws), ws.numel(), _stream(topk_ids)), "moe_permute")
    return off, rows


def moe_grouped_ffn(x, w13, w2, expert_offsets, permuted_rows, top_k: int, ws=None, y=None):
    T, H = x.shape
    E, twoI, _ = w13.shape
    I = twoI // 2
    dev = x.device
    _need(x, "x", torch.bfloat16, (T, H))
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H))
    _need(w2, "w2", torch.bfloat16, (E, H, I))
    _need(expert_offsets, "expert_offsets", torch.int32, (E + 1,))
    _need(permuted_rows, "permuted_rows", torch.int32, (T * top_k,))
    if ws is None:
        ws = workspace(T, E, top_k, H, I, device=dev)
    if y is None:
        y = torch.empty(T * top_k, H, dtype=torch.bfloat16, device=dev)
    _need(y, "y", torch.bfloat16, (T * top_k, H))
    _check(load_library().moe_grouped_ffn(_ptr(x), _ptr(w13), _ptr(w2), _ptr(expert_offsets),
                                          _ptr(permuted_rows), Shape(T, E, top_k, H, I), _ptr(y),
                                          _ptr(ws), ws.numel(), _stream(x)), "moe_grouped_ffn")
    return y


def moe_combine(y, topk_weights, out=None):
    T, k = topk_weights.shape
    H = y.shape[1]
    _need(y, "y", torch.bfloat16, (T * k, H))
    _need(topk_weights, "topk_weights", torch.float32, (T, k))
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=y.device)
    _need(out, "out", torch.bfloat16, (T, H))
    _check(load_library().moe_combine(_ptr(y), _ptr(topk_weights), Shape(T, k, k, H, 0),
                                      _ptr(out), _stream(y)), "moe_combine")
    return out


def _forward(x, logits, w13, w2, top_k, ws, out, topk_ids, topk_weights, expert_offsets,
             permuted_rows, events, scales=None):
    T, H = x.shape
    E = logits.shape[1]
    I = w13.shape[1] // 2
    dev = x.device
    wdt = torch.bfloat16 if scales is None else torch.uint8
    _need(x, "x", torch.bfloat16, (T, H))
    _need(logits, "logits", torch.float32, (T, E))
    _need(w13, "w13", wdt, (E, 2 * I, H))
    _need(w2, "w2", wdt, (E, H, I))
    if scales is not None:
        _need(scales[0], "w13_scale", torch.float32, (E, 2 * I))
        _need(scales[1], "w2_scale", torch.float32, (E, H))
    if ws is None:
        ws = workspace(T, E, top_k, H, I, device=dev)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (T, H))
    for t, name, dt, shp in ((topk_ids, "topk_ids", torch.int32, (T, top_k)),
                             (topk_weights, "topk_weights", torch.float32, (T, top_k)),
                             (expert_offsets, "expert_offsets", torch.int32, (E + 1,)),
                             (permuted_rows, "permuted_rows", torch.int32, (T * top_k,))):
        if t is not None:
            _need(t, name, dt, shp)
    weights = ((_ptr(w13), _ptr(w2)) if scales is None else
               (_ptr(w13), _ptr(scales[0]), _ptr(w2), _ptr(scales[1])))
    args = (_ptr(x), _ptr(logits), *weights, Shape(T, E, top_k, H, I), _ptr(out),
            _ptr(topk_ids), _ptr(topk_weights), _ptr(expert_offsets), _ptr(permuted_rows),
            _ptr(ws), ws.numel(), _stream(x))
    lib = load_library()
    name = "moe_forward" if scales is None else "moe_forward_w8"
    if events is None:
        _check(getattr(lib, name)(*args), name)
    else:
        arr = (_vp * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
        _check(getattr(lib, name + "_timed")(*args, arr, len(events)), name + "_timed")
    return out


def moe_forward(x, logits, w13, w2, top_k: int, ws=None, out=None, topk_ids=None,
                topk_weights=None, expert_offsets=None, permuted_rows=None):
    return _forward(x, logits, w13, w2, top_k, ws, out, topk_ids, topk_weights, expert_offsets,
                    permuted_rows, None)


def moe_forward_timed(x, logits, w13, w2, top_k: int, events, ws=None, out=None, topk_ids=None,
                      topk_weights=None, expert_offsets=None, permuted_rows=None):
    """moe_forward that records the 5 torch.cuda.Event objects in `events` at the
    stage boundaries (before routing, after permute, after w13, after w2, after
    combine)."""
    if len(events) != 5:
        raise ValueError("moe_forward_timed needs 5 events")
    return _forward(x, logits, w13, w2, top_k, ws, out, topk_ids, topk_weights, expert_offsets,
                    permuted_rows, events)


def moe_forward_w8(x, logits, w13, w13_scale, w2, w2_scale, top_k: int, ws=None, out=None,
                   topk_ids=None, topk_weights=None, expert_offsets=None, permuted_rows=None,
                   events=None):
    """The layer with FP8 (E4M3) expert weights: w13 / w2 uint8 codes [E, 2I, H] /
    [E, H, I], w13_scale / w2_scale fp32 [E, 2I] / [E, H] (one scale per weight
    row).  Other arguments and outputs as moe_forward; `events` (5
    torch.cuda.Event, optional) as moe_forward_timed."""
    if events is not None and len(events) != 5:
        raise ValueError("moe_forward_w8 needs 5 events")
    return _forward(x, logits, w13, w2, top_k, ws, out, topk_ids, topk_weights, expert_offsets,
                    permuted_rows, events, scales=(w13_scale, w2_scale))


def moe_forward_w8_supported(T: int, E: int, top_k: int, H: int, I: int) -> bool:
    return bool(load_library().moe_forward_w8_supported(Shape(T, E, top_k, H, I)))


def moe_forward_kernel_count(T: int, E: int, top_k: int, H: int, I: int) -> int:
    return int(load_library().moe_forward_kernel_count(Shape(T, E, top_k, H, I)))


def moe_forward_fused(T: int, E: int, top_k: int, H: int, I: int) -> bool:
    """True if moe_forward runs the FFN and the combine as one persistent launch."""
    return bool(load_library().moe_forward_fused(Shape(T, E, top_k, H, I)))


def moe_selftest_wait_timeout(ws: torch.Tensor, limit_us: int) -> None:
    """Queue the failure-detection self-test: two unsatisfiable bounded waits that
    give up after limit_us and record a timeout in ws (see moe_device_status)."""
    _check(load_library().moe_selftest_wait_timeout(_ptr(ws), ws.numel(), int(limit_us),
                                                    _stream(ws)), "moe_selftest_wait_timeout")


def moe_device_status(ws: torch.Tensor) -> int:
    """Synchronise the current stream and return (and clear) the device error status."""
    return int(load_library().moe_device_status(_ptr(ws), ws.numel(), _stream(ws)))
