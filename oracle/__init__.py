"""fp64 CPU oracle of the MoE layer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
``--impl reference`` legs may import this package.  The product path (the CUDA
library and its binding) never does, and shares no code with it.

Thin ctypes wrapper over ``moe_oracle.c`` (compiled by ``oracle/build.py`` into
``oracle/libmoe_oracle.so``).  Inputs are numpy arrays on the host: logits
float32 [T,E]; x bf16 bits as uint16 [T,H]; w13 uint16 [E,2I,H]; w2 uint16
[E,H,I]; FP8 weights as uint8 E4M3 codes (q13 [E,2I,H], q2 [E,H,I]) with
float32 per-row scales (s13 [E,2I], s2 [E,H]).  What each function computes, and the passages it follows, is stated in
``moe_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from . import build as _build

        _build.build()
    lib = ctypes.CDLL(_LIB_PATH)
    i = ctypes.c_int
    lib.oracle_route.argtypes = [_f32p, i, i, i, _i32p, _f32p]
    lib.oracle_permute.argtypes = [_i32p, i, i, i, _i32p, _i32p]
    lib.oracle_ffn.argtypes = [_u16p, _u16p, _u16p, _i32p, _i32p, i, i, i, i, i, i, _f64p]
    lib.oracle_combine.argtypes = [_f64p, _f32p, i, i, i, _f64p]
    lib.oracle_forward.argtypes = [_u16p, _f32p, _u16p, _u16p, i, i, i, i, i, i, _f64p,
                                   _i32p, _f32p, _i32p, _i32p]
    lib.oracle_forward_tokens.argtypes = [_u16p, _f32p, ctypes.POINTER(_u16p),
                                          ctypes.POINTER(_u16p), i, i, i, i, i, i, i, _i32p,
                                          _f64p]
    lib.oracle_e4m3_to_double.argtypes = [_u8p, ctypes.c_long, _f64p]
    lib.oracle_round_to_bf16.argtypes = [_f64p, ctypes.c_long, _f64p]
    lib.oracle_forward_w8.argtypes = [_u16p, _f32p, _u8p, _f32p, _u8p, _f32p, i, i, i, i, i,
                                      _f64p, _i32p, _f32p, _i32p, _i32p]
    lib.oracle_forward_tokens_w8.argtypes = [_u16p, _f32p, ctypes.POINTER(_u8p),
                                             ctypes.POINTER(_f32p), ctypes.POINTER(_u8p),
                                             ctypes.POINTER(_f32p), i, i, i, i, i, i, _i32p,
                                             _f64p]
    lib.oracle_num_threads.argtypes = []
    for fn in (lib.oracle_num_threads, lib.oracle_route, lib.oracle_permute, lib.oracle_ffn, lib.oracle_combine,
               lib.oracle_forward, lib.oracle_forward_tokens, lib.oracle_e4m3_to_double,
               lib.oracle_round_to_bf16,
               lib.oracle_forward_w8, lib.oracle_forward_tokens_w8):
        fn.restype = ctypes.c_int
    _lib = lib
    return lib


def _p(a, ptype):
    return a.ctypes.data_as(ptype)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name} rejected its arguments (rc={rc})")


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else the host's cores)."""
    return int(_load().oracle_num_threads())


def route(logits: np.ndarray, k: int):
    """Top-k by raw logit (ties -> lower index), softmax over the selected k.
    Returns (topk_ids int32 [T,k], topk_weights float32 [T,k])."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _check(_load().oracle_route(_p(logits, _f32p), T, E, k, _p(ids, _i32p), _p(w, _f32p)), "route")
    return ids, w


def permute(topk_ids: np.ndarray, E: int):
    """Stable counting sort of expanded rows by expert.
    Returns (expert_offsets int32 [E+1], permuted_rows int32 [T*k])."""
    ids = _c(topk_ids, np.int32)
    T, k = ids.shape
    off = np.empty(E + 1, np.int32)
    rows = np.empty(T * k, np.int32)
    _check(_load().oracle_permute(_p(ids, _i32p), T, k, E, _p(off, _i32p), _p(rows, _i32p)),
           "permute")
    return off, rows


def ffn(x, w13, w2, expert_offsets, permuted_rows, k, round_intermediates=False):
    """Per expanded row: y = w2[e] . (silu(gate) * up).  Returns y float64 [T*k, H]
    in expanded-id order."""
    x = _c(x, np.uint16)
    w13 = _c(w13, np.uint16)
    w2 = _c(w2, np.uint16)
    off = _c(expert_offsets, np.int32)
    rows = _c(permuted_rows, np.int32)
    T, H = x.shape
    E, twoI, _ = w13.shape
    I = twoI // 2
    y = np.empty((T * k, H), np.float64)
    _check(_load().oracle_ffn(_p(x, _u16p), _p(w13, _u16p), _p(w2, _u16p), _p(off, _i32p),
                              _p(rows, _i32p), T, E, k, H, I, int(round_intermediates),
                              _p(y, _f64p)), "ffn")
    return y


def combine(y, topk_weights):
    """out[t] = sum_j w[t,j] * y[t*k+j] in j order.  Returns float64 [T,H]."""
    y = _c(y, np.float64)
    w = _c(topk_weights, np.float32)
    T, k = w.shape
    H = y.shape[1]
    out = np.empty((T, H), np.float64)
    _check(_load().oracle_combine(_p(y, _f64p), _p(w, _f32p), T, k, H, _p(out, _f64p)), "combine")
    return out


def forward(x, logits, w13, w2, k, round_intermediates=False):
    """Whole layer.  Returns dict(out float64 [T,H], topk_ids, topk_weights,
    expert_offsets, permuted_rows)."""
    x = _c(x, np.uint16)
    logits = _c(logits, np.float32)
    w13 = _c(w13, np.uint16)
    w2 = _c(w2, np.uint16)
    T, H = x.shape
    E = logits.shape[1]
    I = w13.shape[1] // 2
    out = np.empty((T, H), np.float64)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    off = np.empty(E + 1, np.int32)
    rows = np.empty(T * k, np.int32)
    _check(_load().oracle_forward(_p(x, _u16p), _p(logits, _f32p), _p(w13, _u16p), _p(w2, _u16p),
                                  T, E, k, H, I, int(round_intermediates), _p(out, _f64p),
                                  _p(ids, _i32p), _p(w, _f32p), _p(off, _i32p), _p(rows, _i32p)),
           "forward")
    return dict(out=out, topk_ids=ids, topk_weights=w, expert_offsets=off, permuted_rows=rows)


def forward_tokens(x, logits, w13_experts, w2_experts, k, tokens, I, round_intermediates=False):
    """Layer output of the listed tokens only.

    ``w13_experts`` / ``w2_experts`` are length-E sequences whose entry e is the
    expert's uint16 [2I,H] / [H,I] array, or None for an expert the listed tokens
    do not select.  Returns float64 [len(tokens), H]."""
    x = _c(x, np.uint16)
    logits = _c(logits, np.float32)
    T, H = x.shape
    E = logits.shape[1]
    keep = []
    w13p = (_u16p * E)()
    w2p = (_u16p * E)()
    for e in range(E):
        a, b = w13_experts[e], w2_experts[e]
        if a is not None and b is not None:
            a = _c(a, np.uint16)
            b = _c(b, np.uint16)
            if a.shape != (2 * I, H) or b.shape != (H, I):
                raise ValueError(f"expert {e}: bad weight shapes {a.shape} {b.shape}")
            keep += [a, b]
            w13p[e] = _p(a, _u16p)
            w2p[e] = _p(b, _u16p)
    toks = np.ascontiguousarray(np.asarray(tokens, np.int32))
    out = np.empty((len(toks), H), np.float64)
    rc = _load().oracle_forward_tokens(_p(x, _u16p), _p(logits, _f32p), w13p, w2p, T, E, k, H, I,
                                       int(round_intermediates), len(toks), _p(toks, _i32p),
                                       _p(out, _f64p))
    if rc == -3:
        raise ValueError("a listed token selects an expert whose weights were not given")
    _check(rc, "forward_tokens")
    del keep
    return out


def e4m3_to_float64(q):
    """E4M3 (E4M3FN) codes (uint8) -> float64 values, NaN for 0x7F / 0xFF."""
    q = _c(q, np.uint8)
    out = np.empty(q.shape, np.float64)
    _check(_load().oracle_e4m3_to_double(_p(q, _u8p), q.size, _p(out, _f64p)), "e4m3_to_double")
    return out


def round_to_bf16(v):
    """float64 values -> the nearest bf16 values (via fp32, round to nearest even at
    both steps), returned as float64: the rounding of the diagnostic
    ``round_intermediates`` mode."""
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.float64)
    _check(_load().oracle_round_to_bf16(_p(v, _f64p), v.size, _p(out, _f64p)), "round_to_bf16")
    return out


def forward_w8(x, logits, q13, s13, q2, s2, k):
    """Whole layer with FP8 weights: weight = e4m3(q) * per-row scale.  Returns the
    same dict as forward()."""
    x = _c(x, np.uint16)
    logits = _c(logits, np.float32)
    q13 = _c(q13, np.uint8)
    q2 = _c(q2, np.uint8)
    s13 = _c(s13, np.float32)
    s2 = _c(s2, np.float32)
    T, H = x.shape
    E = logits.shape[1]
    I = q13.shape[1] // 2
    if q13.shape != (E, 2 * I, H) or q2.shape != (E, H, I) or s13.shape != (E, 2 * I) \
            or s2.shape != (E, H):
        raise ValueError("FP8 weight or scale shapes do not match")
    out = np.empty((T, H), np.float64)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    off = np.empty(E + 1, np.int32)
    rows = np.empty(T * k, np.int32)
    _check(_load().oracle_forward_w8(_p(x, _u16p), _p(logits, _f32p), _p(q13, _u8p),
                                     _p(s13, _f32p), _p(q2, _u8p), _p(s2, _f32p), T, E, k, H, I,
                                     _p(out, _f64p), _p(ids, _i32p), _p(w, _f32p),
                                     _p(off, _i32p), _p(rows, _i32p)), "forward_w8")
    return dict(out=out, topk_ids=ids, topk_weights=w, expert_offsets=off, permuted_rows=rows)


def forward_tokens_w8(x, logits, experts, k, tokens, I):
    """Layer output of the listed tokens only, FP8 weights.  ``experts`` is a
    length-E sequence whose entry e is (q13 [2I,H] uint8, s13 [2I] f32,
    q2 [H,I] uint8, s2 [H] f32), or None for an expert the tokens do not select.
    Returns float64 [len(tokens), H]."""
    x = _c(x, np.uint16)
    logits = _c(logits, np.float32)
    T, H = x.shape
    E = logits.shape[1]
    keep = []
    q13p, s13p, q2p, s2p = (_u8p * E)(), (_f32p * E)(), (_u8p * E)(), (_f32p * E)()
    for e in range(E):
        if experts[e] is None:
            continue
        a, sa, b, sb = (_c(experts[e][0], np.uint8), _c(experts[e][1], np.float32),
                        _c(experts[e][2], np.uint8), _c(experts[e][3], np.float32))
        if a.shape != (2 * I, H) or sa.shape != (2 * I,) or b.shape != (H, I) or sb.shape != (H,):
            raise ValueError(f"expert {e}: bad FP8 weight or scale shapes")
        keep += [a, sa, b, sb]
        q13p[e], s13p[e], q2p[e], s2p[e] = _p(a, _u8p), _p(sa, _f32p), _p(b, _u8p), _p(sb, _f32p)
    toks = np.ascontiguousarray(np.asarray(tokens, np.int32))
    out = np.empty((len(toks), H), np.float64)
    rc = _load().oracle_forward_tokens_w8(_p(x, _u16p), _p(logits, _f32p), q13p, s13p, q2p, s2p,
                                          T, E, k, H, I, len(toks), _p(toks, _i32p),
                                          _p(out, _f64p))
    if rc == -3:
        raise ValueError("a listed token selects an expert whose weights were not given")
    _check(rc, "forward_tokens_w8")
    del keep
    return out
