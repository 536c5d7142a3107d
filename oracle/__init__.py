"""CPU oracle for MoE expert-parallel dispatch / combine.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product path never does.
It shares no code with the CUDA library (see ep_oracle.c for what it
computes, the readings it takes, and where each step is stated).

Thin numpy wrappers over the C functions; all arrays are host numpy arrays.
bf16 values are carried as their uint16 bit patterns, e4m3 as uint8.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

X_BF16, X_FP8_PREQUANT, X_BF16_QUANT_FP8, X_BF16_QUANT_NVFP4 = 0, 1, 2, 3


def lib():
    """The oracle library.  EP_ORACLE_LIB names another build of it (the
    mutation tests load deliberately broken copies that way)."""
    global _lib
    if _lib is None:
        path = os.environ.get("EP_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, u32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_float
        L.oracle_f32_to_bf16_n.argtypes = [P, P, i64]
        L.oracle_f32_to_bf16_n.restype = None
        L.oracle_e4m3_encode_n.argtypes = [P, P, i64]
        L.oracle_e4m3_encode_n.restype = None
        L.oracle_quantize_rows.argtypes = [i64, i32, P, P, P]
        L.oracle_quantize_rows.restype = None
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_decode.restype = ctypes.c_float
        L.oracle_e2m1_encode_n.argtypes = [P, P, i64]
        L.oracle_e2m1_encode_n.restype = None
        L.oracle_nvfp4_rows.argtypes = [i64, i32, P, P, P]
        L.oracle_nvfp4_rows.restype = None
        L.oracle_max_recv_rows.argtypes = [i32, i32, i32, i32]
        L.oracle_max_recv_rows.restype = i32
        L.oracle_layout.argtypes = [i32, i32, i32, i32, i32, P, P, i32, P, P, P, P, P, P, P]
        L.oracle_layout.restype = u32
        L.oracle_dispatch.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P]
        L.oracle_dispatch.restype = None
        L.oracle_combine.argtypes = [i32, i32, i32, P, P, P, P, P, P]
        L.oracle_combine.restype = None
        L.oracle_combine_fp8.argtypes = [i32, i32, i32, P, P, P, P, P]
        L.oracle_combine_fp8.restype = None
        L.oracle_combine_backward.argtypes = [i32, i32, i32, i32, P, P, P, P, P, P, P]
        L.oracle_combine_backward.restype = None
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ formats

def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bits -> float32 (exact)."""
    b = _c(b, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().oracle_f32_to_bf16_n(_p(v), _p(out), v.size)
    return out


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_n(_p(v), _p(out), v.size)
    return out


def e4m3_decode(c: np.ndarray) -> np.ndarray:
    c = _c(c, np.uint8)
    L = lib()
    table = np.array([L.oracle_e4m3_decode(i) for i in range(256)], dtype=np.float32)
    return table[c]


def quantize_rows(x_bf16: np.ndarray):
    """bf16 bits [rows, H] -> (e4m3 [rows, H] uint8, scales [rows, H/128] f32)."""
    x = _c(x_bf16, np.uint16)
    rows, H = x.shape
    q = np.empty((rows, H), dtype=np.uint8)
    s = np.empty((rows, H // 128), dtype=np.float32)
    lib().oracle_quantize_rows(rows, H, _p(x), _p(q), _p(s))
    return q, s


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e2m1_encode_n(_p(v), _p(out), v.size)
    return out


def e2m1_decode(c: np.ndarray) -> np.ndarray:
    c = _c(c, np.uint8)
    L = lib()
    table = np.array([L.oracle_e2m1_decode(i) for i in range(16)], dtype=np.float32)
    return table[c & 0xF]


def nvfp4_rows(x_bf16: np.ndarray):
    """bf16 bits [rows, H] -> (packed e2m1 [rows, H/2] uint8, e4m3 scales [rows, H/16] uint8)."""
    x = _c(x_bf16, np.uint16)
    rows, H = x.shape
    q = np.empty((rows, H // 2), dtype=np.uint8)
    s = np.empty((rows, H // 16), dtype=np.uint8)
    lib().oracle_nvfp4_rows(rows, H, _p(x), _p(q), _p(s))
    return q, s


# ------------------------------------------------------------------- layout

def max_recv_rows(T: int, k: int, E: int, align: int) -> int:
    return int(lib().oracle_max_recv_rows(T, k, E, align))


def layout(topk_idx: np.ndarray, E: int, S: int, align: int, topk_weights=None,
           max_rows: int | None = None) -> dict:
    idx = _c(topk_idx, np.int64)
    T, k = idx.shape
    cap = max_recv_rows(T, k, E, align) if max_rows is None else max_rows
    w = None if topk_weights is None else _c(topk_weights, np.float32)
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    seg = np.zeros(S, np.int32)
    slot_map = np.zeros(T * k, np.int32)
    recv_src = np.full(max(cap, 1), -7, np.int32)          # -7: never written
    recv_idx = np.full(max(cap, 1), -7, np.int32)
    recv_w = np.full(max(cap, 1), np.nan, np.float32)
    flags = lib().oracle_layout(T, k, E, S, align, _p(idx), _p(w), cap, _p(counts),
                                _p(offsets), _p(seg), _p(slot_map), _p(recv_src), _p(recv_idx),
                                _p(recv_w))
    return {"T": T, "k": k, "E": E, "S": S, "align": align, "max_rows": cap,
            "counts": counts, "offsets": offsets, "seg_tokens": seg, "slot_map": slot_map,
            "recv_src": recv_src[:cap], "recv_topk_idx": recv_idx[:cap],
            "recv_topk_weights": recv_w[:cap], "R": int(offsets[E]), "flags": int(flags)}


# ----------------------------------------------------------------- dispatch

UNWRITTEN = 0x5A  # every byte of the dispatch outputs starts as this


def dispatch(lay: dict, x: np.ndarray, mode: int, x_scales=None):
    """Returns (recv_x [max_rows, H], recv_scales [max_rows, H/128] or None).
    Every output byte starts as UNWRITTEN, so rows the oracle does not
    write (rows >= R) keep it and a missing write shows."""
    T, k, cap, R = lay["T"], lay["k"], lay["max_rows"], lay["R"]
    if mode == X_BF16:
        x = _c(x, np.uint16)
        recv = np.full((cap, x.shape[1]), UNWRITTEN * 0x0101, np.uint16)
        scales = None
    elif mode == X_BF16_QUANT_NVFP4:
        x = _c(x, np.uint16)
        recv = np.full((cap, x.shape[1] // 2), UNWRITTEN, np.uint8)
        scales = np.full((cap, x.shape[1] // 16), UNWRITTEN, np.uint8)
    else:
        x = _c(x, np.uint8 if mode == X_FP8_PREQUANT else np.uint16)
        recv = np.full((cap, x.shape[1]), UNWRITTEN, np.uint8)
        scales = np.full((cap, x.shape[1] // 128), UNWRITTEN * 0x01010101, np.uint32).view(np.float32)
    H = x.shape[1]
    xs = None if x_scales is None else _c(x_scales, np.float32)
    lib().oracle_dispatch(mode, T, k, H, R, _p(lay["slot_map"]), _p(lay["recv_src"]), _p(x),
                          _p(xs), _p(recv), _p(scales))
    return recv, scales


# ------------------------------------------------------------------ combine

def combine(slot_map: np.ndarray, T: int, k: int, y: np.ndarray, weights=None,
            recv_weights_in=None, want_out_weights: bool = False):
    """Returns (out bf16 bits [T, H], out_weights [T, k] or None)."""
    y = _c(y, np.uint16)
    H = y.shape[1]
    sm = _c(slot_map, np.int32)
    w = None if weights is None else _c(weights, np.float32)
    rw = None if recv_weights_in is None else _c(recv_weights_in, np.float32)
    out = np.empty((T, H), np.uint16)
    ow = np.empty((T, k), np.float32) if want_out_weights else None
    lib().oracle_combine(T, k, H, _p(sm), _p(y), _p(w), _p(rw), _p(ow), _p(out))
    return out, ow


def combine_fp8(slot_map: np.ndarray, T: int, k: int, yq: np.ndarray, ys: np.ndarray, weights=None):
    """FP8 expert outputs (e4m3 codes [rows, H], f32 scales [rows, H/128])
    -> out bf16 bits [T, H]."""
    q = _c(yq, np.uint8)
    H = q.shape[1]
    s = _c(ys, np.float32)
    sm = _c(slot_map, np.int32)
    w = None if weights is None else _c(weights, np.float32)
    out = np.empty((T, H), np.uint16)
    lib().oracle_combine_fp8(T, k, H, _p(sm), _p(q), _p(s), _p(w), _p(out))
    return out


def combine_backward(lay: dict, grad_out: np.ndarray, y: np.ndarray, weights: np.ndarray):
    """Backward of the weighted combine.  Returns (grad_y bf16 bits
    [max_rows, H] -- rows >= R keep UNWRITTEN --, grad_w float64 [T, k])."""
    T, k, cap, R = lay["T"], lay["k"], lay["max_rows"], lay["R"]
    g = _c(grad_out, np.uint16)
    yy = _c(y, np.uint16)
    w = _c(weights, np.float32)
    H = g.shape[1]
    grad_y = np.full((cap, H), UNWRITTEN * 0x0101, np.uint16)
    grad_w = np.empty((T, k), np.float64)
    lib().oracle_combine_backward(T, k, H, R, _p(lay["slot_map"]), _p(lay["recv_src"]), _p(g), _p(yy),
                                  _p(w), _p(grad_y), _p(grad_w))
    return grad_y, grad_w
