"""CPU oracle for the LLM.int8() linear layer (test infrastructure only).

Only the test-suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package. The product path (the CUDA library and
its Python binding) never does, and this package never imports the product.

The arithmetic lives in ``llmint8_oracle.c`` (plain C loops, int64 / fp64,
fp32 where a quantised code is decided). This module only marshals numpy
arrays into that library with ctypes.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from .build_oracle import build_oracle, library_path

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        build_oracle()
    lib = ctypes.CDLL(path)
    i64, i32, f32 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    vp = ctypes.c_void_p
    lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_half_to_double.restype = ctypes.c_double
    lib.oracle_double_to_half.argtypes = [ctypes.c_double]
    lib.oracle_double_to_half.restype = ctypes.c_uint16
    lib.oracle_quantize_value.argtypes = [f32, f32]
    lib.oracle_quantize_value.restype = ctypes.c_int
    lib.oracle_prepare_weight.argtypes = [vp, i64, i64, vp, vp]
    lib.oracle_prepare_weight_mode.argtypes = [vp, i64, i64, ctypes.c_int, vp, vp]
    lib.oracle_quantize_rows_mode.argtypes = [vp, i64, i64, vp, vp, i64,
                                              ctypes.c_int, vp, vp]
    lib.oracle_detect_outliers.argtypes = [vp, i64, i64, f32, vp, vp, vp]
    lib.oracle_quantize_rows.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp]
    lib.oracle_int8_gemm.argtypes = [vp, i64, i64, vp, i64, vp, i64, vp]
    lib.oracle_outlier_weights.argtypes = [vp, vp, i64, i64, vp, i32, vp]
    lib.oracle_matmul.argtypes = [vp, i64, i64, vp, vp, i64, vp, f32,
                                  ctypes.c_int, vp, i64, vp, i64, vp, vp]
    lib.oracle_num_threads.argtypes = []
    for fn in ("oracle_prepare_weight", "oracle_prepare_weight_mode",
               "oracle_detect_outliers", "oracle_quantize_rows",
               "oracle_quantize_rows_mode", "oracle_int8_gemm",
               "oracle_outlier_weights", "oracle_matmul",
               "oracle_num_threads"):
        getattr(lib, fn).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _bits(x: np.ndarray) -> np.ndarray:
    """binary16 array -> contiguous uint16 view of its bit patterns."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        return x.view(np.uint16)
    assert x.dtype == np.uint16
    return x


def _check(rc: int, what: str):
    if rc == -2:
        raise OverflowError(f"{what}: int32 accumulator overflow")
    if rc != 0:
        raise ValueError(f"{what}: oracle returned {rc}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def half_to_double(bits: int) -> float:
    return float(_load().oracle_half_to_double(int(bits)))


def double_to_half(v: float) -> int:
    return int(_load().oracle_double_to_half(float(v)))


def quantize_value(x: float, a: float) -> int:
    return int(_load().oracle_quantize_value(float(x), float(a)))


def prepare_weight(W: np.ndarray, tensor: bool = False):
    """W float16 [h,o] -> (Wq int8 [o,h], aw float32 [o]).

    tensor: one absmax constant for the whole weight (every aw[j] equal)."""
    Wb = _bits(W)
    h, o = Wb.shape
    Wq = np.empty((o, h), dtype=np.int8)
    aw = np.empty((o,), dtype=np.float32)
    _check(_load().oracle_prepare_weight_mode(_ptr(Wb), h, o, int(bool(tensor)),
                                              _ptr(Wq), _ptr(aw)),
           "prepare_weight")
    return Wq, aw


def detect_outliers(X: np.ndarray, alpha: float):
    """X float16 [s,h] -> (flags uint8 [h], idx int32 [n], n)."""
    Xb = _bits(X)
    s, h = Xb.shape
    flags = np.zeros((h,), dtype=np.uint8)
    idx = np.zeros((max(h, 1),), dtype=np.int32)
    n = np.zeros((1,), dtype=np.int32)
    _check(_load().oracle_detect_outliers(_ptr(Xb), s, h, alpha, _ptr(flags),
                                          _ptr(idx), _ptr(n)),
           "detect_outliers")
    n = int(n[0])
    return flags, idx[:n].copy(), n


def quantize_rows(X: np.ndarray, flags: np.ndarray,
                  rows: Optional[Sequence[int]] = None, tensor: bool = False):
    """Row scales and codes for the given rows -> (Xq int8 [r,h], ax f32 [r]).

    tensor: one absmax constant for all of X (every ax[r] equal)."""
    Xb = _bits(X)
    s, h = Xb.shape
    flags = np.ascontiguousarray(flags, dtype=np.uint8)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = s if r is None else r.shape[0]
    Xq = np.empty((nr, h), dtype=np.int8)
    ax = np.empty((nr,), dtype=np.float32)
    _check(_load().oracle_quantize_rows_mode(_ptr(Xb), s, h, _ptr(flags), _ptr(r),
                                             nr, int(bool(tensor)), _ptr(Xq), _ptr(ax)),
           "quantize_rows")
    return Xq, ax


def int8_gemm(Xq: np.ndarray, Wq: np.ndarray,
              cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """Exact Ci = Xq . Wq^T for Xq [r,h], Wq [o,h] -> int32 [r, ncols]."""
    Xq = np.ascontiguousarray(Xq, dtype=np.int8)
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    nr, h = Xq.shape
    o = Wq.shape[0]
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nc = o if c is None else c.shape[0]
    Ci = np.empty((nr, nc), dtype=np.int32)
    _check(_load().oracle_int8_gemm(_ptr(Xq), nr, h, _ptr(Wq), o, _ptr(c), nc,
                                    _ptr(Ci)), "int8_gemm")
    return Ci


def outlier_weights(Wq: np.ndarray, aw: np.ndarray,
                    idx: np.ndarray) -> np.ndarray:
    """fp16 outlier rows of W recovered from the int8 weight -> [n, o]."""
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    aw = np.ascontiguousarray(aw, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    o, h = Wq.shape
    n = idx.shape[0]
    WO = np.zeros((max(n, 0), o), dtype=np.uint16)
    _check(_load().oracle_outlier_weights(_ptr(Wq), _ptr(aw), h, o, _ptr(idx),
                                          n, _ptr(WO)), "outlier_weights")
    return WO.view(np.float16)


def matmul(X: np.ndarray, Wq: np.ndarray, aw: np.ndarray, alpha: float,
           rows: Optional[Sequence[int]] = None,
           cols: Optional[Sequence[int]] = None, want_ci: bool = False,
           W16: Optional[np.ndarray] = None, x_tensor: bool = False):
    """Full LLM.int8() output (float16) for the chosen rows x cols.

    With ``W16`` (the fp16 weight [h, o]) the outlier rows of W are its own
    fp16 values; without it they are recovered from Wq and aw. With
    ``x_tensor`` X is quantised with one constant for the whole tensor (the
    tensor-wise baseline; pair it with a ``prepare_weight(W, tensor=True)``
    weight for tensor-wise W). Returns out
    [nr, nc] float16, plus Ci int32 of the same shape when ``want_ci``.
    """
    Xb = _bits(X)
    s, h = Xb.shape
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    aw = np.ascontiguousarray(aw, dtype=np.float32)
    o = Wq.shape[0]
    assert Wq.shape[1] == h
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nr = s if r is None else r.shape[0]
    nc = o if c is None else c.shape[0]
    out = np.empty((nr, nc), dtype=np.uint16)
    Ci = np.empty((nr, nc), dtype=np.int32) if want_ci else None
    w16 = None
    if W16 is not None:
        w16 = _bits(W16)
        assert w16.shape == (h, o)
    _check(_load().oracle_matmul(_ptr(Xb), s, h, _ptr(Wq), _ptr(aw), o, _ptr(w16),
                                 alpha, int(bool(x_tensor)), _ptr(r), nr, _ptr(c), nc,
                                 _ptr(out), _ptr(Ci)),
           "matmul")
    out = out.view(np.float16)
    return (out, Ci) if want_ci else out
