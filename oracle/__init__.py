"""numpy-facing wrapper around the CPU oracle (liboracle.so).

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the
benchmark's CPU-baseline leg may import this package; the product path
(``int8_quantized_row_b200``) never does.  fp16 arrays are passed as
``np.float16`` and reinterpreted as their binary16 bit patterns; the oracle
converts them with its own code.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_lib = None


def lib(path=None):
    """Load (building first if needed) the oracle shared library.

    ``path`` selects another build of the same source, e.g. a copy with a
    planted mistake made by a test; the default is the committed source.
    """
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


def _bind(so):
    so.orc_half_to_float.argtypes = [ctypes.c_uint16]
    so.orc_half_to_float.restype = _F
    so.orc_double_to_half.argtypes = [ctypes.c_double]
    so.orc_double_to_half.restype = ctypes.c_uint16
    so.orc_rhaz.argtypes = [_F]
    so.orc_rhaz.restype = _F
    so.orc_quantize_weight_colwise.argtypes = [_P, _I, _I, _P, _P]
    so.orc_quantize_weight_colwise.restype = None
    so.orc_outlier_columns.argtypes = [_P, _I, _I, _F, _P, _P]
    so.orc_outlier_columns.restype = _I
    so.orc_outlier_hits.argtypes = [_P, _I, _I, _F, _P]
    so.orc_outlier_hits.restype = None
    so.orc_frac_8bit.argtypes = [_I, _I]
    so.orc_frac_8bit.restype = _F
    so.orc_quantize_rows.argtypes = [_P, _I, _I, _P, _P, _P]
    so.orc_quantize_rows.restype = None
    so.orc_int8_gemm.argtypes = [_P, _P, _I, _I, _I, _P, _I, _P]
    so.orc_int8_gemm.restype = _I
    so.orc_dequantize_weight.argtypes = [_P, _P, _I, _I, _P]
    so.orc_dequantize_weight.restype = None
    so.orc_mixed_linear.argtypes = [_P, _I, _I, _P, _P, _P, _I, _F, _P, _I, _P, _P, _P]
    so.orc_mixed_linear.restype = _I
    so.orc_int4_quantize_groupwise.argtypes = [_P, _I, _I, _I, _P, _P, _P]
    so.orc_int4_quantize_groupwise.restype = None
    so.orc_int4_dequantize.argtypes = [_P, _P, _P, _I, _I, _I, _P]
    so.orc_int4_dequantize.restype = None
    so.orc_int4_linear.argtypes = [_P, _I, _I, _P, _P, _P, _I, _I, _P, _I, _P, _P]
    so.orc_int4_linear.restype = None
    return so


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


class Oracle:
    """The oracle's functions over numpy arrays, bound to one library build."""

    def __init__(self, so=None):
        self.so = so if so is not None else lib()

    # --- scalar helpers (exposed for the pins) ---
    def half_to_float(self, bits):
        return self.so.orc_half_to_float(int(bits))

    def double_to_half(self, x):
        return self.so.orc_double_to_half(float(x))

    def rhaz(self, v):
        return self.so.orc_rhaz(float(v))

    # --- a0 ---
    def quantize_weight_colwise(self, W16):
        W16 = _c(W16, np.float16)
        K, N = W16.shape
        Wq = np.empty((K, N), np.int8)
        sW = np.empty(N, np.float32)
        self.so.orc_quantize_weight_colwise(_ptr(W16), K, N, _ptr(Wq), _ptr(sW))
        return Wq, sW

    # --- a1 ---
    def outlier_columns(self, X, alpha):
        X = _c(X, np.float16)
        T, K = X.shape
        is_out = np.zeros(K, np.uint8)
        idx = np.zeros(K, np.int32)
        cnt = self.so.orc_outlier_columns(_ptr(X), T, K, float(alpha), _ptr(is_out), _ptr(idx))
        return is_out.astype(bool), idx[:cnt].copy()

    def outlier_hits(self, X, alpha):
        X = _c(X, np.float16)
        T, K = X.shape
        hits = np.zeros(K, np.int32)
        self.so.orc_outlier_hits(_ptr(X), T, K, float(alpha), _ptr(hits))
        return hits

    def frac_8bit(self, count, K):
        return self.so.orc_frac_8bit(int(count), int(K))

    # --- a2 ---
    def quantize_rows(self, X, is_outlier):
        X = _c(X, np.float16)
        T, K = X.shape
        m = _c(np.asarray(is_outlier, dtype=np.uint8), np.uint8)
        Xq = np.empty((T, K), np.int8)
        sX = np.empty(T, np.float32)
        self.so.orc_quantize_rows(_ptr(X), T, K, _ptr(m), _ptr(Xq), _ptr(sX))
        return Xq, sX

    # --- a4 ---
    def int8_gemm(self, Xq, Wq, rows=None):
        Xq = _c(Xq, np.int8)
        Wq = _c(Wq, np.int8)
        T, K = Xq.shape
        N = Wq.shape[1]
        rows = _c(np.arange(T) if rows is None else rows, np.int32)
        acc = np.empty((len(rows), N), np.int32)
        rc = self.so.orc_int8_gemm(_ptr(Xq), _ptr(Wq), T, K, N, _ptr(rows), len(rows), _ptr(acc))
        if rc != 0:
            raise ArithmeticError("oracle: an int32 accumulator disagreed with its int64 sum")
        return acc

    # --- a1..a6 ---
    def dequantize_weight(self, Wq, sW):
        """fp16 [K,N]: binary16 RNE of q * fl32(sW/127), the Wq-only variant's outlier rows."""
        Wq = _c(Wq, np.int8)
        sW = _c(sW, np.float32)
        K, N = Wq.shape
        out = np.empty((K, N), np.uint16)
        self.so.orc_dequantize_weight(_ptr(Wq), _ptr(sW), K, N, _ptr(out))
        return out.view(np.float16)

    def mixed_linear(self, X, Wq, sW, W16, alpha, rows=None):
        """Returns (Y fp16 [r,N], Ypre float64 [r,N], acc int32 [r,N], n_outliers).
        W16 None: the Wq-only variant (the outlier rows of W are dequantised from Wq)."""
        X = _c(X, np.float16)
        Wq = _c(Wq, np.int8)
        sW = _c(sW, np.float32)
        W16 = None if W16 is None else _c(W16, np.float16)
        T, K = X.shape
        N = Wq.shape[1]
        rows = _c(np.arange(T) if rows is None else rows, np.int32)
        R = len(rows)
        Y = np.empty((R, N), np.uint16)
        Ypre = np.empty((R, N), np.float64)
        acc = np.empty((R, N), np.int32)
        cnt = self.so.orc_mixed_linear(_ptr(X), T, K, _ptr(Wq), _ptr(sW), None if W16 is None else _ptr(W16), N,
                                       float(alpha), _ptr(rows), R, _ptr(Y), _ptr(Ypre), _ptr(acc))
        if cnt < 0:
            raise ArithmeticError("oracle: an int32 accumulator disagreed with its int64 sum")
        return Y.view(np.float16), Ypre, acc, cnt

    # --- the group-wise 4-bit weight codec (FlexGen summary) ---
    def int4_quantize_groupwise(self, W16, G=64):
        """W16 fp16 [K,N] -> (codes uint8 [K,N] in 0..15, scale fp16 [K/G,N], lo fp16 [K/G,N])."""
        W16 = _c(W16, np.float16)
        K, N = W16.shape
        if K % G:
            raise ValueError("K must be a multiple of the group size")
        codes = np.empty((K, N), np.uint8)
        scale = np.empty((K // G, N), np.uint16)
        lo = np.empty((K // G, N), np.uint16)
        self.so.orc_int4_quantize_groupwise(_ptr(W16), K, N, G, _ptr(codes), _ptr(scale), _ptr(lo))
        return codes, scale.view(np.float16), lo.view(np.float16)

    def int4_dequantize(self, codes, scale, lo):
        """fp16 [K,N]: the decoded 4-bit weight, binary16 of q*s + lo."""
        codes = _c(codes, np.uint8)
        scale = _c(scale, np.float16)
        lo = _c(lo, np.float16)
        K, N = codes.shape
        G = K // scale.shape[0]
        out = np.empty((K, N), np.uint16)
        self.so.orc_int4_dequantize(_ptr(codes), _ptr(scale), _ptr(lo), K, N, G, _ptr(out))
        return out.view(np.float16)

    def int4_linear(self, X, codes, scale, lo, rows=None):
        """(Y fp16 [r,N], Ypre float64 [r,N]) = X times the decoded 4-bit weight."""
        X = _c(X, np.float16)
        codes = _c(codes, np.uint8)
        scale = _c(scale, np.float16)
        lo = _c(lo, np.float16)
        T, K = X.shape
        N = codes.shape[1]
        G = K // scale.shape[0]
        rows = _c(np.arange(T) if rows is None else rows, np.int32)
        Y = np.empty((len(rows), N), np.uint16)
        Ypre = np.empty((len(rows), N), np.float64)
        self.so.orc_int4_linear(_ptr(X), T, K, _ptr(codes), _ptr(scale), _ptr(lo), N, G, _ptr(rows), len(rows),
                                _ptr(Y), _ptr(Ypre))
        return Y.view(np.float16), Ypre


def default():
    return Oracle()
