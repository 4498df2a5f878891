"""LLM.int8() mixed-precision linear layer for B200 (sm_100a).

Thin Python binding over the C ABI in ``include/int8row.h`` (``libint8row.so``
beside this file, built by ``python -m int8_quantized_row_b200.build``).  The
functions carry the C names; they only marshal arguments: every step of the
computation runs in the library's CUDA kernels.  PyTorch provides device
memory and the current stream.  There is no CPU fallback: without the
compiled library, or without a CUDA device, every call raises.
"""
import ctypes
import os

__all__ = [
    "lib", "I8RError",
    "int8_quantize_weight_colwise", "int8_mixed_linear_workspace_size", "int8_mixed_linear",
    "int8_mixed_linear_wq_workspace_size", "int8_mixed_linear_wq_max_outliers", "int8_mixed_linear_wq",
    "int8_outlier_stats_workspace_size", "int8_outlier_stats", "int8_quantize_activation",
    "int8_gemm_i8_s32", "int8_read_and_clear_device_status", "int8_status_string",
    "int8_selftest_wait_timeout",
    "int8_time_next_gemm", "int8_kernel_launch_count", "LIB_PATH",
    "int4_packed_code_bytes", "int4_packed_scale_bytes", "int4_quantize_weight_groupwise",
    "int4_dequantize_weight", "int4_linear_workspace_size", "int4_linear", "int4_debug_set_product_path",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libint8row.so")
DECODE_MAX_T = 128
INT4_MAX_T = 64

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t

_lib = None


class I8RError(RuntimeError):
    """A non-zero i8r_status returned by the library."""

    def __init__(self, fn, status):
        self.status = status
        msg = _lib.int8_status_string(status).decode() if _lib else str(status)
        extra = f" (cuda error {_lib.int8_last_cuda_error()})" if _lib and status == 5 else ""
        super().__init__(f"{fn}: {msg}{extra}")


def lib():
    """The loaded C library (ctypes.CDLL) with argument types declared."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m int8_quantized_row_b200.build`")
    so = ctypes.CDLL(LIB_PATH)
    so.int8_quantize_weight_colwise.argtypes = [_P, _I, _I, _P, _P, _P]
    so.int8_mixed_linear_workspace_size.argtypes = [_I, _I, _I]
    so.int8_mixed_linear_workspace_size.restype = _Z
    so.int8_mixed_linear.argtypes = [_P, _I, _I, _P, _P, _P, _I, _F, _P, _P, _Z, _P]
    so.int8_mixed_linear_wq_workspace_size.argtypes = [_I, _I, _I]
    so.int8_mixed_linear_wq_workspace_size.restype = _Z
    so.int8_mixed_linear_wq_max_outliers.argtypes = [_I]
    so.int8_mixed_linear_wq_max_outliers.restype = _I
    so.int8_mixed_linear_wq.argtypes = [_P, _I, _I, _P, _P, _I, _F, _P, _P, _Z, _P]
    so.int8_mixed_linear_chain_workspace_size.argtypes = [_I, _P]
    so.int8_mixed_linear_chain_workspace_size.restype = _Z
    so.int8_mixed_linear_chain.argtypes = [_I, _P, _P, _Z, _P]
    so.int8_debug_set_activation_path.argtypes = [_I]
    so.int8_debug_set_activation_path.restype = None
    so.int4_debug_set_product_path.argtypes = [_I]
    so.int4_debug_set_product_path.restype = None
    so.int8_outlier_stats_workspace_size.argtypes = [_I]
    so.int8_outlier_stats_workspace_size.restype = _Z
    so.int8_outlier_stats.argtypes = [_P, _I, _I, _F, _P, _P, _P, _P, _P, _Z, _P]
    so.int8_quantize_activation_workspace_size.argtypes = [_I, _I]
    so.int8_quantize_activation_workspace_size.restype = _Z
    so.int8_quantize_activation.argtypes = [_P, _I, _I, _F, _P, _P, _P, _P, _P, _P, _P, _Z, _P]
    so.int8_gemm_i8_s32_workspace_size.argtypes = [_I, _I, _I]
    so.int8_gemm_i8_s32_workspace_size.restype = _Z
    so.int8_gemm_i8_s32.argtypes = [_P, _I, _I, _P, _I, _P, _P, _Z, _P]
    so.int8_read_and_clear_device_status.argtypes = [ctypes.POINTER(ctypes.c_int), _P]
    so.int8_selftest_wait_timeout.argtypes = [_I, _P]
    so.int8_selftest_wait_timeout.restype = _I
    so.int8_status_string.argtypes = [_I]
    so.int8_status_string.restype = ctypes.c_char_p
    so.int8_last_cuda_error.restype = _I
    so.int8_time_next_gemm.argtypes = [_P, _P]
    so.int8_time_next_gemm.restype = None
    so.int8_kernel_launch_count.restype = ctypes.c_uint64
    so.int4_packed_code_bytes.argtypes = [_I, _I]
    so.int4_packed_code_bytes.restype = _Z
    so.int4_packed_scale_bytes.argtypes = [_I, _I]
    so.int4_packed_scale_bytes.restype = _Z
    so.int4_quantize_weight_groupwise.argtypes = [_P, _I, _I, _P, _P, _P]
    so.int4_dequantize_weight.argtypes = [_P, _P, _I, _I, _P, _P]
    so.int4_linear_workspace_size.argtypes = [_I, _I, _I]
    so.int4_linear_workspace_size.restype = _Z
    so.int4_linear.argtypes = [_P, _I, _I, _P, _P, _I, _P, _P, _Z, _P]
    for name in ("int8_quantize_weight_colwise", "int8_mixed_linear", "int8_outlier_stats",
                 "int8_quantize_activation", "int8_gemm_i8_s32", "int8_read_and_clear_device_status",
                 "int4_quantize_weight_groupwise", "int4_dequantize_weight", "int4_linear"):
        getattr(so, name).restype = _I
    _lib = so
    return so


def _check(fn, status):
    if status != 0:
        raise I8RError(fn, status)


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name, ndim=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def int8_quantize_weight_colwise(W16, Wq=None, sW=None, stream=None):
    """W16 fp16 [K,N] -> (Wq int8 [K,N], sW fp32 [N])."""
    import torch
    K, N = W16.shape
    Wq = torch.empty((K, N), dtype=torch.int8, device=W16.device) if Wq is None else Wq
    sW = torch.empty((N,), dtype=torch.float32, device=W16.device) if sW is None else sW
    _check("int8_quantize_weight_colwise", lib().int8_quantize_weight_colwise(
        _dev(W16, torch.float16, "W16", 2), K, N, _dev(Wq, torch.int8, "Wq"), _dev(sW, torch.float32, "sW"),
        _stream(stream)))
    return Wq, sW


def int8_mixed_linear_workspace_size(T, K, N):
    return int(lib().int8_mixed_linear_workspace_size(int(T), int(K), int(N)))


def workspace(T, K, N, device="cuda"):
    """A device buffer large enough for int8_mixed_linear(T, K, N)."""
    import torch
    return torch.empty(max(1, int8_mixed_linear_workspace_size(T, K, N)), dtype=torch.uint8, device=device)


def int8_mixed_linear(X, Wq, sW, W16, alpha=6.0, Y=None, workspace_buf=None, stream=None):
    """Y fp16 [T,N] = LLM.int8() linear of X fp16 [T,K] with (Wq, sW, W16)."""
    import torch
    T, K = X.shape
    N = Wq.shape[1]
    Y = torch.empty((T, N), dtype=torch.float16, device=X.device) if Y is None else Y
    ws = workspace(T, K, N, X.device) if workspace_buf is None else workspace_buf
    _check("int8_mixed_linear", lib().int8_mixed_linear(
        _dev(X, torch.float16, "X", 2), T, K, _dev(Wq, torch.int8, "Wq", 2), _dev(sW, torch.float32, "sW"),
        _dev(W16, torch.float16, "W16", 2), N, float(alpha), _dev(Y, torch.float16, "Y"),
        ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(), _stream(stream)))
    return Y


def int8_mixed_linear_wq_workspace_size(T, K, N):
    return int(lib().int8_mixed_linear_wq_workspace_size(int(T), int(K), int(N)))


def int8_mixed_linear_wq_max_outliers(K):
    return int(lib().int8_mixed_linear_wq_max_outliers(int(K)))


def int8_mixed_linear_wq(X, Wq, sW, alpha=6.0, Y=None, workspace_buf=None, stream=None):
    """Y fp16 [T,N] = the Wq-only variant: the outlier rows of W are dequantised from (Wq, sW)."""
    import torch
    T, K = X.shape
    N = Wq.shape[1]
    Y = torch.empty((T, N), dtype=torch.float16, device=X.device) if Y is None else Y
    if workspace_buf is None:
        workspace_buf = torch.empty(max(1, int8_mixed_linear_wq_workspace_size(T, K, N)), dtype=torch.uint8,
                                    device=X.device)
    ws = workspace_buf
    _check("int8_mixed_linear_wq", lib().int8_mixed_linear_wq(
        _dev(X, torch.float16, "X", 2), T, K, _dev(Wq, torch.int8, "Wq", 2), _dev(sW, torch.float32, "sW"),
        N, float(alpha), _dev(Y, torch.float16, "Y"),
        ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(), _stream(stream)))
    return Y


class I8rLayer(ctypes.Structure):
    """One layer of int8_mixed_linear_chain (the C struct i8r_layer)."""
    _fields_ = [("X", _P), ("T", _I), ("K", _I), ("Wq", _P), ("sW", _P), ("W16", _P), ("N", _I),
                ("alpha", _F), ("Y", _P)]


def _chain_layers(layers):
    import torch
    descs, outs = [], []
    for X, Wq, sW, W16, alpha, Y in layers:
        T, K = X.shape
        N = Wq.shape[1]
        Y = torch.empty((T, N), dtype=torch.float16, device=X.device) if Y is None else Y
        w16 = _dev(W16, torch.float16, "W16", 2) if W16 is not None else _P()
        descs.append(I8rLayer(_dev(X, torch.float16, "X", 2), T, K, _dev(Wq, torch.int8, "Wq", 2),
                              _dev(sW, torch.float32, "sW"), w16, N, float(alpha), _dev(Y, torch.float16, "Y")))
        outs.append(Y)
    return (I8rLayer * max(1, len(descs)))(*descs), outs


def int8_mixed_linear_chain_workspace_size(layers):
    arr, _ = _chain_layers(layers)
    return int(lib().int8_mixed_linear_chain_workspace_size(len(layers), ctypes.cast(arr, _P)))


def int8_mixed_linear_chain(layers, workspace_buf=None, stream=None):
    """Run layers in order on one stream with one workspace.  layers: a list of
    (X, Wq, sW, W16 or None, alpha, Y or None); returns the list of Y."""
    import torch
    arr, outs = _chain_layers(layers)
    if workspace_buf is None:
        need = int(lib().int8_mixed_linear_chain_workspace_size(len(layers), ctypes.cast(arr, _P)))
        dev = layers[0][0].device if layers else "cuda"
        workspace_buf = torch.empty(max(1, need), dtype=torch.uint8, device=dev)
    _check("int8_mixed_linear_chain", lib().int8_mixed_linear_chain(
        len(layers), ctypes.cast(arr, _P), ctypes.c_void_p(workspace_buf.data_ptr()),
        workspace_buf.numel() * workspace_buf.element_size(), _stream(stream)))
    return outs


def int8_outlier_stats_workspace_size(K):
    return int(lib().int8_outlier_stats_workspace_size(int(K)))


def int8_outlier_stats(X, alpha=6.0, with_hits=True, stream=None):
    """-> (count int32 [1], col_idx int32 [K], col_hit_count int32 [K] or None, frac_8bit fp32 [1])."""
    import torch
    T, K = X.shape
    dev = X.device
    count = torch.zeros(1, dtype=torch.int32, device=dev)
    idx = torch.full((K,), -1, dtype=torch.int32, device=dev)
    hits = torch.empty(K, dtype=torch.int32, device=dev) if with_hits else None
    frac = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, int8_outlier_stats_workspace_size(K)), dtype=torch.uint8, device=dev)
    _check("int8_outlier_stats", lib().int8_outlier_stats(
        _dev(X, torch.float16, "X", 2), T, K, float(alpha), _dev(count, torch.int32, "count"),
        _dev(idx, torch.int32, "idx"), _dev(hits, torch.int32, "hits") if hits is not None else None,
        _dev(frac, torch.float32, "frac"), ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)))
    return count, idx, hits, frac


def int8_debug_set_activation_path(mode):
    """1 (default): the one cooperative activation kernel for 8 <= T <= 128 when X fits in
    shared memory; 2: that kernel whenever X fits; 0: scan + quantiser."""
    lib().int8_debug_set_activation_path(int(mode))


def int4_debug_set_product_path(mode):
    """0 (default): int4_linear's product on the CUDA cores for T <= 2, else the tensor
    cores; 1: always the tensor cores; 2: the CUDA cores whenever T <= 4."""
    lib().int4_debug_set_product_path(int(mode))


def int8_quantize_activation(X, alpha=6.0, with_xo=True, stream=None):
    """-> dict(mask, idx, count, sX, Xq, Xo) (device tensors)."""
    import torch
    T, K = X.shape
    dev = X.device
    out = dict(
        mask=torch.full(((K + 31) // 32 + 3,), -1, dtype=torch.int32, device=dev),
        idx=torch.full((K,), -1, dtype=torch.int32, device=dev),
        count=torch.zeros(4, dtype=torch.int32, device=dev),
        sX=torch.empty(max(T, 1), dtype=torch.float32, device=dev),
        Xq=torch.empty((max(T, 1), K), dtype=torch.int8, device=dev),
        Xo=torch.full((max(T, 1), K), float("nan"), dtype=torch.float16, device=dev) if with_xo else None,
    )
    wsb = int(lib().int8_quantize_activation_workspace_size(T, K))
    ws = torch.empty(max(1, wsb), dtype=torch.uint8, device=dev)
    _check("int8_quantize_activation", lib().int8_quantize_activation(
        _dev(X, torch.float16, "X", 2), T, K, float(alpha), _dev(out["mask"], torch.int32, "mask"),
        _dev(out["idx"], torch.int32, "idx"), _dev(out["count"], torch.int32, "count"),
        _dev(out["sX"], torch.float32, "sX"), _dev(out["Xq"], torch.int8, "Xq"),
        _dev(out["Xo"], torch.float16, "Xo") if with_xo else None, ctypes.c_void_p(ws.data_ptr()), wsb,
        _stream(stream)))
    out["mask"] = out["mask"][:(K + 31) // 32]
    out["count"] = out["count"][:1]
    return out


def int8_gemm_i8_s32(Xq, Wq, acc=None, stream=None):
    """acc int32 [T,N] = Xq int8 [T,K] @ Wq int8 [K,N], exact."""
    import torch
    T, K = Xq.shape
    N = Wq.shape[1]
    acc = torch.empty((T, N), dtype=torch.int32, device=Xq.device) if acc is None else acc
    _check("int8_gemm_i8_s32", lib().int8_gemm_i8_s32(
        _dev(Xq, torch.int8, "Xq", 2), T, K, _dev(Wq, torch.int8, "Wq", 2), N,
        _dev(acc, torch.int32, "acc"), None, 0, _stream(stream)))
    return acc


def int8_read_and_clear_device_status(stream=None):
    code = ctypes.c_int(0)
    _check("int8_read_and_clear_device_status", lib().int8_read_and_clear_device_status(
        ctypes.byref(code), _stream(stream)))
    return code.value


def int8_selftest_wait_timeout(limit_us=1000, stream=None):
    """Enqueue the bounded-wait self-test kernel (see include/int8row.h)."""
    _check("int8_selftest_wait_timeout", lib().int8_selftest_wait_timeout(int(limit_us), _stream(stream)))


def int8_status_string(status):
    return lib().int8_status_string(int(status)).decode()


def int8_time_next_gemm(before, after):
    """Record two torch.cuda.Event objects around the next call's GEMM kernel."""
    lib().int8_time_next_gemm(ctypes.c_void_p(before.cuda_event) if before is not None else None,
                              ctypes.c_void_p(after.cuda_event) if after is not None else None)


def int8_kernel_launch_count():
    return int(lib().int8_kernel_launch_count())


# ---------------------------------------------------------------- group-wise 4-bit codec

def int4_packed_code_bytes(K, N):
    return int(lib().int4_packed_code_bytes(int(K), int(N)))


def int4_packed_scale_bytes(K, N):
    return int(lib().int4_packed_scale_bytes(int(K), int(N)))


def int4_quantize_weight_groupwise(W16, stream=None):
    """W16 fp16 [K,N] -> (W4 uint8, S4 uint8): the packed codes and (s, lo) pairs
    in the layout include/int8row.h describes."""
    import torch
    K, N = W16.shape
    nc, ns = int4_packed_code_bytes(K, N), int4_packed_scale_bytes(K, N)
    if nc == 0:
        raise I8RError("int4_quantize_weight_groupwise", 2 if K % 256 or N % 16 else 3)
    W4 = torch.empty(nc, dtype=torch.uint8, device=W16.device)
    S4 = torch.empty(ns, dtype=torch.uint8, device=W16.device)
    _check("int4_quantize_weight_groupwise", lib().int4_quantize_weight_groupwise(
        _dev(W16, torch.float16, "W16", 2), K, N, _dev(W4, torch.uint8, "W4"), _dev(S4, torch.uint8, "S4"),
        _stream(stream)))
    return W4, S4


def int4_dequantize_weight(W4, S4, K, N, stream=None):
    """The decoded weight W~ fp16 [K,N] of a packed 4-bit weight."""
    import torch
    out = torch.empty((K, N), dtype=torch.float16, device=W4.device)
    _check("int4_dequantize_weight", lib().int4_dequantize_weight(
        _dev(W4, torch.uint8, "W4"), _dev(S4, torch.uint8, "S4"), int(K), int(N), _dev(out, torch.float16, "W16d"),
        _stream(stream)))
    return out


def int4_linear_workspace_size(T, K, N):
    return int(lib().int4_linear_workspace_size(int(T), int(K), int(N)))


def int4_linear(X, W4, S4, N, Y=None, workspace_buf=None, stream=None):
    """Y fp16 [T,N] = X fp16 [T,K] times the decoded 4-bit weight (T <= 64)."""
    import torch
    T, K = X.shape
    Y = torch.empty((T, N), dtype=torch.float16, device=X.device) if Y is None else Y
    if workspace_buf is None:
        workspace_buf = torch.empty(max(1, int4_linear_workspace_size(T, K, N)), dtype=torch.uint8,
                                    device=X.device)
    ws = workspace_buf
    _check("int4_linear", lib().int4_linear(
        _dev(X, torch.float16, "X", 2), T, K, _dev(W4, torch.uint8, "W4"), _dev(S4, torch.uint8, "S4"), int(N),
        _dev(Y, torch.float16, "Y"), ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(),
        _stream(stream)))
    return Y
