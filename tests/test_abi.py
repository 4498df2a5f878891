"""The C-ABI library: it loads, exports every entry point the header declares,
and rejects bad arguments on the host before touching the device (CPU only:
no compute call is made)."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "int8row.h")


@pytest.fixture(scope="module")
def so():
    from int8_quantized_row_b200 import build
    build.build()
    import int8_quantized_row_b200 as m
    return m.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(int[48]_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("int8_quantize_weight_colwise", "int8_mixed_linear", "int8_outlier_stats",
                     "int8_mixed_linear_workspace_size", "int8_quantize_activation", "int8_gemm_i8_s32",
                     "int8_read_and_clear_device_status", "int8_status_string",
                     "int4_quantize_weight_groupwise", "int4_dequantize_weight", "int4_linear",
                     "int4_linear_workspace_size", "int4_packed_code_bytes", "int4_packed_scale_bytes"):
        assert required in names


def test_every_declared_symbol_is_exported(so):
    for name in declared_functions():
        assert hasattr(so, name), name


def test_library_exports_no_oracle_symbols(so):
    for name in ("orc_mixed_linear", "orc_quantize_rows", "orc_int8_gemm", "orc_half_to_float"):
        assert not hasattr(so, name)


def test_status_strings(so):
    for code in range(8):
        assert len(so.int8_status_string(code)) >= 2
    assert so.int8_status_string(99) == b"unknown status"


def _null():
    return ctypes.c_void_p(0)


def _p(addr=4096):
    return ctypes.c_void_p(addr)


def test_host_rejects_bad_shapes_before_any_launch(so):
    f = so.int8_mixed_linear
    ws = so.int8_mixed_linear_workspace_size(16, 1024, 1024)
    args = lambda T, K, N, alpha=6.0, x=_p(), y=_p(), wsp=_p(), wsb=ws: (
        x, T, K, _p(), _p(), _p(), N, alpha, y, wsp, wsb, _null())
    assert f(*args(16, 1000, 1024)) == 2          # K % 16
    assert f(*args(16, 1024, 1000)) == 2          # N % 16
    assert f(*args(16, 133152, 1024)) == 3        # K too large for exact int32 accumulation
    assert f(*args(16, 0, 1024)) == 3
    assert f(*args(-1, 1024, 1024)) == 1
    assert f(*args(16, 1024, 1024, alpha=float("nan"))) == 1
    assert f(*args(16, 1024, 1024, alpha=-1.0)) == 1
    assert f(*args(16, 1024, 1024, x=_null())) == 1
    assert f(*args(16, 1024, 1024, x=_p(4097))) == 2     # misaligned
    assert f(*args(16, 1024, 1024, wsb=ws - 1)) == 4     # workspace too small
    assert f(*args(16, 1024, 1024, wsp=_null())) == 4
    assert f(*args(0, 1024, 1024)) == 0           # T == 0: a no-op


def test_wq_variant_host_checks_and_capacity(so):
    f = so.int8_mixed_linear_wq
    ws = so.int8_mixed_linear_wq_workspace_size(16, 1024, 1024)
    args = lambda T, K, N, alpha=6.0, x=_p(), wsb=ws: (x, T, K, _p(), _p(), N, alpha, _p(), _p(), wsb, _null())
    assert f(*args(16, 1000, 1024)) == 2          # K % 16
    assert f(*args(16, 133152, 1024)) == 3
    assert f(*args(16, 1024, 1024, alpha=float("nan"))) == 1
    assert f(*args(16, 1024, 1024, x=_null())) == 1
    assert f(*args(16, 1024, 1024, wsb=ws - 1)) == 4
    assert f(*args(0, 1024, 1024)) == 0
    # the plain entry point still needs W16
    g = so.int8_mixed_linear
    assert g(_p(), 16, 1024, _p(), _p(), _null(), 1024, 6.0, _p(), _p(),
             so.int8_mixed_linear_workspace_size(16, 1024, 1024), _null()) == 1
    # rows of dequantised outlier weights the workspace holds:
    # at least 256 and K/16, rounded up to 64, at most K rounded up to 64
    cap = so.int8_mixed_linear_wq_max_outliers
    assert [cap(k) for k in (16, 64, 1024, 5120, 12288, 49152)] == [64, 64, 256, 320, 768, 3072]
    # the workspace holds exactly those rows where the plain one holds its
    # compacted W16 rows: 256 at prefill sizes; at decode sizes at least 256
    # and K/64 (rounded up to 64), at most K rounded up to 64
    k64 = lambda K: (K + 63) // 64 * 64
    for T, K, N in ((2048, 12288, 49152), (300, 1024, 512)):
        extra = so.int8_mixed_linear_wq_workspace_size(T, K, N) - so.int8_mixed_linear_workspace_size(T, K, N)
        assert extra == (cap(K) - min(256, k64(K))) * N * 2
    for T, K, N in ((16, 12288, 49152), (128, 1024, 512), (1, 64, 16), (16, 49152, 12288)):
        extra = so.int8_mixed_linear_wq_workspace_size(T, K, N) - so.int8_mixed_linear_workspace_size(T, K, N)
        assert extra == (cap(K) - min(k64(K), max(256, k64((K + 63) // 64)))) * N * 2


def test_chain_host_checks_and_workspace(so):
    from int8_quantized_row_b200 import I8rLayer
    f = so.int8_mixed_linear_chain
    size = so.int8_mixed_linear_chain_workspace_size

    def layer(T, K, N, w16=True, alpha=6.0, x=4096):
        return I8rLayer(ctypes.c_void_p(x), T, K, _p(), _p(), _p() if w16 else _null(), N, alpha, _p())

    def arr(*layers):
        a = (I8rLayer * len(layers))(*layers)
        return ctypes.cast(a, ctypes.c_void_p), a

    # the workspace is the largest layer's need, each layer sized for its variant
    shapes = [(16, 12288, 36864, True), (16, 12288, 12288, True), (16, 12288, 49152, False), (300, 1024, 512, True)]
    ptr, keep = arr(*(layer(*s) for s in shapes))
    want = max(so.int8_mixed_linear_workspace_size(T, K, N) if w else so.int8_mixed_linear_wq_workspace_size(T, K, N)
               for T, K, N, w in shapes)
    assert size(len(shapes), ptr) == want
    assert size(0, _null()) == 0
    # n = 0 is a no-op; bad counts and pointers are rejected
    assert f(0, _null(), _null(), 0, _null()) == 0
    assert f(-1, ptr, _p(), want, _null()) == 1
    assert f(2, _null(), _p(), want, _null()) == 1
    # a bad layer anywhere returns its error before anything is enqueued
    ok = layer(16, 1024, 1024)
    for bad, code in ((layer(16, 1000, 1024), 2), (layer(16, 1024, 1024, alpha=float("nan")), 1),
                      (layer(16, 1024, 1024, x=0), 1), (layer(16, 1024, 1024, x=4097), 2),
                      (layer(16, 133152, 1024), 3)):
        ptr2, keep2 = arr(ok, bad)
        ws = size(1, arr(ok)[0])
        assert f(2, ptr2, _p(), 1 << 30, _null()) == code
    # workspace too small for the largest layer, or misaligned
    ptr3, keep3 = arr(layer(16, 1024, 1024), layer(16, 1024, 4096))
    need = size(2, ptr3)
    assert need == so.int8_mixed_linear_workspace_size(16, 1024, 4096)
    assert f(2, ptr3, _p(), need - 1, _null()) == 4
    assert f(2, ptr3, _p(4096 + 16), need, _null()) == 2


def test_host_rejects_bad_weight_conversion(so):
    f = so.int8_quantize_weight_colwise
    assert f(_p(), 1024, 1000, _p(), _p(), _null()) == 2
    assert f(_null(), 1024, 1024, _p(), _p(), _null()) == 1
    assert f(_p(), 8, 1024, _p(), _p(), _null()) == 3


def test_host_rejects_bad_stats_args(so):
    f = so.int8_outlier_stats
    wsb = so.int8_outlier_stats_workspace_size(1024)
    assert f(_p(), 4, 1024, 6.0, _null(), _p(), _null(), _p(), _p(), wsb, _null()) == 1
    assert f(_p(), 4, 1024, 6.0, _p(), _p(), _null(), _p(), _p(), wsb - 1, _null()) == 4


def test_workspace_size_grows_with_shape(so):
    a = so.int8_mixed_linear_workspace_size(16, 1024, 1024)
    b = so.int8_mixed_linear_workspace_size(32, 1024, 1024)
    c = so.int8_mixed_linear_workspace_size(256, 1024, 1024)
    assert 0 < a < b
    # it covers Xq (T*K) and the fp16 outlier capacity (2*T*K) at least
    assert c >= 3 * 256 * 1024
    assert so.int8_mixed_linear_workspace_size(-1, 1024, 1024) == 0


def test_selftest_rejects_bad_limit(so):
    assert so.int8_selftest_wait_timeout(0, _null()) == 3
    assert so.int8_selftest_wait_timeout(2000000, _null()) == 3


def test_int8_weights_take_half_the_bytes():
    """The stored weight (int8 codes + one fp32 scale per column) takes about
    half the bytes of the fp16 weight (LLM.int8() abstract: inference memory
    cut by half), approaching 1/2 as K grows."""
    for K, N in ((5120, 20480), (12288, 49152), (49152, 12288)):
        ratio = (K * N + 4 * N) / (2 * K * N)
        assert 0.5 < ratio <= 0.5 + 2.0 / K + 1e-15


def test_int4_host_rejections(so):
    """The 4-bit entry points check shapes, pointers and workspace on the host."""
    P = ctypes.c_void_p
    so.int4_linear.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int, P, P, ctypes.c_size_t, P]
    so.int4_linear_workspace_size.argtypes = [ctypes.c_int] * 3
    so.int4_linear_workspace_size.restype = ctypes.c_size_t
    so.int4_packed_code_bytes.argtypes = [ctypes.c_int] * 2
    so.int4_packed_code_bytes.restype = ctypes.c_size_t
    so.int4_quantize_weight_groupwise.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P]
    ws = so.int4_linear_workspace_size(16, 1024, 1024)
    assert ws > 0
    assert so.int4_linear_workspace_size(65, 1024, 1024) == 0           # T > 64
    assert so.int4_linear_workspace_size(16, 1000, 1024) == 0           # K not a multiple of 256
    assert so.int4_packed_code_bytes(1024, 1000) == 0                   # N not a multiple of 16
    assert so.int4_packed_code_bytes(512, 300 * 16) == 512 * 4864 // 2  # 4800 columns padded to 19 x 256
    a = _p()
    assert so.int4_linear(a, 16, 1000, a, a, 1024, a, a, ws, None) == 2         # I8R_EALIGN
    assert so.int4_linear(a, 65, 1024, a, a, 1024, a, a, ws, None) == 3         # I8R_ERANGE
    assert so.int4_linear(a, -1, 1024, a, a, 1024, a, a, ws, None) == 1         # I8R_EINVAL
    assert so.int4_linear(_null(), 16, 1024, a, a, 1024, a, a, ws, None) == 1   # null X
    assert so.int4_linear(_p(4097), 16, 1024, a, a, 1024, a, a, ws, None) == 2  # misaligned X
    assert so.int4_linear(a, 16, 1024, a, a, 1024, a, a, ws - 1, None) == 4     # workspace too small
    assert so.int4_linear(a, 0, 1024, a, a, 1024, a, a, 0, None) == 0           # T = 0: no-op
    assert so.int4_quantize_weight_groupwise(a, 128, 1024, a, a, None) == 3    # K < 256
