"""int8_mixed_linear_noalloc against int8_mixed_linear (GPU).

The allocation-free entry point is for callers that cannot allocate device
memory where they call the layer (a plugin that only receives input and
output buffers from a runtime owning the GPU's memory, or a path where
cudaMalloc may not block or synchronise).  Its scratch is a fixed array
inside the library.  It is called here through the C ABI, twice in a row
(the second call finds the first call's leftovers in the shared scratch),
and must give the workspace entry point's Y, and the oracle's, within the Y
tolerance.  This file is collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import int8_quantized_row_b200 as i8
from gpu_helpers import assert_y_close, outlier_x, to_dev, to_host

pytestmark = pytest.mark.gpu

_P = ctypes.c_void_p


def _entry():
    so = i8.lib()
    f = so.int8_mixed_linear_noalloc
    f.argtypes = [_P, ctypes.c_int, ctypes.c_int, _P, _P, _P, ctypes.c_int, ctypes.c_float, _P, _P]
    f.restype = ctypes.c_int
    so.int8_mixed_linear_noalloc_max_workspace.restype = ctypes.c_size_t
    return f, int(so.int8_mixed_linear_noalloc_max_workspace())


def _ptr(t):
    return _P(t.data_ptr())


@pytest.mark.parametrize("T,K,N", [(16, 1024, 1024), (16, 12288, 4096), (200, 2048, 512)])
def test_noalloc_matches_workspace_entry_point(orc, T, K, N):
    f, cap = _entry()
    assert i8.int8_mixed_linear_workspace_size(T, K, N) <= cap
    rng = np.random.default_rng(T + K + N)
    X = outlier_x(rng, T, K, [3, K // 2, K - 5])
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    Xd, Wd = to_dev(X), to_dev(W)
    Wq, sW = i8.int8_quantize_weight_colwise(Wd)
    ref = to_host(i8.int8_mixed_linear(Xd, Wq, sW, Wd, 6.0))
    Wq_o, sW_o = orc.quantize_weight_colwise(W)
    Y_o, _, _, _ = orc.mixed_linear(X, Wq_o, sW_o, W, 6.0)
    stream = _P(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        Y = torch.full((T, N), float("nan"), dtype=torch.float16, device="cuda")
        rc = f(_ptr(Xd), T, K, _ptr(Wq), _ptr(sW), _ptr(Wd), N, 6.0, _ptr(Y), stream)
        assert rc == 0, i8.int8_status_string(rc)
        torch.cuda.synchronize()
        assert_y_close(to_host(Y), ref, f"noalloc vs workspace entry point T={T} K={K} N={N}")
        assert_y_close(to_host(Y), Y_o, f"noalloc vs oracle T={T} K={K} N={N}")
    assert i8.int8_read_and_clear_device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    f, cap = _entry()
    T, K, N = 128, 12288, 8192                       # needs about 8.9 MB
    assert i8.int8_mixed_linear_workspace_size(T, K, N) > cap
    X = torch.zeros((T, K), dtype=torch.float16, device="cuda")
    Wq = torch.zeros((K, N), dtype=torch.int8, device="cuda")
    sW = torch.zeros(N, dtype=torch.float32, device="cuda")
    W16 = torch.zeros((K, N), dtype=torch.float16, device="cuda")
    Y = torch.full((T, N), 7.0, dtype=torch.float16, device="cuda")
    rc = f(_ptr(X), T, K, _ptr(Wq), _ptr(sW), _ptr(W16), N, 6.0, _ptr(Y), _P(torch.cuda.current_stream().cuda_stream))
    assert rc == 3                                   # I8R_ERANGE, nothing enqueued
    torch.cuda.synchronize()
    assert bool((Y == 7.0).all())
