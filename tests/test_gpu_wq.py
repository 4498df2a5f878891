"""The Wq-only variant (outlier rows dequantised from Wq) against the oracle.

Same tolerance on Y as the fp16-weight layer.  At every T the quantiser's
leading blocks write the dequantised rows into the workspace; shapes cover
the decode kernel (T <= 128) and the prefill kernel, outlier sets of one and
several 64-column blocks, a long schedule, alpha = 0 at decode size, an
outlier count exactly at the workspace's capacity, and counts past it at both
kernels, where the GEMM's producer dequantises the remaining rows by index.
"""
import numpy as np
import pytest
import torch

import int8_quantized_row_b200 as i8
from gpu_helpers import assert_y_close, device_status_clean, outlier_x, to_dev, to_host

pytestmark = pytest.mark.gpu

WQ_CASES = [
    # T, K, N, outlier columns, alpha, rows sampled (None: all)
    (1, 64, 16, [5], 6.0, None),
    (16, 1024, 1024, [171, 918], 6.0, None),
    (128, 1024, 272, list(range(15)), 6.0, None),
    (64, 256, 256, [], 0.0, None),                            # decode: every column an outlier
    (129, 1024, 272, list(range(16)), 6.0, None),
    (200, 1040, 528, list(range(0, 1040, 61)), 6.0, None),
    (300, 2048, 256, list(range(0, 2048, 31)), 6.0, None),   # |O| = 67: two outlier blocks
    (2048, 1024, 4096, list(range(0, 1024, 15)), 6.0, 7),    # long schedule, |O| = 69
    (300, 1024, 512, list(range(0, 1024, 4)), 6.0, None),    # |O| = 256 = the capacity at K = 1024
    (300, 1024, 512, list(range(0, 1024, 3)), 6.0, None),    # |O| = 342: 86 rows past the capacity
    (16, 1024, 1040, list(range(0, 1024, 3)), 6.0, None),    # the same at decode size, ragged N
    (260, 1024, 256, [], 0.0, None),                          # prefill, every column an outlier
]


@pytest.mark.parametrize("T,K,N,cols,alpha,every", WQ_CASES)
def test_wq_variant_matches_oracle(orc, T, K, N, cols, alpha, every):
    rng = np.random.default_rng(T * 7 + K + 3 * N)
    X = outlier_x(rng, T, K, cols)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    Wq_o, sW_o = orc.quantize_weight_colwise(W)
    Wq, sW = i8.int8_quantize_weight_colwise(to_dev(W))
    Y = to_host(i8.int8_mixed_linear_wq(to_dev(X), Wq, sW, alpha))
    torch.cuda.synchronize()
    rows = None if every is None else np.arange(0, T, every, dtype=np.int32)
    Y_o, _, _, cnt = orc.mixed_linear(X, Wq_o, sW_o, None, alpha, rows=rows)
    assert_y_close(Y if rows is None else Y[rows], Y_o, f"wq T={T} K={K} N={N} |O|={cnt}")
    assert device_status_clean()


def test_wq_variant_differs_from_fp16_weights_only_in_outlier_rows(orc):
    # the two entry points share everything but the outlier rows' source
    rng = np.random.default_rng(5)
    T, K, N = 300, 1024, 512
    X = outlier_x(rng, T, K, [3, 500, 1001])
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    Xd, Wd = to_dev(X), to_dev(W)
    Wq, sW = i8.int8_quantize_weight_colwise(Wd)
    Y16 = to_host(i8.int8_mixed_linear(Xd, Wq, sW, Wd, 6.0))
    Yq = to_host(i8.int8_mixed_linear_wq(Xd, Wq, sW, 6.0))
    X0 = X.copy()
    X0[:, [3, 500, 1001]] = 0                                  # no outliers: the variants coincide
    X0d = to_dev(X0)
    assert np.array_equal(to_host(i8.int8_mixed_linear(X0d, Wq, sW, Wd, 6.0)).view(np.uint16),
                          to_host(i8.int8_mixed_linear_wq(X0d, Wq, sW, 6.0)).view(np.uint16))
    assert not np.array_equal(Y16.view(np.uint16), Yq.view(np.uint16))
    assert device_status_clean()


@pytest.mark.parametrize("T", [260, 16])
def test_wq_variant_past_its_workspace_capacity_matches_oracle(orc, T):
    # alpha = 0 makes every column an outlier: 1024 > 256 compacted rows (prefill
    # and decode); the rows past them are dequantised in the GEMM, nothing is dropped
    K, N = 1024, 256
    assert i8.int8_mixed_linear_wq_max_outliers(K) == 256
    rng = np.random.default_rng(9)
    X = rng.standard_normal((T, K)).astype(np.float16)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    Wq_o, sW_o = orc.quantize_weight_colwise(W)
    Wq, sW = i8.int8_quantize_weight_colwise(to_dev(W))
    Y = to_host(i8.int8_mixed_linear_wq(to_dev(X), Wq, sW, 0.0))
    Y_o, _, _, cnt = orc.mixed_linear(X, Wq_o, sW_o, None, 0.0)
    assert cnt == K
    assert_y_close(Y, Y_o, f"wq alpha=0 T={T}")
    assert device_status_clean()
