"""CUDA path vs the CPU oracle, element by element, on small and ragged shapes.

Bit-exact: weight codes and scales, outlier mask / index list / count, row
scales and codes, the gathered outlier columns, int32 accumulators.
Tolerance on Y: relative L2 <= 1e-3 and max abs <= 2^-8 max|Y_oracle|.
Shapes span several 128 x 256 tiles and ragged tails in T, K and N, both
GEMM variants (decode-shaped for T <= 128, prefill above), and the
degenerate cases of the method (no outliers, every column an outlier,
all-zero rows and columns, T = 0).
"""
import numpy as np
import pytest
import torch

import int8_quantized_row_b200 as i8
from gpu_helpers import assert_y_close, device_status_clean, outlier_x, to_dev, to_host

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ weights

@pytest.mark.parametrize("K,N", [(16, 16), (96, 48), (1024, 272), (160, 1040), (5120, 256)])
def test_weight_conversion_bit_exact(orc, K, N):
    rng = np.random.default_rng(K * 7 + N)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    W[:, 3] = 0                                    # all-zero column -> sW = 0, codes 0
    W[5, 7] = np.float16(-0.5)                     # a clear column maximum
    Wq_o, sW_o = orc.quantize_weight_colwise(W)
    Wq, sW = i8.int8_quantize_weight_colwise(to_dev(W))
    torch.cuda.synchronize()
    assert np.array_equal(to_host(sW), sW_o)
    assert np.array_equal(to_host(Wq), Wq_o)
    assert device_status_clean()


def test_weight_conversion_all_fp16_codes(orc):
    """Every finite fp16 value passes through the column quantiser."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    vals = bits[np.isfinite(bits)]
    N = 64
    K = (len(vals) + N - 1) // N // 16 * 16 + 16
    W = np.zeros(K * N, np.float16)
    W[:len(vals)] = vals
    W = W.reshape(K, N)
    Wq_o, sW_o = orc.quantize_weight_colwise(W)
    Wq, sW = i8.int8_quantize_weight_colwise(to_dev(W))
    assert np.array_equal(to_host(sW), sW_o)
    assert np.array_equal(to_host(Wq), Wq_o)


# ------------------------------------------------------------------ activation side

ACT_CASES = [
    # T, K, outlier columns, alpha
    (1, 64, [5], 6.0),
    (3, 96, [0, 95], 6.0),
    (16, 1024, [171, 918], 6.0),
    (127, 1024, list(range(0, 1024, 61)), 6.0),
    (129, 1040, [], 6.0),
    (300, 4096, [1, 2, 3, 4000], 2.5),
    (17, 256, [], 0.0),                      # every column is an outlier
    (17, 256, [10, 20], float("inf")),       # none is
    (5, 12288, [7, 12287], 6.0),
    (2100, 1024, [5, 1000], 6.0),            # eight partial masks of 263 rows
]


@pytest.mark.parametrize("T,K,cols,alpha", ACT_CASES)
def test_activation_quantisation_bit_exact(orc, T, K, cols, alpha):
    rng = np.random.default_rng(T * 1000 + K)
    X = outlier_x(rng, T, K, cols)
    if T > 2:
        X[2] = 0                                   # an all-zero row
    out = i8.int8_quantize_activation(to_dev(X), alpha)
    torch.cuda.synchronize()
    mask_o, idx_o = orc.outlier_columns(X, alpha)
    Xq_o, sX_o = orc.quantize_rows(X, mask_o)
    cnt = int(to_host(out["count"])[0])
    assert cnt == len(idx_o)
    assert np.array_equal(to_host(out["idx"])[:cnt], idx_o)
    words = to_host(out["mask"]).view(np.uint32)
    bits = np.array([(words[k // 32] >> (k % 32)) & 1 for k in range(K)], bool)
    assert np.array_equal(bits, mask_o)
    assert np.array_equal(to_host(out["sX"])[:T], sX_o)
    assert np.array_equal(to_host(out["Xq"])[:T], Xq_o)
    Xo = to_host(out["Xo"])[:T]
    pad = (cnt + 63) // 64 * 64
    assert np.array_equal(Xo[:, :cnt].view(np.uint16), X[:, idx_o].view(np.uint16))
    assert np.all(Xo[:, cnt:pad] == 0)
    assert device_status_clean()


def test_quantiser_ties_round_half_away(orc):
    # Rows whose scale puts x * fl32(127/absmax) exactly on k + 1/2 (and just
    # below 1/2), where round-half-away and other rules part ways.
    K = 576
    X = np.zeros((3, K), np.float16)
    halves = np.arange(-126.5, 127.0, 1.0)                # absmax 127: inv = 1
    X[0, :2] = [127, -127]
    X[0, 2:2 + len(halves)] = halves
    below = np.nextafter(np.float16(0.5), np.float16(0))  # largest fp16 < 1/2
    X[0, 300:306] = [below, -below, 0.5, -0.5, np.nextafter(np.float16(1.5), np.float16(0)), -1.5]
    odd = np.arange(-253, 254, 2)                         # absmax 254: inv = 1/2
    X[1, :2] = [254, -254]
    X[1, 2:2 + len(odd)] = odd
    X[2] = np.linspace(-3.0, 3.0, K).astype(np.float16)   # an ordinary scale
    out = i8.int8_quantize_activation(to_dev(X), float("inf"))
    torch.cuda.synchronize()
    mask_o, _ = orc.outlier_columns(X, float("inf"))
    Xq_o, sX_o = orc.quantize_rows(X, mask_o)
    Xq = to_host(out["Xq"])[:3]
    assert np.array_equal(Xq, Xq_o)
    assert list(Xq[0, 300:306]) == [0, 0, 1, -1, 1, -2]
    assert Xq[0, 2] == -127 and Xq[0, 3] == -126 and Xq[0, 2 + 127] == 1    # -126.5, -125.5, 0.5
    assert device_status_clean()


FUSED_CASES = ACT_CASES + [
    (2048, 5120, [3, 900, 5000], 6.0),        # the OPT-13B prefill batch: 14 rows per block
    (8, 49152, [7, 40000], 6.0),              # one row of 96 KB in a block
    (128, 12288, list(range(0, 12288, 97)), 6.0),
    (4096, 12288, [5], 6.0),                  # too big for shared memory: both calls take the two-kernel path
    # thresholds fp16 does not hold: the one-kernel path compares fp16 bit patterns
    # with the smallest fp16 >= alpha, the two-kernel path compares in fp32
    (64, 1024, [], 1.0 / 3.0),
    (64, 1024, [], 3.1),
    (32, 2048, [], 2.0 ** -20),
    # batches under 8 rows: by default the row quantiser finds the mask itself
    (1, 32768, [7, 32000], 6.0),              # T*K at the one-launch bound
    (1, 16400, [5, 16399], 6.0),              # K % 32 == 16: a half word at the end
    (7, 1040, [], 0.0),                       # every column an outlier
    (6, 1024, [], 1.0 / 3.0),
    (2, 2048, [], 2.0 ** -20),
    (1, 49152, [7, 40000], 6.0),              # the 175B fc2 width, past the bound: scan + quantiser
    (3, 16400, [9], 6.0),
]


@pytest.mark.parametrize("T,K,cols,alpha", FUSED_CASES)
def test_fused_activation_equals_two_kernel_path(orc, T, K, cols, alpha):
    """Every activation path -- the cooperative one-kernel path (X held in
    shared memory, grid barrier, fp16 bit-pattern threshold), the default (for
    batches under 8 rows the row quantiser finding the mask itself, with the
    same bit-pattern threshold) and the outlier scan followed by the row
    quantiser -- gives the oracle's mask, index list, count, row scales, codes
    and gathered outlier columns bit for bit, including at thresholds fp16
    cannot hold."""
    rng = np.random.default_rng(T * 7 + K)
    X = outlier_x(rng, T, K, cols)
    if T > 2:
        X[1] = 0
    if 0.0 < alpha < float("inf"):
        # the fp16 values next to the threshold (which fp16 may not hold exactly)
        a = np.float16(alpha)
        X[0, :4] = [a, np.nextafter(a, np.float16(0)), np.nextafter(a, np.float16(np.inf)), -a]
    mask_o, idx_o = orc.outlier_columns(X, alpha)
    Xq_o, sX_o = orc.quantize_rows(X, mask_o)
    cnt_o = len(idx_o)
    pad = min((cnt_o + 63) // 64 * 64, K)
    Xd = to_dev(X)
    try:
        for fused in (2, 1, 0):         # cooperative wherever X fits, the default, the two kernels
            i8.int8_debug_set_activation_path(fused)
            out = {k: to_host(v).copy() for k, v in i8.int8_quantize_activation(Xd, alpha).items()}
            what = f"path {fused}"
            cnt = int(out["count"][0])
            assert cnt == cnt_o, what
            words = out["mask"].view(np.uint32)
            bits = (words[np.arange(K) // 32] >> (np.arange(K) % 32)) & 1
            assert np.array_equal(bits.astype(bool), mask_o), what
            assert np.array_equal(out["idx"][:cnt], idx_o), what
            assert np.array_equal(out["sX"][:T], sX_o), what
            assert np.array_equal(out["Xq"][:T], Xq_o), what
            Xo = out["Xo"][:T]
            assert np.array_equal(Xo[:, :cnt].view(np.uint16), X[:, idx_o].view(np.uint16)), what
            assert np.all(Xo[:, cnt:pad] == 0), what
            assert device_status_clean()
    finally:
        i8.int8_debug_set_activation_path(1)


@pytest.mark.parametrize("T,K", [(16, 1024), (100, 12288)])
def test_refused_cooperative_launch_falls_back_to_two_kernels(orc, T, K):
    """When the runtime refuses the one-kernel path's cooperative launch, the
    call runs the outlier scan and the row quantiser instead (mode 3 treats
    every cooperative launch as refused): one more launch, the oracle's bits."""
    rng = np.random.default_rng(T + K)
    X = outlier_x(rng, T, K, [1, K // 3])
    mask_o, idx_o = orc.outlier_columns(X, 6.0)
    Xq_o, sX_o = orc.quantize_rows(X, mask_o)
    Xd = to_dev(X)
    launches = {}
    try:
        for mode in (1, 3):
            i8.int8_debug_set_activation_path(mode)
            n0 = i8.int8_kernel_launch_count()
            out = {k: to_host(v).copy() for k, v in i8.int8_quantize_activation(Xd, 6.0).items()}
            launches[mode] = i8.int8_kernel_launch_count() - n0
            cnt = int(out["count"][0])
            assert cnt == len(idx_o) and np.array_equal(out["idx"][:cnt], idx_o)
            assert np.array_equal(out["sX"][:T], sX_o) and np.array_equal(out["Xq"][:T], Xq_o)
            assert device_status_clean()
    finally:
        i8.int8_debug_set_activation_path(1)
    assert launches == {1: 2, 3: 3}     # clear + fused kernel; clear + scan + quantiser


@pytest.mark.parametrize("T,K", [(3, 1040), (16, 1024)])
def test_nan_and_inf_in_x_take_the_oracles_outlier_decision(orc, T, K):
    """|x| >= alpha is false for NaN and true for infinity on every path (the
    bit-pattern compares exclude NaN as the float compare does), so the
    outlier set is the oracle's."""
    rng = np.random.default_rng(T * K)
    X = outlier_x(rng, T, K, [4])
    X[0, 10] = np.float16(np.nan)
    X[T - 1, 11] = -np.float16(np.nan)
    X[1, 12] = np.float16(np.inf)
    X[0, 13] = -np.float16(np.inf)
    mask_o, idx_o = orc.outlier_columns(X, 6.0)
    assert list(idx_o) == [4, 12, 13]
    Xd = to_dev(X)
    try:
        for mode in (2, 1, 0):
            i8.int8_debug_set_activation_path(mode)
            out = {k: to_host(v).copy() for k, v in i8.int8_quantize_activation(Xd, 6.0).items()}
            cnt = int(out["count"][0])
            assert cnt == len(idx_o) and np.array_equal(out["idx"][:cnt], idx_o), f"path {mode}"
            words = out["mask"].view(np.uint32)
            bits = (words[np.arange(K) // 32] >> (np.arange(K) % 32)) & 1
            assert np.array_equal(bits.astype(bool), mask_o), f"path {mode}"
    finally:
        i8.int8_debug_set_activation_path(1)


@pytest.mark.parametrize("T,K,launches", [(1, 12288, 1), (2, 12288, 1), (3, 12288, 3), (7, 1040, 1)])
def test_small_batches_quantise_in_one_launch(orc, T, K, launches):
    """Under 8 rows and T*K <= 32768 the default activation side is one launch
    (the row quantiser finds the mask); past that bound it is the mask clear,
    the scan and the quantiser."""
    rng = np.random.default_rng(T + K)
    X = outlier_x(rng, T, K, [2, K - 1])
    mask_o, idx_o = orc.outlier_columns(X, 6.0)
    Xq_o, sX_o = orc.quantize_rows(X, mask_o)
    Xd = to_dev(X)
    n0 = i8.int8_kernel_launch_count()
    out = {k: to_host(v).copy() for k, v in i8.int8_quantize_activation(Xd, 6.0).items()}
    assert i8.int8_kernel_launch_count() - n0 == launches
    cnt = int(out["count"][0])
    assert cnt == len(idx_o) and np.array_equal(out["idx"][:cnt], idx_o)
    assert np.array_equal(out["sX"][:T], sX_o) and np.array_equal(out["Xq"][:T], Xq_o)
    assert device_status_clean()


def test_activation_t0_is_noop():
    X = torch.zeros((0, 64), dtype=torch.float16, device="cuda")
    out = i8.int8_quantize_activation(X, 6.0)
    torch.cuda.synchronize()
    assert int(out["count"][0]) == 0


# ------------------------------------------------------------------ int8 product

GEMM_CASES = [
    # T, K, N  (T <= 128: decode-shaped kernel; T > 128: prefill kernel)
    (1, 64, 16), (3, 96, 48), (16, 1024, 1024), (100, 160, 272), (128, 1024, 256),
    (129, 1024, 256), (256, 512, 512), (300, 1040, 272), (513, 256, 528), (200, 12288, 64),
    (8, 12288, 1024), (2, 4096, 12288),
]


@pytest.mark.parametrize("T,K,N", GEMM_CASES)
def test_int8_gemm_bit_exact(T, K, N):
    rng = np.random.default_rng(T + 3 * K + 7 * N)
    A = rng.integers(-127, 128, (T, K)).astype(np.int8)
    B = rng.integers(-127, 128, (K, N)).astype(np.int8)
    A[0, :] = 127
    B[:, 0] = 127                                 # the largest accumulator, K * 127^2
    acc = i8.int8_gemm_i8_s32(to_dev(A), to_dev(B))
    torch.cuda.synchronize()
    ref = A.astype(np.int64) @ B.astype(np.int64)
    assert np.array_equal(to_host(acc).astype(np.int64), ref)
    assert device_status_clean()


K_MAX = 133136      # the largest multiple of 16 with K * 127^2 < 2^31 (int32 accumulation exact)


@pytest.mark.parametrize("T", [2, 130])
def test_int8_gemm_at_the_largest_k(T):
    """K = 133136, with a row of 127 codes against a column of 127 codes: the
    accumulator K * 127^2 = 2147350544 is within 2^17 of INT32_MAX.  Decode
    (T = 2) and prefill (T = 130) kernels, checked bit for bit against int64
    sums on a few columns (all of them at T = 2)."""
    K, N = K_MAX, 256
    assert K * 127 * 127 < 2 ** 31 and K % 16 == 0
    rng = np.random.default_rng(T + 1)
    A = rng.integers(-127, 128, (T, K)).astype(np.int8)
    B = rng.integers(-127, 128, (K, N)).astype(np.int8)
    A[0, :] = 127
    B[:, 0] = 127
    A[T - 1, :] = -127                           # the most negative accumulator
    acc = to_host(i8.int8_gemm_i8_s32(to_dev(A), to_dev(B))).astype(np.int64)
    cols = np.arange(N) if T <= 16 else np.array([0, 1, 128, 255])
    ref = A.astype(np.int64) @ B[:, cols].astype(np.int64)
    assert ref[0, 0] == K * 127 * 127 and ref[T - 1, 0] == -K * 127 * 127
    assert np.array_equal(acc[:, cols], ref)
    assert device_status_clean()


def test_mixed_linear_at_the_largest_k(orc):
    """The whole layer at K = 133136 against the oracle (decode shape, outlier
    columns spread over the whole K)."""
    T, K, N = 2, K_MAX, 256
    rng = np.random.default_rng(2)
    X = outlier_x(rng, T, K, [0, 70000, K - 1])
    W = (rng.standard_normal((K, N)) * 0.01).astype(np.float16)
    Wq_o, sW_o = orc.quantize_weight_colwise(W)
    Wd = to_dev(W)
    Wq, sW = i8.int8_quantize_weight_colwise(Wd)
    assert np.array_equal(to_host(Wq), Wq_o) and np.array_equal(to_host(sW), sW_o)
    Y = to_host(i8.int8_mixed_linear(to_dev(X), Wq, sW, Wd, 6.0))
    Y_o, _, _, cnt = orc.mixed_linear(X, Wq_o, sW_o, W, 6.0)
    assert cnt == 3
    assert_y_close(Y, Y_o, f"K={K}")
    assert device_status_clean()


def test_int8_gemm_against_oracle_accumulators(orc):
    rng = np.random.default_rng(99)
    X = outlier_x(rng, 200, 1024, [3, 500])
    W = (rng.standard_normal((1024, 384)) * 0.02).astype(np.float16)
    Wq_o, _ = orc.quantize_weight_colwise(W)
    mask, _ = orc.outlier_columns(X, 6.0)
    Xq_o, _ = orc.quantize_rows(X, mask)
    acc_o = orc.int8_gemm(Xq_o, Wq_o)
    for T in (200, 64):
        acc = i8.int8_gemm_i8_s32(to_dev(Xq_o[:T]), to_dev(Wq_o))
        assert np.array_equal(to_host(acc), acc_o[:T])


# ------------------------------------------------------------------ whole layer

LINEAR_CASES = [
    # T, K, N, outlier columns, alpha, row_prob
    (1, 64, 16, [5], 6.0, 1.0),
    (3, 96, 48, [], 6.0, 1.0),
    (16, 1024, 1024, [171, 918], 6.0, 1.0),          # the single-linear shape
    (16, 1024, 1024, [171, 918], float("inf"), 1.0),
    (128, 1024, 272, list(range(15)), 6.0, 1.0),      # |O| = 15
    (129, 1024, 272, list(range(16)), 6.0, 1.0),      # |O| = 16
    (200, 1040, 528, list(range(0, 1040, 61)), 6.0, 1.0),   # |O| = 18
    (300, 2048, 256, list(range(0, 2048, 31)), 6.0, 0.25),  # |O| = 67 > 64: two outlier blocks
    (257, 512, 1024, [0, 511], 6.0, 0.25),
    (64, 256, 256, [], 0.0, 1.0),                     # alpha = 0: every column in 16-bit
    (200, 256, 256, [], 0.0, 1.0),
    (7, 12288, 1024, [1, 100, 12000], 6.0, 1.0),
    # prefill past the 256 compacted outlier weight rows: the later outlier
    # blocks gather their rows (four at a time, the tail one by one)
    (300, 2048, 512, list(range(0, 2048, 7)), 6.0, 0.5),  # |O| = 293
    (260, 1024, 256, [], 0.0, 1.0),                       # alpha = 0: |O| = K = 1024
]


@pytest.mark.parametrize("T,K,N,cols,alpha,row_prob", LINEAR_CASES)
def test_mixed_linear_matches_oracle(orc, T, K, N, cols, alpha, row_prob):
    rng = np.random.default_rng(T * 31 + K + N)
    X = outlier_x(rng, T, K, cols, row_prob=row_prob)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    Wq_o, sW_o = orc.quantize_weight_colwise(W)
    Wq, sW = i8.int8_quantize_weight_colwise(to_dev(W))
    assert np.array_equal(to_host(Wq), Wq_o) and np.array_equal(to_host(sW), sW_o)
    Y = i8.int8_mixed_linear(to_dev(X), Wq, sW, to_dev(W), alpha)
    torch.cuda.synchronize()
    Y_o, Ypre_o, _, cnt = orc.mixed_linear(X, Wq_o, sW_o, W, alpha)
    assert_y_close(to_host(Y), Y_o, f"T={T} K={K} N={N} |O|={cnt}")
    assert device_status_clean()


SCHEDULE_CASES = [
    # prefill shapes with more tiles than SMs, so CTAs walk several tiles and
    # the outlier blocks of one tile are issued inside the next one
    (2048, 256, 4096, list(range(0, 256, 4)) + [255], 6.0),     # K < 4 k-blocks, |O| = 65: two blocks
    (2048, 1024, 4096, list(range(0, 1024, 15)), 6.0),         # |O| = 69
    (2200, 640, 3856, [7], 6.0),                               # ragged T, N; one outlier
    (2048, 1024, 4096, [], 6.0),                               # no outliers: single-pass epilogue
    # long schedules: every stage is reused after outlier stages many times over
    (2048, 2048, 8192, [5, 900, 2047], 6.0),                   # 3-4 tiles per CTA pair, 16 k-blocks
    (3000, 1024, 16384, list(range(3, 1024, 15)), 6.0),        # ~10 tiles per pair, |O| = 69
    (2048, 1024, 4096, list(range(0, 1024, 3)), 6.0),          # |O| = 342: compacted + gathered blocks
]


@pytest.mark.parametrize("T,K,N,cols,alpha", SCHEDULE_CASES)
def test_prefill_schedule_matches_oracle(orc, T, K, N, cols, alpha):
    rng = np.random.default_rng(T + 5 * K + N)
    X = outlier_x(rng, T, K, cols)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    Wq_o, sW_o = orc.quantize_weight_colwise(W)
    Wq, sW = i8.int8_quantize_weight_colwise(to_dev(W))
    Y = to_host(i8.int8_mixed_linear(to_dev(X), Wq, sW, to_dev(W), alpha))
    rows = np.arange(0, T, 7, dtype=np.int32)              # rows are independent given O
    Y_o, _, _, cnt = orc.mixed_linear(X, Wq_o, sW_o, W, alpha, rows=rows)
    assert cnt == len(cols)
    assert_y_close(Y[rows], Y_o, f"T={T} K={K} N={N} |O|={cnt}")
    assert np.all(np.isfinite(Y.astype(np.float32)))
    assert device_status_clean()


DECODE_SCHEDULE_CASES = [
    # decode shapes whose CTAs run many more stages than the weight ring holds,
    # with outlier segments in between: the ring and the outlier buffer are
    # each reused many times over
    (16, 4096, 12288, list(range(5, 4096, 600)), 6.0),           # |O| = 7, ~10 stages per CTA
    (1, 4096, 12288, list(range(0, 4096, 31)), 6.0),             # |O| = 133: three outlier blocks per tile
    (128, 4096, 8192, list(range(3, 4096, 57)), 6.0),            # T = 128, three-stage ring, |O| = 72
    (64, 2048, 8192, [], 0.0),                                   # alpha = 0: 32 outlier blocks per tile
    # more outlier columns than one 256-rank window of the row compaction:
    (16, 12288, 4096, list(range(0, 12288, 24)), 6.0),          # |O| = 512: 256 compacted rows + 4 gathered blocks
    (8, 49152, 1024, list(range(0, 49152, 97)), 6.0),           # |O| = 507 of 768 compacted rows (two windows)
    (1, 16384, 2048, list(range(0, 16384, 40)), 6.0),           # |O| = 410, row quantiser's compaction blocks
]


@pytest.mark.parametrize("T,K,N,cols,alpha", DECODE_SCHEDULE_CASES)
@pytest.mark.parametrize("variant", ["w16", "wq"])
def test_decode_schedule_matches_oracle(orc, T, K, N, cols, alpha, variant):
    rng = np.random.default_rng(T + 3 * K + N)
    X = outlier_x(rng, T, K, cols)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    Wq_o, sW_o = orc.quantize_weight_colwise(W)
    Wq, sW = i8.int8_quantize_weight_colwise(to_dev(W))
    if variant == "w16":
        Y = to_host(i8.int8_mixed_linear(to_dev(X), Wq, sW, to_dev(W), alpha))
    else:
        Y = to_host(i8.int8_mixed_linear_wq(to_dev(X), Wq, sW, alpha))
    rows = np.unique(np.r_[0:T:5, T - 1]).astype(np.int32)
    Y_o, _, _, cnt = orc.mixed_linear(X, Wq_o, sW_o, W if variant == "w16" else None, alpha, rows=rows)
    assert cnt == (K if alpha == 0.0 else len(cols))
    assert_y_close(Y[rows], Y_o, f"{variant} T={T} K={K} N={N} |O|={cnt}")
    assert device_status_clean()


def test_exact_integer_case_is_exact(orc):
    """alpha = +inf with integer inputs whose row / column absmax is 127: the
    codes are the inputs, and Y is the exact integer product (kept within
    +-2048, where fp16 holds every integer)."""
    rng = np.random.default_rng(5)
    for T in (16, 200):
        K, N = 128, 272
        X = rng.integers(-3, 4, (T, K)).astype(np.float16)
        X[:, 0] = 127                                 # row absmax 127 ...
        X[:, 1] = 0
        W = rng.integers(-3, 4, (K, N)).astype(np.float16)
        W[1, :] = -127                                # ... column absmax 127, and the two
        W[0, :] = 0                                   # 127s only ever meet zeros
        Wq, sW = i8.int8_quantize_weight_colwise(to_dev(W))
        assert np.array_equal(to_host(Wq), W.astype(np.int8))
        Y = i8.int8_mixed_linear(to_dev(X), Wq, sW, to_dev(W), float("inf"))
        exact = X.astype(np.int64) @ W.astype(np.int64)
        assert np.abs(exact).max() <= 2048
        Y_o, _, _, _ = orc.mixed_linear(X, to_host(Wq), to_host(sW), W, float("inf"))
        assert np.array_equal(to_host(Y).astype(np.int64), exact)
        assert np.array_equal(Y_o.astype(np.int64), exact)


def test_repeat_runs_are_bit_identical():
    rng = np.random.default_rng(17)
    for T in (16, 300):
        X = outlier_x(rng, T, 1024, [9, 77])
        W = (rng.standard_normal((1024, 512)) * 0.02).astype(np.float16)
        Wq, sW = i8.int8_quantize_weight_colwise(to_dev(W))
        Xd, Wd = to_dev(X), to_dev(W)
        ws = i8.workspace(T, 1024, 512)
        a = to_host(i8.int8_mixed_linear(Xd, Wq, sW, Wd, 6.0, workspace_buf=ws))
        ws.fill_(0xAB)                              # stale workspace contents must not matter
        b = to_host(i8.int8_mixed_linear(Xd, Wq, sW, Wd, 6.0, workspace_buf=ws))
        assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_mixed_linear_t0_is_noop():
    Wq = torch.zeros((64, 16), dtype=torch.int8, device="cuda")
    sW = torch.zeros(16, dtype=torch.float32, device="cuda")
    W16 = torch.zeros((64, 16), dtype=torch.float16, device="cuda")
    Y = i8.int8_mixed_linear(torch.zeros((0, 64), dtype=torch.float16, device="cuda"), Wq, sW, W16, 6.0)
    assert Y.shape == (0, 16)


# ------------------------------------------------------------------ statistics

@pytest.mark.parametrize("T,K,cols,alpha", ACT_CASES[:6])
def test_outlier_stats_match_oracle(orc, T, K, cols, alpha):
    rng = np.random.default_rng(T + K)
    X = outlier_x(rng, T, K, cols, row_prob=0.5)
    count, idx, hits, frac = i8.int8_outlier_stats(to_dev(X), alpha)
    torch.cuda.synchronize()
    _, idx_o = orc.outlier_columns(X, alpha)
    c = int(to_host(count)[0])
    assert c == len(idx_o)
    assert np.array_equal(to_host(idx)[:c], idx_o)
    assert np.array_equal(to_host(hits), orc.outlier_hits(X, alpha))
    assert to_host(frac)[0] == np.float32(orc.frac_8bit(c, K))


# ------------------------------------------------------------------ failure detection

def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait on a barrier nothing completes gives up after its limit and
    records the timeout code; the GPU keeps working afterwards."""
    assert i8.int8_read_and_clear_device_status() == 0
    i8.int8_selftest_wait_timeout(2000)            # 2 ms
    assert i8.int8_read_and_clear_device_status() == 1
    assert i8.int8_read_and_clear_device_status() == 0   # read clears it
    # the context is still usable
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0
    acc = i8.int8_gemm_i8_s32(torch.ones((4, 64), dtype=torch.int8, device="cuda"),
                              torch.ones((64, 16), dtype=torch.int8, device="cuda"))
    assert int(acc.min()) == 64 and int(acc.max()) == 64
