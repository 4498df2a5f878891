"""The group-wise 4-bit weight codec and its decode-shaped product against the
oracle (GPU).

Bit-exact: the codes, the binary16 step s and base lo of every group (read
back through the packed layout of include/int8row.h), and the decoded weight.
Tolerance on Y (the same bound as the int8 layer: relative L2 <= 1e-3, max
abs <= 2^-8 max|Y_oracle|): the oracle sums in double, the kernel in fp32.
Shapes span several 256-column tiles, tiles split over several CTAs, ragged
column counts (padding), T from 1 to the limit of 64, and groups that are
constant, all zero or hold signed zeros.
"""
import numpy as np
import pytest
import torch

import int8_quantized_row_b200 as i8
import int4_layout as L
from gpu_helpers import assert_y_close, device_status_clean, to_dev, to_host

pytestmark = pytest.mark.gpu


def _weights(rng, K, N, sigma=0.02):
    W = (rng.standard_normal((K, N)) * sigma).astype(np.float16)
    W[0:64, 0] = np.float16(0.5)                         # a constant group: s = 0
    W[64:128, 1] = 0                                     # an all-zero group
    W[0:64, 2] = np.where(np.arange(64) % 2 == 0, np.float16(0.0), np.float16(-0.0))   # signed zeros
    W[128:192, 3] = (rng.standard_normal(64) * 40).astype(np.float16)                 # a wide group
    if N > 4:
        # exact halfway points: step 1/16, base 0, w - lo = (k + 1/2) * s
        tie = np.zeros(64)
        tie[1] = 15.0
        tie[2:17] = np.arange(15) + 0.5
        W[0:64, 4] = (tie / 16.0).astype(np.float16)
    return W


@pytest.mark.parametrize("K,N", [(256, 16), (512, 272), (1024, 1024), (12288, 768)])
def test_int4_codec_bit_exact(orc, K, N):
    rng = np.random.default_rng(K + N)
    W = _weights(rng, K, N)
    codes_o, s_o, lo_o = orc.int4_quantize_groupwise(W)
    W4, S4 = i8.int4_quantize_weight_groupwise(to_dev(W))
    torch.cuda.synchronize()
    W4h, S4h = to_host(W4), to_host(S4)
    codes, s, lo = L.unpack(W4h, S4h, K, N)
    assert np.array_equal(codes, codes_o)
    assert np.array_equal(s.view(np.uint16), s_o.view(np.uint16))
    assert np.array_equal(lo.view(np.uint16), lo_o.view(np.uint16))
    # padding columns are zero codes and zero (s, lo)
    pw, ps = L.pack(codes_o, s_o, lo_o)
    assert np.array_equal(W4h, pw) and np.array_equal(S4h, ps)
    Wd = to_host(i8.int4_dequantize_weight(W4, S4, K, N))
    Wd_o = orc.int4_dequantize(codes_o, s_o, lo_o)
    assert np.array_equal(Wd.view(np.uint16), Wd_o.view(np.uint16))
    assert device_status_clean()


def test_int4_codec_every_fp16_value(orc):
    """Every finite fp16 value passes through the codec (in groups of 64)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    vals = bits[np.isfinite(bits)]
    N = 64
    K = (len(vals) + N - 1) // N // 256 * 256 + 256
    W = np.zeros(K * N, np.float16)
    W[:len(vals)] = vals
    W = W.reshape(K, N)
    codes_o, s_o, lo_o = orc.int4_quantize_groupwise(W)
    W4, S4 = i8.int4_quantize_weight_groupwise(to_dev(W))
    codes, s, lo = L.unpack(to_host(W4), to_host(S4), K, N)
    assert np.array_equal(codes, codes_o)
    assert np.array_equal(s.view(np.uint16), s_o.view(np.uint16))
    assert np.array_equal(lo.view(np.uint16), lo_o.view(np.uint16))
    Wd = to_host(i8.int4_dequantize_weight(W4, S4, K, N))
    assert np.array_equal(Wd.view(np.uint16), orc.int4_dequantize(codes_o, s_o, lo_o).view(np.uint16))


LINEAR_CASES = [
    # T, K, N
    (1, 256, 16),
    (3, 512, 272),          # ragged N: one padded tile
    (16, 1024, 1024),
    (17, 2048, 528),
    (64, 1024, 256),        # the largest T
    (8, 12288, 2048),       # tiles split over several CTAs
    (1, 4096, 12288),
    (33, 4096, 4096),
]


@pytest.mark.parametrize("T,K,N", LINEAR_CASES)
def test_int4_linear_matches_oracle(orc, T, K, N):
    rng = np.random.default_rng(T * 31 + K + N)
    X = rng.standard_normal((T, K)).astype(np.float16)
    W = _weights(rng, K, N)
    W4, S4 = i8.int4_quantize_weight_groupwise(to_dev(W))
    Y = to_host(i8.int4_linear(to_dev(X), W4, S4, N))
    codes_o, s_o, lo_o = orc.int4_quantize_groupwise(W)
    Y_o, _ = orc.int4_linear(X, codes_o, s_o, lo_o)
    assert_y_close(Y, Y_o, f"int4 T={T} K={K} N={N}")
    assert device_status_clean()


SMALL_CASES = [
    # T, K, N: the CUDA-core product (T <= 4), each checked on both products
    (1, 256, 16),
    (2, 512, 272),          # ragged N
    (3, 1024, 1024),
    (4, 2048, 528),
    (1, 12288, 2048),       # tiles split over several CTAs
    (4, 4096, 12288),
    (2, 49152, 256),        # one tile over every CTA
]


@pytest.mark.parametrize("T,K,N", SMALL_CASES)
def test_int4_cuda_core_and_tensor_products_match_oracle(orc, T, K, N):
    """Both products (int4_debug_set_product_path 2: CUDA cores, 1: tensor
    cores) against the oracle, and against each other: the same decoded
    weights and exact fp16 products, fp32 sums in different orders."""
    rng = np.random.default_rng(T * 131 + K + N)
    X = rng.standard_normal((T, K)).astype(np.float16)
    W = _weights(rng, K, N)
    W4, S4 = i8.int4_quantize_weight_groupwise(to_dev(W))
    Xd = to_dev(X)
    codes_o, s_o, lo_o = orc.int4_quantize_groupwise(W)
    Y_o, _ = orc.int4_linear(X, codes_o, s_o, lo_o)
    out = {}
    try:
        for mode in (2, 1):
            i8.int4_debug_set_product_path(mode)
            out[mode] = to_host(i8.int4_linear(Xd, W4, S4, N))
            assert_y_close(out[mode], Y_o, f"int4 path {mode} T={T} K={K} N={N}")
            assert device_status_clean()
    finally:
        i8.int4_debug_set_product_path(0)
    assert_y_close(out[2], out[1].astype(np.float64), f"int4 paths T={T} K={K} N={N}")


@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_int4_cuda_core_product_exact_integers(T):
    """Integer activations and exact 4-bit grids on the CUDA-core product:
    every product and partial sum is exact in fp32, so Y is exact."""
    rng = np.random.default_rng(70 + T)
    K, N = 2048, 768
    Q = rng.integers(0, 16, (K, N))
    Q[0::64] = 0
    Q[1::64] = 15
    W = (Q - 7).astype(np.float16)
    X = rng.integers(-2, 3, (T, K)).astype(np.float16)
    W4, S4 = i8.int4_quantize_weight_groupwise(to_dev(W))
    try:
        i8.int4_debug_set_product_path(2)
        Y = to_host(i8.int4_linear(to_dev(X), W4, S4, N)).astype(np.int64)
    finally:
        i8.int4_debug_set_product_path(0)
    exact = X.astype(np.int64) @ (Q - 7)
    assert np.abs(exact).max() <= 2048
    assert np.array_equal(Y, exact)


def test_int4_cuda_core_product_is_deterministic():
    rng = np.random.default_rng(12)
    T, K, N = 2, 12288, 4096                 # tiles split over CTAs: pieces added in CTA order
    X = to_dev(rng.standard_normal((T, K)).astype(np.float16))
    W4, S4 = i8.int4_quantize_weight_groupwise(to_dev((rng.standard_normal((K, N)) * 0.01).astype(np.float16)))
    a = to_host(i8.int4_linear(X, W4, S4, N))
    b = to_host(i8.int4_linear(X, W4, S4, N))
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


@pytest.mark.parametrize("T", [16, 64])
def test_int4_linear_exact_integers(orc, T):
    """Integer activations and weights on exact 4-bit grids: every product and
    partial sum is exact in fp32, so Y is the exact integer product."""
    rng = np.random.default_rng(7 + T)
    K, N = 1024, 512
    Q = rng.integers(0, 16, (K, N))
    Q[0::64] = 0
    Q[1::64] = 15
    W = (Q - 7).astype(np.float16)                       # s = 1, lo = -7 in every group
    X = rng.integers(-2, 3, (T, K)).astype(np.float16)
    W4, S4 = i8.int4_quantize_weight_groupwise(to_dev(W))
    Y = to_host(i8.int4_linear(to_dev(X), W4, S4, N)).astype(np.int64)
    exact = X.astype(np.int64) @ (Q - 7)
    assert np.abs(exact).max() <= 2048
    assert np.array_equal(Y, exact)


def test_int4_linear_is_deterministic():
    rng = np.random.default_rng(11)
    T, K, N = 16, 12288, 4096
    X = to_dev(rng.standard_normal((T, K)).astype(np.float16))
    W4, S4 = i8.int4_quantize_weight_groupwise(to_dev((rng.standard_normal((K, N)) * 0.01).astype(np.float16)))
    a = to_host(i8.int4_linear(X, W4, S4, N))
    b = to_host(i8.int4_linear(X, W4, S4, N))
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_int4_linear_t0_and_limits():
    W4 = torch.zeros(i8.int4_packed_code_bytes(256, 16), dtype=torch.uint8, device="cuda")
    S4 = torch.zeros(i8.int4_packed_scale_bytes(256, 16), dtype=torch.uint8, device="cuda")
    Y = i8.int4_linear(torch.zeros((0, 256), dtype=torch.float16, device="cuda"), W4, S4, 16)
    assert Y.shape == (0, 16)
    with pytest.raises(i8.I8RError):
        i8.int4_linear(torch.zeros((65, 256), dtype=torch.float16, device="cuda"), W4, S4, 16)


@pytest.mark.parametrize("T", [1, 16])
def test_int4_full_size_fc1_decode(orc, T):
    """The 175B fc1 shape (K=12288, N=49152; 302 MB of packed codes) at T=1 (the
    CUDA-core product) and T=16 (the tensor cores), in the launch configuration
    the sweep times: every group's (s, lo) bit for bit, and Y on sampled rows
    within the tolerance."""
    from int8_quantized_row_b200 import workloads as wl
    K, N = 12288, 49152
    W = wl.make_w(K, N, 0.01)
    X = wl.make_x(T, K, 0, seed=T)
    W4, S4 = i8.int4_quantize_weight_groupwise(to_dev(W))
    Y = to_host(i8.int4_linear(to_dev(X), W4, S4, N))
    codes_o, s_o, lo_o = orc.int4_quantize_groupwise(W)
    NP, KT = L.padded_n(N), K // 256
    sl = to_host(S4).reshape(NP // 256, KT, 256, 4, 2, 2).view("<u2")[..., 0].transpose(1, 3, 0, 2, 4).reshape(K // 64, NP, 2)
    assert np.array_equal(sl[:, :N, 0], s_o.view(np.uint16))
    assert np.array_equal(sl[:, :N, 1], lo_o.view(np.uint16))
    rows = np.array(sorted({0, T // 2, T - 1}), np.int32)
    Y_o, _ = orc.int4_linear(X, codes_o, s_o, lo_o, rows=rows)
    assert_y_close(Y[rows], Y_o, f"int4 fc1 T={T} full size")
    assert device_status_clean()
