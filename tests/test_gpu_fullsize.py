"""CUDA path vs the CPU oracle at the full workload sizes, in the launch
configuration the benchmark times (one int8_mixed_linear call on the whole
batch).  The oracle cannot produce every row of these outputs quickly, so:
  - the outlier set (which depends on every row) is compared in full;
  - weight codes and scales are compared in full, bit for bit;
  - row codes / scales and the int32 accumulators are compared bit for bit on
    sampled rows (first, last and a seeded spread);
  - Y is compared on the same rows with the Y tolerance.
Rows of Y are independent once the outlier set and the weight scales are
fixed, so sampled rows are checked exactly as the full output would be.
"""
import numpy as np
import pytest
import torch

import int8_quantized_row_b200 as i8
from int8_quantized_row_b200 import workloads as wl
from gpu_helpers import assert_y_close, device_status_clean, to_dev, to_host

pytestmark = pytest.mark.gpu


def sample_rows(T, n=6, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, T - 1} | set(rng.integers(0, T, n).tolist())
    return np.array(sorted(rows), np.int32)


class Layer:
    """One weight (generated once per test module) on host and device."""

    def __init__(self, orc, K, N, sigma, seed=0):
        self.W = wl.make_w(K, N, sigma, seed)
        self.Wd = to_dev(self.W)
        self.Wq, self.sW = i8.int8_quantize_weight_colwise(self.Wd)
        torch.cuda.synchronize()
        self.Wq_o, self.sW_o = orc.quantize_weight_colwise(self.W)


def check_layer_call(orc, layer, X, alpha, rows):
    Xd = to_dev(X)
    T, K = X.shape
    Y = i8.int8_mixed_linear(Xd, layer.Wq, layer.sW, layer.Wd, alpha)
    act = i8.int8_quantize_activation(Xd, alpha, with_xo=False)
    torch.cuda.synchronize()
    # outlier set over all rows
    mask_o, idx_o = orc.outlier_columns(X, alpha)
    cnt = int(to_host(act["count"])[0])
    assert cnt == len(idx_o) and np.array_equal(to_host(act["idx"])[:cnt], idx_o)
    # row codes and scales, sampled rows
    Xq_o, sX_o = orc.quantize_rows(X[rows], mask_o)
    Xq = to_host(act["Xq"])[rows]
    assert np.array_equal(Xq, Xq_o) and np.array_equal(to_host(act["sX"])[rows], sX_o)
    # int32 accumulators of those rows, through the tensor-core GEMM (same
    # kernel variant as the full call: it is chosen by T)
    acc = i8.int8_gemm_i8_s32(act["Xq"][:T], layer.Wq)
    acc_rows = to_host(acc[torch.from_numpy(rows).long().cuda()])
    del acc
    Y_o, _, acc_o, _ = orc.mixed_linear(X, layer.Wq_o, layer.sW_o, layer.W, alpha, rows=rows)
    assert np.array_equal(acc_rows, acc_o)
    assert_y_close(to_host(Y)[rows], Y_o, f"T={T} K={K} |O|={cnt}")
    assert device_status_clean()
    return cnt


NAMED = ["single_linear_16x1024x1024", "opt13b_fc1_prefill_2048x5120x20480",
         "b175_fc1_decode_t1_12288x49152", "b175_fc1_decode_t8_12288x49152",
         "b175_fc1_decode_t16_12288x49152", "b175_qkv_prefill_4096x12288x36864"]

_layers = {}


def _layer(orc, cfg):
    key = (cfg["K"], cfg["N"], cfg["w_sigma"], cfg["seed"])
    if key not in _layers:
        _layers.clear()                           # keep one weight resident at a time
        torch.cuda.empty_cache()
        _layers[key] = Layer(orc, *key)
    return _layers[key]


@pytest.mark.parametrize("name", NAMED)
def test_named_workload(orc, name):
    cfg = wl.CONFIGS[name]
    layer = _layer(orc, cfg)
    assert np.array_equal(to_host(layer.Wq), layer.Wq_o)
    assert np.array_equal(to_host(layer.sW), layer.sW_o)
    X, _ = wl.generate(cfg, with_w=False)
    rows = sample_rows(cfg["T"])
    cnt = check_layer_call(orc, layer, X, cfg["alpha"], rows)
    planted = set(wl.planted_columns(cfg["K"], cfg["n_out"], cfg["seed"]).tolist())
    assert cnt >= len(planted) if cfg["row_prob"] == 1.0 else cnt >= 0


SWEEP = wl.sweep_configs()


@pytest.mark.parametrize("name", sorted(SWEEP, key=lambda n: (SWEEP[n]["K"], SWEEP[n]["N"], n)))
def test_layer_sweep(orc, name):
    cfg = SWEEP[name]
    layer = _layer(orc, cfg)
    X, _ = wl.generate(cfg, with_w=False)
    rows = sample_rows(cfg["T"], n=2, seed=cfg["T"])
    cnt = check_layer_call(orc, layer, X, cfg["alpha"], rows)
    if cfg["alpha"] == float("inf"):
        assert cnt == 0
    else:
        assert cnt >= cfg["n_out"]
