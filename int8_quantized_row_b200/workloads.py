"""Seeded synthetic workloads for the int8 mixed-precision linear layer.

This module only draws inputs; it holds none of the method's arithmetic
(no quantisation, no outlier rule, no matmul).  The tests, the smoke check,
the benchmark and the CPU oracle's callers all take their inputs from here,
so the CUDA path and the oracle always see the same bytes.

Recipe (stand-in for activations and weights of OPT-13B / 175B-class models,
which are not available):
  * X ~ N(0, 1) drawn in fp32 and rounded to fp16 (round-to-nearest-even);
  * ``n_out`` planted outlier columns, chosen by seeded sampling without
    replacement; in each, every row (``row_prob`` = 1) or each row
    independently with probability ``row_prob`` gets sign * U(lo, hi), the
    sign +-1 with probability 1/2, replacing the base value;
  * W16 ~ N(0, sigma) drawn in fp32 and rounded to fp16.
Random streams are counter-based (numpy's Philox) with a key built from
(seed, tensor tag, row block), so any block of rows can be regenerated on
its own and blocks can be drawn in parallel.
"""
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

_TAG_X, _TAG_W, _TAG_COLS, _TAG_ROWS, _TAG_VALS = 1, 2, 3, 4, 5
_BLOCK_ROWS = 256


def _rng(seed, tag, block=0):
    key = (int(seed) << 64) | (int(tag) << 32) | int(block)
    return np.random.Generator(np.random.Philox(key=key))


def _normal_fp16(rows, cols, sigma, seed, tag, row0=0, row1=None):
    """N(0, sigma) fp16 matrix [rows, cols], or only its rows [row0, row1)."""
    row1 = rows if row1 is None else row1
    out = np.empty((row1 - row0, cols), np.float16)
    blocks = range(row0 // _BLOCK_ROWS, (row1 + _BLOCK_ROWS - 1) // _BLOCK_ROWS)

    def fill(b):
        r0, r1 = b * _BLOCK_ROWS, min((b + 1) * _BLOCK_ROWS, rows)
        z = _rng(seed, tag, b).standard_normal((r1 - r0, cols), dtype=np.float32)
        if sigma != 1.0:
            z *= np.float32(sigma)
        lo, hi = max(r0, row0), min(r1, row1)
        out[lo - row0:hi - row0] = z[lo - r0:hi - r0].astype(np.float16)

    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, blocks))
    return out


def planted_columns(K, n_out, seed):
    """The planted outlier columns, ascending."""
    if n_out <= 0:
        return np.zeros(0, np.int64)
    return np.sort(_rng(seed, _TAG_COLS).choice(K, size=n_out, replace=False))


def make_x(T, K, n_out=0, lo=6.0, hi=60.0, row_prob=1.0, seed=0, rows=None):
    """Activation X fp16 [T, K] (or only ``rows``, a (start, stop) pair)."""
    r0, r1 = (0, T) if rows is None else rows
    X = _normal_fp16(T, K, 1.0, seed, _TAG_X, r0, r1)
    cols = planted_columns(K, n_out, seed)
    if len(cols):
        for b in range(r0 // _BLOCK_ROWS, (r1 + _BLOCK_ROWS - 1) // _BLOCK_ROWS):
            b0, b1 = b * _BLOCK_ROWS, min((b + 1) * _BLOCK_ROWS, T)
            g_rows = _rng(seed, _TAG_ROWS, b)
            g_vals = _rng(seed, _TAG_VALS, b)
            hit = (g_rows.random((b1 - b0, len(cols))) < row_prob) if row_prob < 1.0 \
                else np.ones((b1 - b0, len(cols)), bool)
            mag = g_vals.uniform(lo, hi, (b1 - b0, len(cols))).astype(np.float32)
            sign = np.where(g_vals.random((b1 - b0, len(cols))) < 0.5, -1.0, 1.0).astype(np.float32)
            vals = (sign * mag).astype(np.float16)
            s0, s1 = max(b0, r0), min(b1, r1)
            for j, c in enumerate(cols):
                sel = hit[s0 - b0:s1 - b0, j]
                blockvals = vals[s0 - b0:s1 - b0, j]
                X[s0 - r0:s1 - r0, c] = np.where(sel, blockvals, X[s0 - r0:s1 - r0, c])
    return X


def make_w(K, N, sigma, seed=0):
    """Weight W16 fp16 [K, N] ~ N(0, sigma)."""
    return _normal_fp16(K, N, float(sigma), seed, _TAG_W)


# --------------------------------------------------------------------------
# Named workloads.  Shapes are (T, K, N): X [T,K] @ W [K,N] -> Y [T,N].
# --------------------------------------------------------------------------

def _cfg(T, K, N, w_sigma, n_out, lo, hi, row_prob, alpha=6.0, seed=0):
    return dict(T=T, K=K, N=N, w_sigma=w_sigma, n_out=n_out, lo=lo, hi=hi,
                row_prob=row_prob, alpha=alpha, seed=seed)


CONFIGS = {
    # one 1024 -> 1024 linear at 16 tokens, 2 outlier columns in every row
    "single_linear_16x1024x1024": _cfg(16, 1024, 1024, 0.02, 2, 6.0, 20.0, 1.0),
    # OPT-13B-shaped FFN fc1 at prefill: 6 outlier columns (0.12%) in 25% of rows
    "opt13b_fc1_prefill_2048x5120x20480": _cfg(2048, 5120, 20480, 0.02, 6, 6.0, 60.0, 0.25),
    # 175B-shaped fc1 at decode sizes (T in {1, 8, 16}), 7 outlier columns
    "b175_fc1_decode_t1_12288x49152": _cfg(1, 12288, 49152, 0.01, 7, 6.0, 60.0, 1.0),
    "b175_fc1_decode_t8_12288x49152": _cfg(8, 12288, 49152, 0.01, 7, 6.0, 60.0, 1.0),
    "b175_fc1_decode_t16_12288x49152": _cfg(16, 12288, 49152, 0.01, 7, 6.0, 60.0, 1.0),
    # 175B-shaped QKV projection at prefill: 0.1% outlier columns in every row
    "b175_qkv_prefill_4096x12288x36864": _cfg(4096, 12288, 36864, 0.01, 12, 6.0, 60.0, 1.0),
}

# 175B decoder-layer sweep: four projections x T x outlier fraction x alpha.
SWEEP_LAYERS = {"qkv": (12288, 36864), "out": (12288, 12288),
                "fc1": (12288, 49152), "fc2": (49152, 12288)}
SWEEP_T = (1, 16, 128, 2048)
SWEEP_FRAC = (0.0, 0.001, 0.01)
SWEEP_ALPHA = (6.0, float("inf"))


def sweep_configs():
    out = {}
    for layer, (K, N) in SWEEP_LAYERS.items():
        for T in SWEEP_T:
            for frac in SWEEP_FRAC:
                for alpha in SWEEP_ALPHA:
                    name = f"b175_sweep_{layer}_t{T}_f{frac:g}_a{alpha:g}"
                    out[name] = _cfg(T, K, N, 0.01, int(round(frac * K)), 6.0, 60.0, 1.0, alpha)
    return out


def generate(cfg, x_rows=None, with_w=True):
    """Draw (X, W16) for a config dict; W16 is None when ``with_w`` is False."""
    X = make_x(cfg["T"], cfg["K"], cfg["n_out"], cfg["lo"], cfg["hi"], cfg["row_prob"],
               cfg["seed"], rows=x_rows)
    W = make_w(cfg["K"], cfg["N"], cfg["w_sigma"], cfg["seed"]) if with_w else None
    return X, W
