"""Shared helpers for the GPU parity tests: run the CUDA path through the
Python binding (which calls the C ABI) and compare with the CPU oracle."""
import numpy as np
import torch

import int8_quantized_row_b200 as i8

# Y tolerance: relative L2 error <= 1e-3 and max abs error <= 2^-8 max|Y_oracle|
REL_L2 = 1e-3
MAX_ABS_FRAC = 2.0 ** -8


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host(t):
    return t.detach().cpu().numpy()


def y_errors(y_gpu, y_orc):
    g = y_gpu.astype(np.float64)
    o = y_orc.astype(np.float64)
    assert np.all(np.isfinite(g)), "non-finite output"
    rel = np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30)
    mx = np.abs(g - o).max() if g.size else 0.0
    bound = MAX_ABS_FRAC * (np.abs(o).max() if o.size else 0.0)
    return rel, mx, bound


def assert_y_close(y_gpu, y_orc, what=""):
    rel, mx, bound = y_errors(y_gpu, y_orc)
    assert rel <= REL_L2, f"{what}: relative L2 error {rel:.3e} > {REL_L2}"
    assert mx <= bound, f"{what}: max abs error {mx:.3e} > {bound:.3e}"


def device_status_clean():
    return i8.int8_read_and_clear_device_status() == 0


def outlier_x(rng, T, K, cols, lo=6.0, hi=60.0, row_prob=1.0):
    """N(0,1) activation with planted outlier columns (test-local shapes)."""
    X = rng.standard_normal((T, K), dtype=np.float32)
    for c in cols:
        hit = rng.random(T) < row_prob
        X[hit, c] = rng.uniform(lo, hi, hit.sum()) * rng.choice([-1.0, 1.0], hit.sum())
    return X.astype(np.float16)
