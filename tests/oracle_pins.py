"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with what the pages or the mathematics fix:
hand-worked values, library routines (numpy's binary16 conversion, numpy's
int64 / float64 matmul, Python's decimal rounding), closed forms, invariants
and brute force on tiny inputs.  They are collected by ``test_oracle_pins``
for the committed oracle, and by ``test_oracle_mutants`` for copies of the
oracle with planted mistakes, each of which some pin must catch.
"""
from decimal import Decimal, ROUND_HALF_UP
from fractions import Fraction
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _all_finite_halves():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    h = bits.view(np.float16)
    return h[np.isfinite(h)]


def _rhaz_exact(v):
    """Round half away from zero of the exact binary value of v (decimal)."""
    return int(Decimal(float(v)).quantize(Decimal(1), rounding=ROUND_HALF_UP))


# ---------------------------------------------------------------- conversions

def pin_half_decode_exhaustive(o):
    """Every binary16 code decodes like numpy's float16 (a library routine)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([o.half_to_float(int(b)) for b in bits], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def pin_half_encode(o):
    """double -> binary16 rounds to nearest-even like numpy's conversion."""
    rng = np.random.default_rng(1234)
    vals = [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0**-24, 2.0**-25,
            2.0**-25 * 1.0000001, 3 * 2.0**-25, 2.0**-14, 2.0**-14 - 2.0**-25]
    fin = _all_finite_halves().astype(np.float64)
    fin = np.unique(fin)
    mids = (fin[:-1] + fin[1:]) / 2.0                 # exact ties
    vals += list(mids[::7]) + list(np.nextafter(mids[::11], np.inf))
    vals += list(np.nextafter(mids[::13], -np.inf))
    vals += list(rng.standard_normal(4000) * 10.0 ** rng.integers(-8, 5, 4000))
    vals = np.array(vals, np.float64)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([o.double_to_half(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, ref), vals[got != ref][:8]


def pin_rhaz(o):
    """rhaz agrees with decimal ROUND_HALF_UP (ties away from zero)."""
    vs = []
    for k in list(range(-130, 131)) + [1 << 20, -(1 << 20), 8388607]:
        for f in (0.0, 0.25, 0.5, 0.75, 0.49999997, 0.50000006):
            vs += [np.float32(k + f), np.float32(k - f)]
    vs += list(np.float32(np.random.default_rng(5).uniform(-200, 200, 5000)))
    for v in vs:
        assert o.rhaz(float(v)) == _rhaz_exact(v), v


# ---------------------------------------------------------------- quantisers

def pin_quantizer_all_halves(o):
    """Every finite fp16 x, quantised in a row whose absmax is s (s >= |x|),
    lands within 1/2 (+ fp32 rounding) of the exact 127 x / s, ties away from
    zero; codes are odd-symmetric and stay inside [-127, 127]."""
    xs = _all_finite_halves()
    pos = np.unique(np.abs(xs))[1:]
    scales = [np.float16(1.0), np.float16(3.0), np.float16(0.1), np.float16(65504.0),
              np.float16(6.1e-5)] + list(pos[::50])
    for s in scales:
        x = xs[np.abs(xs.astype(np.float32)) <= np.float32(s)]
        X = np.stack([x, np.full_like(x, s)], axis=1)          # row absmax = s
        Xq, sX = o.quantize_rows(X, np.zeros(2, bool))
        assert np.all(sX == np.float32(s))
        q = Xq[:, 0].astype(np.int64)
        exact = 127.0 * x.astype(np.float64) / float(s)
        assert np.all(np.abs(q - exact) <= 0.5 + 127 * 2.0 ** -22), s
        assert np.all(Xq[:, 1] == 127)
        # library recomputation: the fp32 reciprocal and product by numpy's IEEE
        # float32 arithmetic, then half-away rounding of that exact fp32 value
        # as sign * floor(|v| + 1/2) in float64 (exact for fp32 inputs) for
        # every element, and by decimal ROUND_HALF_UP for a sample
        inv = np.float32(127.0) / np.float32(s)
        v = (x.astype(np.float32) * inv).astype(np.float32)
        v64 = v.astype(np.float64)
        lib = (np.sign(v64) * np.floor(np.abs(v64) + 0.5)).astype(np.int64)
        assert np.array_equal(np.clip(lib, -127, 127), q), s
        dec = np.array([_rhaz_exact(t) for t in v[::997]], np.int64)
        assert np.array_equal(np.clip(dec, -127, 127), q[::997])
        # odd symmetry
        Xn, _ = o.quantize_rows(-X, np.zeros(2, bool))
        assert np.array_equal(Xn[:, 0].astype(np.int64), -q)


def pin_quantizer_invariants(o):
    rng = np.random.default_rng(7)
    X = rng.standard_normal((64, 96)).astype(np.float16)
    X[np.abs(X) < 2.0 ** -10] = 0          # keep every value normal under the 2^j scalings
    Xq, sX = o.quantize_rows(X, np.zeros(96, bool))
    # absmax element maps to +-127; the scale is the absmax
    am = np.abs(X.astype(np.float32)).max(axis=1)
    assert np.array_equal(sX, am)
    arg = np.abs(X.astype(np.float32)).argmax(axis=1)
    assert np.all(np.abs(Xq[np.arange(64), arg]) == 127)
    # scaling a row by 2^j (no overflow or loss) keeps codes, scales sX exactly
    for j in (-3, 1, 4):
        Xs = (X.astype(np.float32) * 2.0 ** j).astype(np.float16)
        assert np.array_equal(Xs.astype(np.float32), X.astype(np.float32) * 2.0 ** j)
        Xq2, sX2 = o.quantize_rows(Xs, np.zeros(96, bool))
        assert np.array_equal(Xq2, Xq)
        assert np.array_equal(sX2, sX * np.float32(2.0 ** j))
    # idempotence: dequantised codes quantise back to the same codes
    deq = (Xq.astype(np.float64) * sX[:, None].astype(np.float64) / 127.0).astype(np.float16)
    Xq3, _ = o.quantize_rows(deq, np.zeros(96, bool))
    assert np.array_equal(Xq3, Xq)
    # an all-zero row quantises to zeros with scale 0
    Z = np.zeros((2, 96), np.float16)
    Zq, sZ = o.quantize_rows(Z, np.zeros(96, bool))
    assert not Zq.any() and not sZ.any()


def pin_rows_skip_outlier_columns(o):
    """The row scale ignores outlier columns and their codes are 0."""
    X = np.array([[1.0, 40.0, -2.0, 0.5], [0.0, -9.0, 0.0, 0.0]], np.float16)
    mask = np.array([False, True, False, False])
    Xq, sX = o.quantize_rows(X, mask)
    assert list(sX) == [2.0, 0.0]
    assert list(Xq[0]) == [64, 0, -127, 32]
    assert not Xq[1].any()


def pin_weight_colwise(o):
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((80, 48)) * 0.02).astype(np.float16)
    W[:, 5] = 0                                      # an all-zero column
    Wq, sW = o.quantize_weight_colwise(W)
    ref = np.abs(W.astype(np.float32)).max(axis=0)
    assert np.array_equal(sW, ref)
    assert not Wq[:, 5].any() and sW[5] == 0
    nz = ref > 0
    exact = 127.0 * W.astype(np.float64)[:, nz] / ref[nz].astype(np.float64)
    assert np.all(np.abs(Wq[:, nz] - exact) <= 0.5 + 127 * 2.0 ** -22)
    assert np.all(np.abs(Wq).max(axis=0)[nz] == 127)
    # the column quantiser is the row quantiser applied to W's transpose
    WqT, sWT = o.quantize_rows(np.ascontiguousarray(W.T), np.zeros(80, bool))
    assert np.array_equal(WqT.T, Wq) and np.array_equal(sWT, sW)


# ---------------------------------------------------------------- outliers

def _brute_outliers(X, alpha):
    T, K = X.shape
    cols = []
    for k in range(K):
        if any(abs(float(X[t, k])) >= alpha for t in range(T)):
            cols.append(k)
    return cols


def pin_outlier_scan(o):
    rng = np.random.default_rng(3)
    X = rng.standard_normal((9, 37)).astype(np.float16)
    X[2, 5] = 6.0          # exactly alpha: counts (>=)
    X[7, 30] = -6.0
    X[4, 11] = np.float16(5.99609375)   # largest fp16 below 6: does not count
    for alpha in (6.0, 2.5, 1.0, 0.0, float("inf")):
        mask, idx = o.outlier_columns(X, alpha)
        assert list(idx) == _brute_outliers(X, alpha), alpha
        assert list(np.nonzero(mask)[0]) == list(idx)
        hits = o.outlier_hits(X, alpha)
        ref = [sum(abs(float(X[t, k])) >= alpha for t in range(9)) for k in range(37)]
        assert list(hits) == ref
        assert o.frac_8bit(len(idx), 37) == np.float32(1.0 - len(idx) / 37.0)
    assert list(o.outlier_columns(X, 6.0)[1]) == [5, 30]
    assert len(o.outlier_columns(X, 0.0)[1]) == 37
    assert len(o.outlier_columns(X, float("inf"))[1]) == 0
    # monotone in alpha
    prev = set(range(37))
    for alpha in (0.0, 0.5, 1.0, 2.0, 3.0, 6.0):
        cur = set(o.outlier_columns(X, alpha)[1])
        assert cur <= prev
        prev = cur


# ---------------------------------------------------------------- products

def pin_int8_gemm(o):
    rng = np.random.default_rng(9)
    A = rng.integers(-127, 128, (13, 70)).astype(np.int8)
    B = rng.integers(-127, 128, (70, 29)).astype(np.int8)
    acc = o.int8_gemm(A, B)
    assert np.array_equal(acc, A.astype(np.int64) @ B.astype(np.int64))
    rows = np.array([12, 0, 5])
    assert np.array_equal(o.int8_gemm(A, B, rows), (A.astype(np.int64) @ B.astype(np.int64))[rows])
    # closed form: all-ones operands give K; extremes give K * 127^2
    K = 1000
    assert np.all(o.int8_gemm(np.ones((2, K), np.int8), np.ones((K, 3), np.int8)) == K)
    Kmax = 133144                                 # largest K with K*127^2 < 2^31
    big = o.int8_gemm(np.full((1, Kmax), 127, np.int8), np.full((Kmax, 1), -127, np.int8))
    assert big[0, 0] == -127 * 127 * Kmax
    try:
        o.int8_gemm(np.full((1, Kmax + 1), 127, np.int8), np.full((Kmax + 1, 1), 127, np.int8))
    except ArithmeticError:
        pass
    else:
        raise AssertionError("int32 overflow went unnoticed")


def pin_exact_integer_case(o):
    """alpha = +inf, inputs that quantise exactly: integer rows/columns whose
    absmax is 127, times a power of two per row of X and per column of W.
    Then the codes are the integers, and Y is the exact scaled integer
    product (representable in fp16 by construction)."""
    rng = np.random.default_rng(21)
    T, K, N = 6, 24, 10
    mx = rng.integers(-3, 4, (T, K)).astype(np.int64)
    mw = rng.integers(-3, 4, (K, N)).astype(np.int64)
    mx[np.arange(T), rng.integers(0, K // 2, T)] = 127 * rng.choice([-1, 1], T)
    mw[rng.integers(K // 2, K, N), np.arange(N)] = 127 * rng.choice([-1, 1], N)
    ex = rng.integers(-3, 3, T)
    ew = rng.integers(-3, 3, N)
    X = (mx * 2.0 ** ex[:, None]).astype(np.float16)
    W = (mw * 2.0 ** ew[None, :]).astype(np.float16)
    assert np.array_equal(X.astype(np.float64), mx * 2.0 ** ex[:, None])
    Wq, sW = o.quantize_weight_colwise(W)
    assert np.array_equal(Wq, mw.astype(np.int8))
    Y, Ypre, acc, cnt = o.mixed_linear(X, Wq, sW, W, float("inf"))
    assert cnt == 0
    exact = (mx @ mw) * 2.0 ** (ex[:, None] + ew[None, :])
    assert np.array_equal(acc, mx @ mw)
    assert np.array_equal(Ypre, exact)
    assert np.all(np.abs(exact) <= 2048 * 2.0 ** (ex[:, None] + ew[None, :]))
    assert np.array_equal(Y.astype(np.float64), exact)


def pin_outlier_part_exact(o):
    """Outlier columns go through the 16-bit product: with dyadic values the
    result is exact and every outlier term must be present, at its index."""
    T, K, N = 3, 8, 5
    X = np.zeros((T, K), np.float16)
    X[:, 0] = [127, -127, 127]                       # sX = 127 per row
    X[:, 3] = [8.0, -12.0, 0.0]                      # outlier column 3
    X[:, 6] = [0.0, 7.0, -16.0]                      # outlier column 6
    X[:, 2] = [1.0, 2.0, -5.0]
    W = np.zeros((K, N), np.float16)
    W[0] = [127, -127, 127, 127, -127]               # sW = 127 per column
    W[2] = [1, 2, 3, 4, 5]
    W[3] = [0.5, -0.25, 0.125, 1.0, -2.0]
    W[6] = [0.75, 0.0, -1.5, 0.25, 2.0]
    Wq, sW = o.quantize_weight_colwise(W)
    Y, Ypre, acc, cnt = o.mixed_linear(X, Wq, sW, W, 6.0)
    assert cnt == 3                                 # columns 0, 3, 6 (127 >= 6 too)
    # column 0 is an outlier as well, so the int8 part only sees column 2
    Xd, Wd = X.astype(np.float64), W.astype(np.float64)
    q = np.zeros((T, K)); q[:, 2] = Xd[:, 2]
    sx = np.abs(Xd[:, [1, 2, 4, 5, 7]]).max(axis=1)
    assert np.array_equal(Ypre, (Xd[:, [0, 3, 6]] @ Wd[[0, 3, 6]])
                          + np.round(Xd[:, 2:3] * 127 / sx[:, None]) * Wq[2:3].astype(np.float64)
                          * sx[:, None] * sW[None, :].astype(np.float64) / 16129.0)


def pin_alpha_zero_is_fp_matmul(o):
    """alpha = 0 sends every column to the 16-bit product: Y is the plain
    matmul (numpy float64) rounded to fp16."""
    rng = np.random.default_rng(4)
    X = rng.standard_normal((7, 40)).astype(np.float16)
    W = (rng.standard_normal((40, 12)) * 0.05).astype(np.float16)
    Wq, sW = o.quantize_weight_colwise(W)
    Y, Ypre, acc, cnt = o.mixed_linear(X, Wq, sW, W, 0.0)
    assert cnt == 40 and not acc.any()
    ref = X.astype(np.float64) @ W.astype(np.float64)
    scale = np.abs(X.astype(np.float64)) @ np.abs(W.astype(np.float64))
    assert np.all(np.abs(Ypre - ref) <= 1e-13 * scale)
    assert np.array_equal(Y, Ypre.astype(np.float16))


def error_bound(X, W, sW, is_out, sX):
    """Per-element worst case of |Y_method - X W| from |x - q s/127| <= s/254."""
    Xd = np.abs(X.astype(np.float64)) * (~is_out)[None, :]
    Wd = np.abs(W.astype(np.float64)) * (~is_out)[:, None]
    h = 0.5 + 127 * 2.0 ** -22
    K8 = float((~is_out).sum())
    return (Xd @ np.ones_like(Wd) * sW[None, :] * h / 127.0
            + np.ones_like(Xd) @ Wd * sX[:, None] * h / 127.0
            + K8 * sX[:, None] * sW[None, :] * h * h / 16129.0) * (1 + 1e-9) + 1e-12


def pin_error_bound(o):
    rng = np.random.default_rng(8)
    for (T, K, N, nout) in ((5, 64, 16, 2), (17, 200, 33, 0), (3, 96, 8, 5)):
        X = rng.standard_normal((T, K)).astype(np.float16)
        cols = rng.choice(K, nout, replace=False)
        X[:, cols] = (rng.uniform(6, 60, (T, nout)) * rng.choice([-1, 1], (T, nout))).astype(np.float16)
        W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
        Wq, sW = o.quantize_weight_colwise(W)
        Y, Ypre, acc, cnt = o.mixed_linear(X, Wq, sW, W, 6.0)
        is_out = np.zeros(K, bool); is_out[cols] = True
        assert cnt == is_out.sum()
        Xq, sX = o.quantize_rows(X, is_out)
        ref = X.astype(np.float64) @ W.astype(np.float64)
        assert np.all(np.abs(Ypre - ref) <= error_bound(X, W, sW.astype(np.float64), is_out,
                                                         sX.astype(np.float64)))


def pin_k_permutation(o):
    """Permuting K (columns of X with rows of W) permutes O and leaves Y."""
    rng = np.random.default_rng(12)
    T, K, N = 6, 48, 20
    X = rng.standard_normal((T, K)).astype(np.float16)
    X[:, 7] = 9.0
    X[2, 30] = -20.0
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    Wq, sW = o.quantize_weight_colwise(W)
    Y, Ypre, acc, cnt = o.mixed_linear(X, Wq, sW, W, 6.0)
    p = rng.permutation(K)
    Xp, Wp = np.ascontiguousarray(X[:, p]), np.ascontiguousarray(W[p])
    Wqp, sWp = o.quantize_weight_colwise(Wp)
    assert np.array_equal(Wqp, Wq[p]) and np.array_equal(sWp, sW)
    Y2, Ypre2, acc2, cnt2 = o.mixed_linear(Xp, Wqp, sWp, Wp, 6.0)
    assert cnt2 == cnt and np.array_equal(acc2, acc)
    assert np.allclose(Ypre2, Ypre, rtol=0, atol=1e-12)
    _, idx = o.outlier_columns(X, 6.0)
    _, idx2 = o.outlier_columns(Xp, 6.0)
    assert sorted(p[idx2]) == list(idx)


def pin_row_subset(o):
    """Rows of Y are independent given O: a row subset equals the full run."""
    rng = np.random.default_rng(13)
    X = rng.standard_normal((11, 64)).astype(np.float16)
    X[4, 9] = 30.0
    W = (rng.standard_normal((64, 24)) * 0.02).astype(np.float16)
    Wq, sW = o.quantize_weight_colwise(W)
    Y, Ypre, acc, _ = o.mixed_linear(X, Wq, sW, W, 6.0)
    rows = np.array([10, 0, 4])
    Ys, Ypres, accs, _ = o.mixed_linear(X, Wq, sW, W, 6.0, rows=rows)
    assert np.array_equal(accs, acc[rows]) and np.array_equal(Ys.view(np.uint16), Y[rows].view(np.uint16))


def pin_golden_worked_example(o):
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    X = np.array(g["X"], np.float16)
    W = np.array(g["W16"], np.float16)
    Wq, sW = o.quantize_weight_colwise(W)
    assert Wq.tolist() == g["Wq"] and sW.tolist() == g["sW"]
    mask, idx = o.outlier_columns(X, g["alpha"])
    assert idx.tolist() == g["outlier_idx"]
    Xq, sX = o.quantize_rows(X, mask)
    assert Xq.tolist() == g["Xq"] and sX.tolist() == g["sX"]
    Y, Ypre, acc, cnt = o.mixed_linear(X, Wq, sW, W, g["alpha"])
    assert acc.tolist() == g["acc"]
    for r in range(2):
        for n in range(2):
            expr = g["Y_exact_rational"][r][n]
            a, op, b = expr.split(" ")
            val = Fraction(a) + (Fraction(b) if op == "+" else -Fraction(b))
            assert abs(Ypre[r, n] - float(val)) <= 1e-12
    assert Y.astype(np.float64).tolist() == g["Y_fp16"]



# ------------------------------------------------- the Wq-only variant (NEXT-1)

def _grid_weights(rng, K, N):
    """fp16 weights on the quantisation grid: W[:, n] = q * 2^e[n] with
    |q| <= 127 and a +-127 in every column, so conversion gives codes q and
    scale 127 * 2^e[n] exactly (all values are exact in fp16)."""
    e = rng.integers(-8, 4, size=N)
    q = rng.integers(-127, 128, size=(K, N))
    q[rng.integers(0, K, size=N), np.arange(N)] = 127 * rng.choice([-1, 1], size=N)
    return q, e, (q * 2.0 ** e[None, :]).astype(np.float16)


def pin_dequantize_weight_grid(o):
    """On the grid, sW/127 = 2^e and q * 2^e are exact, so dequantising the
    converted weight gives it back bit for bit; a zero column stays zero."""
    rng = np.random.default_rng(11)
    q, e, W = _grid_weights(rng, 37, 24)
    W[:, 5] = 0
    Wq, sW = o.quantize_weight_colwise(W)
    q[:, 5] = 0
    assert np.array_equal(Wq.astype(np.int64), q)
    Wd = o.dequantize_weight(Wq, sW)
    assert np.array_equal(Wd.view(np.uint16), W.view(np.uint16))


def _half_ulp(v):
    """Half the binary16 spacing at the magnitude of the binary16 value v."""
    a = abs(float(v))
    if a < 2.0 ** -14:
        return 2.0 ** -25
    return 2.0 ** (math.floor(math.log2(a)) - 11)


def pin_dequantize_weight_rounding(o):
    """Against exact rationals: every dequantised value is within half an fp16
    ulp of q * sW / 127, plus the fp32 division and product (2^-23 relative
    each); odd in q and non-decreasing in q for a positive scale."""
    rng = np.random.default_rng(12)
    scales = np.concatenate([rng.uniform(1e-3, 3.0, 20), [1e-6, 2.0 ** -14, 0.5, 127.0, 3000.0]]).astype(np.float32)
    q = np.arange(-127, 128, dtype=np.int8)
    Wq = np.repeat(q[:, None], len(scales), axis=1)
    Wd = o.dequantize_weight(Wq, scales)
    for n, s in enumerate(scales):
        col = Wd[:, n]
        for i, qi in enumerate(q):
            exact = Fraction(int(qi)) * Fraction(float(s)) / 127
            err = abs(Fraction(float(col[i])) - exact)
            assert err <= Fraction(_half_ulp(col[i])) + abs(exact) * Fraction(2, 2 ** 22), (float(s), int(qi))
        assert np.array_equal(col[::-1].astype(np.float64), -col.astype(np.float64))   # q -> -q
        assert np.all(np.diff(col.astype(np.float64)) >= 0)


def pin_wq_only_variant_on_grid(o):
    """With W16 on the quantisation grid the Wq-only variant is the same
    computation as the fp16-weight one: identical Y, at every outlier index."""
    rng = np.random.default_rng(13)
    T, K, N = 9, 48, 20
    _, _, W = _grid_weights(rng, K, N)
    X = rng.standard_normal((T, K)).astype(np.float16)
    X[:, [4, 17, 40]] = rng.uniform(6.5, 30.0, size=(T, 3)).astype(np.float16)
    Wq, sW = o.quantize_weight_colwise(W)
    Y1, P1, _, c1 = o.mixed_linear(X, Wq, sW, W, 6.0)
    Y2, P2, _, c2 = o.mixed_linear(X, Wq, sW, None, 6.0)
    assert c1 == c2 >= 3
    assert np.array_equal(P1, P2) and np.array_equal(Y1.view(np.uint16), Y2.view(np.uint16))


def pin_wq_only_variant_error(o):
    """Off the grid the variants differ only through the outlier rows:
    |Ypre_wq - Ypre_w16| <= sum over outlier k of |x_k| (sW/254 + half ulp + 2^-22 sW)."""
    rng = np.random.default_rng(14)
    T, K, N = 6, 64, 16
    W = (rng.standard_normal((K, N)) * 0.05).astype(np.float16)
    X = rng.standard_normal((T, K)).astype(np.float16)
    cols = [3, 30, 63]
    X[:, cols] = rng.uniform(7.0, 40.0, size=(T, 3)).astype(np.float16)
    Wq, sW = o.quantize_weight_colwise(W)
    _, P1, _, c1 = o.mixed_linear(X, Wq, sW, W, 6.0)
    _, P2, _, c2 = o.mixed_linear(X, Wq, sW, None, 6.0)
    assert c1 == c2 == 3
    xs = np.abs(X[:, cols].astype(np.float64))
    per_w = sW.astype(np.float64) / 254.0 * (1 + 2.0 ** -20) + 2.0 ** -11 * (np.abs(W[cols].astype(np.float64)) + sW / 254.0)
    bound = xs @ per_w
    assert np.all(np.abs(P2 - P1) <= bound * (1 + 1e-9) + 1e-12)
    assert np.any(P2 != P1)                     # the variant really uses other rows

# ---------------------------------------------------------------- group-wise 4-bit codec

def _int4_grid_weights(rng, K, N, G):
    """Weights that sit exactly on a 4-bit grid: per (group, column) a power-of-two
    step s and a base lo (both exact in binary16), every level 0..15 present."""
    Q = np.empty((K, N), np.int64)
    S = np.empty((K // G, N))
    L = np.empty((K // G, N))
    W = np.empty((K, N))
    for g in range(K // G):
        for n in range(N):
            q = np.r_[0, 15, rng.integers(0, 16, G - 2)]
            rng.shuffle(q)
            s = 2.0 ** int(rng.integers(-12, -2))
            lo = float(rng.integers(-64, 64)) * s
            Q[g * G:(g + 1) * G, n] = q
            S[g, n], L[g, n] = s, lo
            W[g * G:(g + 1) * G, n] = lo + q * s
    return Q, S, L, W.astype(np.float16)


def pin_int4_grid_exact(o):
    """Weights already on a 16-level grid per (group of 64 rows, column) are coded
    exactly: codes, step and base recovered, and the decoded weight is the weight
    bit for bit.  Steps and bases differ per group and per column, so a group taken
    along the wrong axis, or a wrong step (/16 for /15), fails here."""
    rng = np.random.default_rng(41)
    K, N, G = 192, 24, 64
    Q, S, L, W = _int4_grid_weights(rng, K, N, G)
    codes, scale, lo = o.int4_quantize_groupwise(W, G)
    assert np.array_equal(codes.astype(np.int64), Q)
    assert np.array_equal(scale.astype(np.float64), S)
    assert np.array_equal(lo.astype(np.float64), L)
    Wd = o.int4_dequantize(codes, scale, lo)
    assert np.array_equal(Wd.view(np.uint16), W.view(np.uint16))


def pin_int4_nearest_level(o):
    """Brute force over the 16 levels of each group: the chosen level is the one
    nearest the weight (exact rationals), up to the fp32 rounding of the step's
    reciprocal, and the levels span the group (lo is its minimum, the top level
    within rounding of its maximum)."""
    rng = np.random.default_rng(42)
    K, N, G = 128, 16, 64
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    W[64:128, 3] = (rng.standard_normal(64) * 3.0).astype(np.float16)     # a wide group
    codes, scale, lo = o.int4_quantize_groupwise(W, G)
    assert codes.max() <= 15
    for g in range(K // G):
        for n in range(N):
            s, l = Fraction(float(scale[g, n])), Fraction(float(lo[g, n]))
            grp = W[g * G:(g + 1) * G, n]
            assert float(lo[g, n]) == float(grp.astype(np.float64).min())
            rng_ = Fraction(float(grp.astype(np.float64).max())) - l
            assert abs(15 * s - rng_) <= rng_ * Fraction(1, 1024) + Fraction(2.0 ** -24)   # binary16 step
            assert codes[g * G + int(np.argmin(grp)), n] == 0
            assert codes[g * G + int(np.argmax(grp)), n] == 15 or s == 0
            for i, w in enumerate(grp):
                wf = Fraction(float(w))
                q = int(codes[g * G + i, n])
                d = abs(wf - (l + q * s))
                best = min(abs(wf - (l + j * s)) for j in range(16))
                assert d <= best + s * Fraction(1, 2 ** 20), (g, n, i)


def pin_int4_ties_round_away_from_zero(o):
    """Exact halfway weights: a group spanning 0 .. 15 has step s = 1 (exact in
    binary16, reciprocal exact in fp32) and base 0, so w = k + 1/2 gives
    (w - lo) / s = k + 1/2 exactly, and the codec's rounding (half away from
    zero, the same rule as the int8 codes) must give k + 1.  Scaled by 2^-4
    (s = 1/16) the same holds.  Ties to even would give k for even k."""
    for scale in (1.0, 1.0 / 16.0):
        col = np.zeros(64, np.float64)
        col[0], col[1] = 0.0, 15.0                     # the group's minimum and maximum
        halves = np.arange(15) + 0.5                   # 0.5, 1.5, ..., 14.5
        col[2:17] = halves
        W = (col * scale).astype(np.float16).reshape(64, 1)
        assert np.array_equal(W.astype(np.float64).ravel(), col * scale)     # all exact in binary16
        codes, step, lo = o.int4_quantize_groupwise(np.repeat(W, 16, axis=1), 64)
        assert float(step[0, 0]) == scale and float(lo[0, 0]) == 0.0
        assert np.array_equal(codes[2:17, 0].astype(np.int64), np.arange(15) + 1), codes[2:17, 0]


def pin_int4_invariants(o):
    """A constant group has step 0 and decodes exactly; scaling a column by 2^j
    (no binary16 overflow or underflow) leaves its codes unchanged and scales step,
    base and decoded weights by exactly 2^j."""
    rng = np.random.default_rng(43)
    K, N, G = 128, 8, 64
    # magnitudes in [0.01, 0.2]: scaled by 2^-3 or 2^2 they stay normal binary16
    W = (rng.uniform(0.01, 0.2, (K, N)) * rng.choice([-1.0, 1.0], (K, N))).astype(np.float16)
    W[0:64, 0] = np.float16(0.375)
    W[64:128, 1] = np.float16(-2.0)
    codes, scale, lo = o.int4_quantize_groupwise(W, G)
    assert scale[0, 0] == 0 and scale[1, 1] == 0
    assert np.all(codes[0:64, 0] == 0) and np.all(codes[64:128, 1] == 0)
    Wd = o.int4_dequantize(codes, scale, lo)
    assert np.array_equal(Wd[:64, 0], W[:64, 0]) and np.array_equal(Wd[64:, 1], W[64:, 1])
    for j in (-3, 2):
        W2 = (W.astype(np.float64) * 2.0 ** j).astype(np.float16)
        assert np.array_equal(W2.astype(np.float64), W.astype(np.float64) * 2.0 ** j)
        c2, s2, l2 = o.int4_quantize_groupwise(W2, G)
        assert np.array_equal(c2, codes)
        assert np.array_equal(s2.astype(np.float64), scale.astype(np.float64) * 2.0 ** j)
        assert np.array_equal(l2.astype(np.float64), lo.astype(np.float64) * 2.0 ** j)
        assert np.array_equal(o.int4_dequantize(c2, s2, l2).astype(np.float64), Wd.astype(np.float64) * 2.0 ** j)


def pin_int4_error_bound(o):
    """|W~ - W| is at most half a step (plus the shortfall of 15 steps against the
    group's range when the binary16 step rounded down) plus half a binary16 ulp
    of W~, and the decoded value is binary16(q*s + lo) for the stored q, s, lo."""
    rng = np.random.default_rng(44)
    K, N, G = 256, 32, 64
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    codes, scale, lo = o.int4_quantize_groupwise(W, G)
    Wd = o.int4_dequantize(codes, scale, lo)
    s = np.repeat(scale.astype(np.float64), G, axis=0)
    l = np.repeat(lo.astype(np.float64), G, axis=0)
    exact = codes.astype(np.float64) * s + l                      # exact in double
    assert np.array_equal(Wd.view(np.uint16), exact.astype(np.float16).view(np.uint16))   # numpy's RNE
    grp = W.astype(np.float64).reshape(K // G, G, N)
    short = np.repeat(np.maximum(grp.max(1) - grp.min(1) - 15 * scale.astype(np.float64), 0), G, axis=0)
    bound = s / 2 * (1 + 2.0 ** -20) + short + np.array([_half_ulp(v) for v in Wd.ravel()]).reshape(K, N) / 2
    assert np.all(np.abs(Wd.astype(np.float64) - W.astype(np.float64)) <= bound)


def pin_int4_linear_is_the_matmul_of_the_decoded_weight(o):
    """The 4-bit product is X times the decoded weight: numpy's float64 matmul of
    the same operands, rounded by numpy to binary16 (equal except at exact
    ties of the rounding); and with small integers and exact grids it is the
    exact integer product."""
    rng = np.random.default_rng(45)
    T, K, N, G = 5, 192, 40, 64
    X = rng.standard_normal((T, K)).astype(np.float16)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    codes, scale, lo = o.int4_quantize_groupwise(W, G)
    Wd = o.int4_dequantize(codes, scale, lo)
    Y, Ypre = o.int4_linear(X, codes, scale, lo)
    ref = X.astype(np.float64) @ Wd.astype(np.float64)
    mag = np.abs(X.astype(np.float64)) @ np.abs(Wd.astype(np.float64))
    assert np.all(np.abs(Ypre - ref) <= 1e-12 * mag + 1e-300)
    assert np.array_equal(Y.view(np.uint16), Ypre.astype(np.float16).view(np.uint16))
    rows = np.array([4, 1], np.int32)
    Ys, _ = o.int4_linear(X, codes, scale, lo, rows=rows)
    assert np.array_equal(Ys.view(np.uint16), Y[rows].view(np.uint16))
    # exact integers: X in -3..3, weights on integer grids (s = 1)
    Q = rng.integers(0, 16, (K, N))
    Q[0::64] = 0
    Q[1::64] = 15
    Wi = (Q - 7).astype(np.float16)
    Xi = rng.integers(-3, 4, (T, K)).astype(np.float16)
    ci, si, li = o.int4_quantize_groupwise(Wi, G)
    assert np.array_equal(ci.astype(np.int64), Q) and np.all(si == 1) and np.all(li == -7)
    Yi, _ = o.int4_linear(Xi, ci, si, li)
    exact = Xi.astype(np.int64) @ (Q - 7)
    assert np.abs(exact).max() <= 2048
    assert np.array_equal(Yi.astype(np.int64), exact)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
