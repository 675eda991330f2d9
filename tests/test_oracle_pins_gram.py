"""Pins of the oracle's block-Hessian objective ("quantization_algorithms.txt", section 1:
choose s minimising || X_b (W_b - s Q(W_b / s))^T ||_F^2; the diagonal h_j = E[x_j^2] is its
cheap approximation). For one row's block the objective is R d^T G d with the Gram block
G = X_b^T X_b / R, stored as float32.

Checks against closed forms (exact integer Gram sums, the identity with ||X_b d||^2),
exact rational brute force, and reductions to the diagonal and plain searches.
"""
from fractions import Fraction as Fr

import numpy as np
import pytest

from tests.test_oracle_pins import E2M1_POS, E4M3_POS, nearest_even_argmin, synthetic


def test_gram_exact_on_dyadic_inputs(orc):
    """Entries k/8 with |k| <= 64: every partial sum is exact in double, so G is the
    correctly rounded X_b^T X_b / R in any order -- numpy's product must agree bit for bit."""
    rng = np.random.default_rng(1)
    X = (rng.integers(-64, 65, (300, 64)) / 8).astype(np.float32)
    for B in (16, 32):
        G = orc.block_gram(X, B)
        ref = (X.astype(np.float64).T @ X.astype(np.float64)) / 300
        for b in range(64 // B):
            blk = ref[b * B:(b + 1) * B, b * B:(b + 1) * B].astype(np.float32)
            assert np.array_equal(G[b], blk), (B, b)


def test_gram_symmetric_diagonal_is_h(orc):
    X = synthetic(400, 128, 3)                     # bf16 bits, heavy columns included
    h = orc.act_sqmean(X)
    for B in (16, 32):
        G = orc.block_gram(X, B)
        assert np.array_equal(G, np.transpose(G, (0, 2, 1)))
        assert np.array_equal(np.diagonal(G, axis1=1, axis2=2).reshape(-1), h)
        ev = np.linalg.eigvalsh(G.astype(np.float64))
        assert ev.min() > -1e-6 * ev.max()                 # positive semi-definite


def test_diagonal_gram_is_hopt_and_identity_is_sse(orc):
    """With G = diag(h) the block-Hessian search is the H-optimal search, bit for bit
    (off-diagonal terms add exact zeros); with G = I it is the SSE search."""
    W = synthetic(12, 256, 5)
    h = np.exp(np.random.default_rng(6).normal(0, 1, 256)).astype(np.float32)
    for fmt, sfmt, B in (("nvfp4", "e4m3", 16), ("nvfp4", "ue8m0", 32), ("int4", "e4m3", 16),
                         ("int8", "e4m3", 32)):
        Gd = np.zeros((256 // B, B, B), np.float32)
        Gi = np.zeros((256 // B, B, B), np.float32)
        for b in range(256 // B):
            Gd[b] = np.diag(h[b * B:(b + 1) * B])
            Gi[b] = np.eye(B, dtype=np.float32)
        for window in (-1, 3):
            a = orc.quantize_gram(W, fmt, B, Gd, window=window, sfmt=sfmt)
            r = orc.quantize(W, fmt, "hopt", B, h=h, window=window, sfmt=sfmt)
            for key in ("codes", "scales", "best", "second", "naive"):
                np.testing.assert_array_equal(a[key], r[key], err_msg=f"{fmt} {sfmt} {key}")
            a = orc.quantize_gram(W, fmt, B, Gi, window=window, sfmt=sfmt)
            r = orc.quantize(W, fmt, "sse", B, window=window, sfmt=sfmt)
            for key in ("codes", "scales", "best", "second"):
                np.testing.assert_array_equal(a[key], r[key], err_msg=f"{fmt} {sfmt} {key}")


def exact_gram_errors(w, G, fmt="nvfp4"):
    """Every E4M3 candidate's exact d^T G d (Fractions; G's float values; d signed)."""
    grid = E2M1_POS if fmt == "nvfp4" else np.arange(8, dtype=np.float32)
    a = np.abs(w).astype(np.float32)
    errs = []
    for code in range(1, 127):
        s = np.float32(E4M3_POS[code])
        q = nearest_even_argmin(a / s, grid)
        d = [Fr(float(wj)) - (1 if wj >= 0 and not (wj == 0 and np.signbit(wj)) else -1)
             * Fr(float(s)) * Fr(float(grid[qi])) for wj, qi in zip(w, q)]
        errs.append(sum(Fr(float(G[i, j])) * d[i] * d[j]
                        for i in range(len(w)) for j in range(len(w))))
    return errs


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_gram_search_equals_exact_bruteforce(orc, fmt):
    rng = np.random.default_rng(9)
    B = 16
    X = (rng.standard_normal((64, B)) * np.exp(rng.normal(0, 1, B))).astype(np.float32)
    X[:, 3] += 0.8 * X[:, 7]                         # correlated inputs
    G = orc.block_gram(X, B)
    for _ in range(6):
        w = (rng.standard_normal(B) * np.exp(rng.normal(-3, 0.5))).astype(np.float32)
        r = orc.quantize_gram(w.reshape(1, -1), fmt, B, G)
        errs = exact_gram_errors(w, G[0], fmt)
        e1 = min(errs)
        assert int(r.scales[0, 0]) == 1 + errs.index(e1)
        assert r.best[0, 0] == pytest.approx(float(e1), rel=1e-12, abs=1e-300)


def test_objective_is_output_error(orc):
    """R d^T G d equals ||X_b d||^2 (the page's output-error objective) up to the float32
    rounding of G: |difference| <= 2^-24 sum_ij |(X^T X)_ij| |d_i d_j|."""
    rng = np.random.default_rng(12)
    R, B = 50, 16
    X = (rng.standard_normal((R, B)) * 0.5).astype(np.float32)
    X[:, 0] += X[:, 1]
    G = orc.block_gram(X, B)[0]
    w = (rng.standard_normal(B) * 0.05).astype(np.float32)
    r = orc.quantize_gram(w.reshape(1, -1), "nvfp4", B, G.reshape(1, B, B))
    What = orc.dequant(r.codes, r.scales, "nvfp4", B, 1, B)[0]
    d = [Fr(float(a)) - Fr(float(b)) for a, b in zip(w, What)]
    xd = [sum(Fr(float(X[t, j])) * d[j] for j in range(B)) for t in range(R)]
    out = sum(v * v for v in xd)
    XtX = [[sum(Fr(float(X[t, i])) * Fr(float(X[t, j])) for t in range(R)) for j in range(B)]
           for i in range(B)]
    bound = Fr(1, 2 ** 24) * sum(abs(XtX[i][j]) * abs(d[i] * d[j])
                                  for i in range(B) for j in range(B))
    assert abs(Fr(r.best[0, 0]) * R - out) <= bound * 1.001 + Fr(1, 10 ** 30)
