"""Pins of the oracle's FP8-GPTQ on 64 x 64 tiles ("quantization_algorithms.txt", section 1:
"For a 64x64 tile scheme": fix or search the tile scale, H = X^T X + lambda I over the tile's
64 input dimensions, quantise the columns sequentially to E4M3, propagate each residual
through H^-1 -- GPTQ's update in Cholesky form, err = (w - q) / U_ii, w_j -= err U_ij).

Checks: hand-derived worked examples, the reduction to plain projection when U is diagonal,
closed forms of the prepared factor, the output-error improvement GPTQ exists for, and the
residual relation W - Q = E U with every code nearest to its column's value at its turn.
"""
import numpy as np
import pytest

T = 64


def one_row_tile(w0, w1, u00, u01):
    W = np.zeros((T, T), np.float32)
    W[0, 0], W[0, 1] = w0, w1
    U = np.eye(T, dtype=np.float32)
    U[0, 0], U[0, 1] = u00, u01
    return W, U.reshape(1, T, T), np.ones((1, 1), np.float32)


@pytest.mark.parametrize("u00,u01", [(1.0, 0.5), (2.0, 1.0)])
def test_worked_example(orc, u00, u01):
    """w = (1.0625, 0.5) at scale 1. Column 0: 1.0625 is the midpoint of the E4M3 values 1.0
    (0x38) and 1.125 (0x39), ties to the even code: 1.0. err = 0.0625 / U_00; column 1 becomes
    0.5 - err U_01 = 0.46875 = 1.875 * 2^-2, exactly the E4M3 value 0x2F (without the
    propagation it would be 0.5 = 0x30)."""
    W, U, s = one_row_tile(1.0625, 0.5, u00, u01)
    codes, prop = orc.gptq_tiles(W, U, s, want_prop=True)
    assert codes[0, 0] == 0x38 and codes[0, 1] == 0x2F
    assert prop[0, 1] == 0.46875
    assert np.all(codes[1:] == 0) and np.all(codes[0, 2:] == 0)


def test_negative_weights_propagate_with_sign(orc):
    """The mirror image: w = (-1.0625, -0.5) gives -1.0 and -0.46875 (0xB8, 0xAF)."""
    W, U, s = one_row_tile(-1.0625, -0.5, 1.0, 0.5)
    codes = orc.gptq_tiles(W, U, s)
    assert codes[0, 0] == 0xB8 and codes[0, 1] == 0xAF


def test_diagonal_factor_is_plain_projection(orc):
    """With U diagonal nothing propagates: every code is the E4M3 projection at the tile's
    scale (as orc_project_e4m3)."""
    rng = np.random.default_rng(2)
    W = (rng.standard_t(4, (128, 128)) * 0.05).astype(np.float32)
    U = np.stack([np.diag(rng.uniform(0.5, 2.0, T)).astype(np.float32) for _ in range(2)])
    scales = np.array([[0.001, 0.0004], [0.0007, 0.002]], np.float32)
    codes = orc.gptq_tiles(W, U, scales)
    for ti in range(2):
        for tj in range(2):
            blk = W[ti * T:(ti + 1) * T, tj * T:(tj + 1) * T]
            q, _ = orc.project_e4m3_many(float(scales[ti, tj]), blk.reshape(-1))
            q = q.reshape(T, T) | (np.signbit(blk).astype(np.uint8) << 7)
            assert np.array_equal(codes[ti * T:(ti + 1) * T, tj * T:(tj + 1) * T], q)


def test_prepare_closed_form_and_factor(orc):
    rng = np.random.default_rng(3)
    g = rng.uniform(0.1, 3.0, T)
    G = np.diag(g).astype(np.float32)[None]
    U = orc.gptq_prepare(G)
    lam = 0.01 * np.mean(g.astype(np.float32).astype(np.float64))
    np.testing.assert_allclose(np.diag(U[0]), 1 / np.sqrt(g.astype(np.float32) + lam),
                               rtol=2e-7)
    assert np.all(U[0][~np.eye(T, dtype=bool)] == 0)
    X = rng.standard_normal((500, T)).astype(np.float32)
    X[:, 3] += X[:, 4]
    Gx = orc.block_gram(X, T)
    Ux = orc.gptq_prepare(Gx).astype(np.float64)[0]
    assert np.all(np.tril(Ux, -1) == 0)
    H = Gx[0].astype(np.float64) + 0.01 * np.mean(np.diag(Gx[0].astype(np.float64))) * np.eye(T)
    np.testing.assert_allclose(Ux.T @ Ux, np.linalg.inv(H), rtol=1e-5, atol=1e-6)
    Z = orc.gptq_prepare(np.zeros((1, T, T), np.float32))      # all-zero block: lambda = 1
    assert np.array_equal(Z[0], np.eye(T, dtype=np.float32))


def test_gptq_lowers_output_error(orc):
    """What the method is for: with correlated inputs, the propagated quantization has a
    smaller output error ||X (W - Q)^T||^2 than plain projection at the same tile scales."""
    rng = np.random.default_rng(4)
    R, n, k = 2000, 128, 128
    X = rng.standard_normal((R, k)).astype(np.float32)
    X[:, 1::2] += 0.8 * X[:, 0::2]
    W = (rng.standard_t(4, (n, k)) * 0.05).astype(np.float32)
    h = orc.act_sqmean(X)
    r = orc.quantize(W, "e4m3", "hopt", 64, h=h)
    U = orc.gptq_prepare(orc.block_gram(X, 64))
    codes = orc.gptq_tiles(W, U, r.scales)
    plain = orc.dequant(r.codes, r.scales, "e4m3", 64, n, k).astype(np.float64)
    gptq = orc.dequant(codes, r.scales, "e4m3", 64, n, k).astype(np.float64)
    Xd = X.astype(np.float64)
    e_plain = np.sum((Xd @ (W - plain).T) ** 2)
    e_gptq = np.sum((Xd @ (W - gptq).T) ** 2)
    assert e_gptq < 0.9 * e_plain


def e4m3_magnitudes():
    """The 127 finite E4M3 magnitudes (OCP FP8: bias 7, 3 mantissa bits, subnormals below
    2^-6, S.1111.111 the only NaN), ascending."""
    v = [m / 8 * 2.0 ** -6 for m in range(8)]
    v += [(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8) if (e, m) != (15, 7)]
    return np.array(v)


def test_residual_relation_and_nearest_codes(orc):
    """GPTQ's residual relation per tile, checked from the outside: after the sweep of a tile
    row, W - Q = E U_b with E_c the residual of column c (every update adds -err_c U_c,: to
    the tile's later columns; w_c - q_c = err_c U_cc at column c's turn). E is recovered from
    W, Q and U by a float64 triangular solve, so the value column c had at its turn is
    q_c + E_c U_cc, and its code must be the E4M3 value nearest to that value over the tile's
    scale (the top value 448 takes everything beyond the last midpoint)."""
    from scipy.linalg import solve_triangular
    rng = np.random.default_rng(17)
    n, k = 128, 192
    X = rng.standard_normal((1500, k)).astype(np.float32)
    X[:, 1::2] += 0.8 * X[:, 0::2]
    U = orc.gptq_prepare(orc.block_gram(X, T)).astype(np.float64)
    W = (rng.standard_t(4, (n, k)) * 0.05).astype(np.float32)
    scales = (np.abs(W).reshape(n // T, T, k // T, T).max(axis=(1, 3)) / 400).astype(np.float32)
    codes = orc.gptq_tiles(W, U.astype(np.float32), scales)
    g = e4m3_magnitudes()
    mag = g[codes & 0x7F]
    sign = np.where(codes & 0x80, -1.0, 1.0)
    S = np.repeat(np.repeat(scales.astype(np.float64), T, 0), T, 1)
    Q = sign * (mag * S).astype(np.float32)               # fl32(s q), as dequantized
    seen = np.empty_like(Q)
    for tj in range(k // T):
        c = slice(tj * T, (tj + 1) * T)
        E = solve_triangular(U[tj], (W[:, c].astype(np.float64) - Q[:, c]).T, trans="T",
                             lower=False).T
        seen[:, c] = Q[:, c] + E * np.diagonal(U[tj])[None, :]
    v = np.abs(seen) / S
    i = codes & 0x7F
    lo = np.where(i > 0, (g[np.maximum(i - 1, 0)] + g[i]) / 2, 0.0)
    hi = np.where(i < len(g) - 1, (g[i] + g[np.minimum(i + 1, len(g) - 1)]) / 2, np.inf)
    ok = (v >= lo * (1 - 1e-5)) & (v <= hi * (1 + 1e-5)) & ((np.sign(seen) == sign) | (mag == 0))
    assert ok.all(), (int((~ok).sum()), np.argwhere(~ok)[:3].tolist())
    plain = orc.gptq_tiles(W, np.stack([np.diag(np.diag(u)) for u in U]).astype(np.float32), scales)
    assert np.mean(codes != plain) > 0.05                 # the propagation changed many codes
