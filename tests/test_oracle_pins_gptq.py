"""Pins of the oracle's FP8-GPTQ on 64 x 64 tiles ("quantization_algorithms.txt", section 1:
"For a 64x64 tile scheme": fix or search the tile scale, H = X^T X + lambda I over the tile's
64 input dimensions, quantise the columns sequentially to E4M3, propagate each residual
through H^-1 -- GPTQ's update in Cholesky form, err = (w - q) / U_ii, w_j -= err U_ij).

Checks: hand-derived worked examples, the reduction to plain projection when U is diagonal,
closed forms of the prepared factor, and the output-error improvement GPTQ exists for.
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
