"""Pins of the oracle's GPTQ with the block quantizer as its inner step (qwantize "Results",
"GPTQ Quantization": the GPTQ block is the quantization block; sequential and ordered
variants; Frantar et al. 2022, Algorithm 1, in its Cholesky form).

Checks: a hand-derived worked example in which the propagated residual changes the next
block's scale, the reduction to the plain quantizer when nothing propagates, the ordered
variant against a physical permutation of the columns, the block losses against their
definition, and the output-error improvement GPTQ exists for.
"""
import numpy as np
import pytest


def worked(sign=1.0, u00=1.0):
    k = 32
    W = np.zeros((1, k), np.float32)
    W[0, [0, 1, 2, 16]] = np.array([1.25, 5.0625, 6.0, 5.0], np.float32) * sign
    U = np.eye(k, dtype=np.float32)
    U[0, 0], U[0, 1], U[0, 16] = u00, 0.5, 4.0
    return W, U, np.ones(k, np.float32)


@pytest.mark.parametrize("u00,scale1", [(1.0, 0x33), (2.0, 0x34)])
def test_worked_example(orc, u00, scale1):
    """NVFP4 block 16, naive scales. Block 0: amax 6 gives scale E4M3(6 / 6) = 1.0 (0x38);
    w0 = 1.25 is the midpoint of E2M1 1.0 (code 2) and 1.5 (code 3), ties to the even code
    2; err = 0.25 / U_00.
    U_00 = 1: err = 0.25 moves w1 to 5.0625 - 0.25 * 0.5 = 4.9375, below the E2M1 midpoint
    5, so code 6 (4.0) where the plain quantizer gives code 7 (6.0); w16 becomes
    5 - 0.25 * 4 = 4, and block 1 is reached with amax 4: scale E4M3(4 / 6 = 0.667) = 0.6875
    (0x33), 4 / 0.6875 = 5.82 rounds to E2M1 6 (code 7).
    U_00 = 2: err = 0.125; w1 = 5.0 exactly, the midpoint, ties to the even code 6; w16 =
    4.5, scale E4M3(0.75) = 0x34, 4.5 / 0.75 = 6 (code 7).
    Without GPTQ block 1's scale is E4M3(5 / 6 = 0.833) = 0.8125 (0x35)."""
    W, U, h = worked(u00=u00)
    r = orc.gptq_blocks(W, U, h, "nvfp4", "naive", 16)
    assert r.scales[0].tolist() == [0x38, scale1]
    assert r.codes[0, 0] == 0x62 and r.codes[0, 1] == 0x07 and r.codes[0, 8] == 0x07
    assert np.all(np.delete(r.codes[0], [0, 1, 8]) == 0)
    p = orc.quantize(W, "nvfp4", "naive", 16)
    assert p.scales[0].tolist() == [0x38, 0x35] and p.codes[0, 0] == 0x72


def test_worked_example_negative(orc):
    """The mirror image: the same scales, sign bits set (nibbles 0xA, 0xE, 0xF)."""
    W, U, h = worked(-1.0)
    r = orc.gptq_blocks(W, U, h, "nvfp4", "naive", 16)
    assert r.scales[0].tolist() == [0x38, 0x33]
    assert r.codes[0, 0] == 0xEA and r.codes[0, 1] == 0x0F and r.codes[0, 8] == 0x0F


def test_block_product_subtracted_once(orc):
    """Past its block a residual is applied as one product per block (the page's
    w_rem -= err @ h_cross), not column by column, and the two differ in rounding: block 0
    leaves residuals err_0 = err_1 = 0.25 (1.25 at scale 1 ties to E2M1 1.0), and
    U[0][16] = U[1][16] = 2^-22, so column 16 (1.75) receives 2^-24 twice. One subtraction of
    their sum gives 1.75 - 2^-23, which at block 1's scale 0.5 (amax 3) is 3.4999998: E2M1
    3.0 (code 5). Two subtractions of 2^-24 each tie back to 1.75 (the even neighbour):
    3.5, the E2M1 midpoint, ties to 4.0 (code 6). Column 17 (3.0) is E2M1 6.0 (code 7)."""
    k = 32
    W = np.zeros((1, k), np.float32)
    W[0, [0, 1, 2, 16, 17]] = [1.25, 1.25, 6.0, 1.75, 3.0]
    U = np.eye(k, dtype=np.float32)
    U[0, 16] = U[1, 16] = 2.0 ** -22
    r = orc.gptq_blocks(W, U, np.ones(k, np.float32), "nvfp4", "naive", 16)
    assert r.scales[0].tolist() == [0x38, 0x30]
    assert r.codes[0, 8] == 0x75 and r.codes[0, 0] == 0x22 and r.codes[0, 1] == 0x07
    assert orc.quantize(W, "nvfp4", "naive", 16).codes[0, 8] == 0x76


@pytest.mark.parametrize("fmt,sfmt,block", [("nvfp4", "e4m3", 16), ("nvfp4", "ue8m0", 32),
                                            ("int4", "e4m3", 16), ("int8", "e4m3", 32)])
@pytest.mark.parametrize("mode", ["naive", "sse", "hopt"])
def test_diagonal_factor_is_plain_quantization(orc, fmt, sfmt, block, mode):
    """A diagonal U propagates nothing (products with +0 leave nonzero weights alone), so
    every scale and code is the plain quantizer's (weights without exact zeros)."""
    rng = np.random.default_rng(11)
    n, k = 7, 4 * block
    W = (rng.standard_t(4, (n, k)) * 0.05).astype(np.float32)
    W[W == 0] = 1e-3
    h = np.exp(rng.normal(0, 1, k)).astype(np.float32)
    U = np.diag(rng.uniform(0.5, 2.0, k)).astype(np.float32)
    r = orc.gptq_blocks(W, U, h, fmt, mode, block, sfmt=sfmt)
    p = orc.quantize(W, fmt, mode, block, h=h if mode == "hopt" else None, sfmt=sfmt)
    assert np.array_equal(r.scales, p.scales) and np.array_equal(r.codes, p.codes)


def correlated(rng, R, k):
    X = rng.standard_normal((R, k)).astype(np.float32)
    X[:, 1::2] += 0.8 * X[:, 0::2]
    X[:, 2::3] += 0.5 * X[:, 1::3][:, :X[:, 2::3].shape[1]]
    return X


def test_ordered_equals_physical_permutation(orc):
    """The sweep in a permuted block order equals the natural-order sweep of the physically
    permuted matrix (columns, h and H permuted block-wise), mapped back."""
    rng = np.random.default_rng(12)
    n, k, B = 9, 128, 16
    X = correlated(rng, 800, k)
    W = (rng.standard_t(4, (n, k)) * 0.05).astype(np.float32)
    H = orc.gram(X)
    h = np.diagonal(H).copy()
    perm = rng.permutation(k // B).astype(np.int32)
    cols = (perm[:, None] * B + np.arange(B)[None, :]).reshape(-1)
    U = orc.gptq_prepare(H[np.ix_(cols, cols)][None])[0]
    a = orc.gptq_blocks(W, U, h, "nvfp4", "hopt", B, perm=perm)
    b = orc.gptq_blocks(np.ascontiguousarray(W[:, cols]), U, h[cols], "nvfp4", "hopt", B)
    assert np.array_equal(a.scales[:, perm], b.scales)
    qa = orc.dequant(a.codes, a.scales, "nvfp4", B, n, k)
    qb = orc.dequant(b.codes, b.scales, "nvfp4", B, n, k)
    assert np.array_equal(qa[:, cols], qb)


def test_block_losses_and_order(orc):
    rng = np.random.default_rng(13)
    n, k, B = 6, 96, 16
    W = (rng.standard_t(4, (n, k)) * 0.05).astype(np.float32)
    W[:, 32:48] *= 4.0                                   # the costliest block
    h = np.exp(rng.normal(0, 1, k)).astype(np.float32)
    L = orc.block_losses(W, h, "nvfp4", "hopt", B)
    r = orc.quantize(W, "nvfp4", "hopt", B, h=h)
    np.testing.assert_allclose(L, r.best.sum(axis=0), rtol=1e-12)  # hopt's own objective
    order = orc.block_order(L)
    assert order[0] == 2 and sorted(order.tolist()) == list(range(k // B))
    assert np.all(np.diff(L[order]) <= 0)
    assert orc.block_order([1.0, 3.0, 3.0, 2.0]).tolist() == [1, 2, 3, 0]


@pytest.mark.parametrize("ordered", [False, True])
def test_gptq_lowers_output_error(orc, ordered):
    """What GPTQ is for: a smaller output error ||X (W - Q)^T|| than the plain quantizer,
    with correlated inputs (the weight error itself grows, as on the page's tables)."""
    rng = np.random.default_rng(14)
    R, n, k, B = 3000, 48, 256, 16
    X = correlated(rng, R, k)
    W = (rng.standard_t(4, (n, k)) * 0.05).astype(np.float32)
    H = orc.gram(X)
    h = np.diagonal(H).copy()
    g = orc.gptq(W, H, h, "nvfp4", "hopt", B, ordered=ordered)
    p = orc.quantize(W, "nvfp4", "hopt", B, h=h)
    Xd, Wd = X.astype(np.float64), W.astype(np.float64)
    out = {}
    for nm, r in (("gptq", g), ("plain", p)):
        Q = orc.dequant(r.codes, r.scales, "nvfp4", B, n, k).astype(np.float64)
        out[nm] = (np.linalg.norm(Xd @ (Wd - Q).T), np.linalg.norm(Wd - Q))
    assert out["gptq"][0] < 0.92 * out["plain"][0]
    assert out["gptq"][1] > out["plain"][1]


def test_gram_is_the_mean_outer_product(orc):
    rng = np.random.default_rng(15)
    X = rng.standard_normal((5, 4)).astype(np.float32)
    H = orc.gram(X)
    ref = sum(np.outer(x.astype(np.float64), x.astype(np.float64)) for x in X) / 5
    np.testing.assert_allclose(H, ref.astype(np.float32), rtol=1e-7)
    assert np.array_equal(np.diagonal(H), orc.act_sqmean(X))


def test_gram_entries_exact_sums(orc):
    """Sampled Gram entries on small-integer bf16 inputs: every product and every partial sum
    is an integer below 2^53, so the float64 sums are exact and must equal Python's integer
    sums over the rows, divided by R once; chunking the rows (3 rows a chunk here) must not
    change the result. The diagonal equals the h pass."""
    rng = np.random.default_rng(16)
    R, K = 11, 9
    Xi = rng.integers(-40, 41, (R, K))
    X = (np.asarray(Xi, np.float32).view(np.uint32) >> 16).astype(np.uint16)   # exact bf16
    pairs = np.array([(0, 0), (0, 8), (8, 0), (3, 5), (5, 3), (7, 7), (2, 6)])
    got = orc.gram_entries(X, pairs, chunk_rows=3)
    ref = [sum(int(Xi[r, i]) * int(Xi[r, j]) for r in range(R)) / R for i, j in pairs]
    assert got.tolist() == ref
    d = np.arange(K)
    diag = orc.gram_entries(X, np.stack([d, d], axis=1))
    assert np.array_equal(diag.astype(np.float32), orc.act_sqmean(X))


GRIDS = {"nvfp4": [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0],
         "int4": [0.0, 1.0, 2.0, 3.0, 4.0, 5.0, 6.0, 7.0]}


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
@pytest.mark.parametrize("mode", ["naive", "hopt"])
@pytest.mark.parametrize("ordered", [False, True])
def test_residual_relation_and_nearest_codes(orc, fmt, mode, ordered):
    """GPTQ's residual relation, checked from the outside: after the sweep W - Q = E U in
    sweep order, with E_c the residual err_c of column c (Frantar et al. 2022, Algorithm 1:
    every update adds -err_c U_c,: to the later columns, and w_c - q_c = err_c U_cc at column
    c's turn). So E is recovered from W, Q and U alone by a float64 triangular solve; the value
    column c had when the sweep reached it is q_c + E_c U_cc, and q_c must be the grid point
    nearest to it at its block's scale (a saturated top code: anything beyond the last
    midpoint); and each block's scale must be the plain quantizer's pick on the block's
    weights as they stood when the sweep reached the block. A dropped or misplaced update, a
    wrong sign, a transposed U, a missing division by U_cc, a scale searched on the original
    weights or a block order ignored breaks this for many elements."""
    from scipy.linalg import solve_triangular
    rng = np.random.default_rng(16)
    R, n, k, B = 2000, 48, 256, 16
    X = correlated(rng, R, k)
    W = (rng.standard_t(4, (n, k)) * 0.05).astype(np.float32)
    H = orc.gram(X)
    h = np.diagonal(H).copy()
    perm = rng.permutation(k // B).astype(np.int32) if ordered else np.arange(k // B, dtype=np.int32)
    cols = (perm[:, None] * B + np.arange(B)[None, :]).reshape(-1)   # sweep position -> column
    U = orc.gptq_prepare(H[np.ix_(cols, cols)][None])[0].astype(np.float64)
    r = orc.gptq_blocks(W, U.astype(np.float32), h, fmt, mode, B, perm=perm if ordered else None)
    # everything below in sweep order
    Q = orc.dequant(r.codes, r.scales, fmt, B, n, k).astype(np.float64)[:, cols]
    # every nibble the value 1 (E2M1 code 2, INT4 code 1): dequantizes to the block scale
    ones = np.full_like(r.codes, 0x22 if fmt == "nvfp4" else 0x11)
    S = orc.dequant(ones, r.scales, fmt, B, n, k).astype(np.float64)[:, cols]
    Wp, hp, scales = W[:, cols].astype(np.float64), h[cols], r.scales[:, perm]
    E = solve_triangular(U, (Wp - Q).T, trans="T", lower=False).T
    seen = Q + E * np.diagonal(U)[None, :]              # column c's value at its turn
    v, q = np.abs(seen / S), np.abs(Q / S)
    g = np.asarray(GRIDS[fmt])
    i = np.searchsorted(g, q)
    assert np.array_equal(g[i], q)                      # Q is on the grid
    lo = np.where(i > 0, (g[np.maximum(i - 1, 0)] + g[i]) / 2, 0.0)
    hi = np.where(i < len(g) - 1, (g[i] + g[np.minimum(i + 1, len(g) - 1)]) / 2, np.inf)
    same_sign = (np.sign(seen) == np.sign(Q)) | (Q == 0)
    ok = (v >= lo - 1e-4) & (v <= hi + 1e-4) & same_sign
    assert ok.all(), (int((~ok).sum()), np.argwhere(~ok)[:3].tolist())
    start = np.empty_like(seen)
    for b in range(k // B):
        c0 = b * B
        start[:, c0:c0 + B] = Wp[:, c0:c0 + B] - E[:, :c0] @ U[:c0, c0:c0 + B]
    hq = hp if mode == "hopt" else None
    plain_start = orc.quantize(start.astype(np.float32), fmt, mode, B, h=hq)
    assert np.sum(plain_start.scales != scales) <= 2         # float32 vs float64 near-ties
    plain = orc.quantize(Wp.astype(np.float32), fmt, mode, B, h=hq)   # before the sweep:
    assert np.sum(plain.scales != scales) >= 20              # the propagation moves many scales
