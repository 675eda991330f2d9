"""GPU Gram blocks (tensor cores) against the oracle's G = fl32(X_b^T X_b / R).

Bar: the GPU sums bf16 products exactly in float32 inside the tensor cores over at most 512
rows, then in double; each entry is within (512 + 2) 2^-23 (|X|^T |X|)_ij / R of the
oracle's (a per-addition error of at most one float32 ulp of the running partial), and h is
diag(G) bit for bit and within 1e-5 of the h pass.
"""
import numpy as np
import pytest
import torch

from gpu_util import oracle_view

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def mxq():
    from block_scaled_weight_b200.build import build
    build()
    from block_scaled_weight_b200 import mxq as m
    return m


@pytest.fixture(scope="module")
def synth():
    from block_scaled_weight_b200 import synth as s
    return s


def check_gram(orc, X, G, B):
    Xo = oracle_view(X)
    ref = orc.block_gram(Xo, B)
    Xf = np.abs(orc.to_float(Xo).astype(np.float64))
    R, K = Xf.shape
    for b in range(K // B):
        A = Xf[:, b * B:(b + 1) * B]
        tol = (A.T @ A) / R * (514 * 2.0 ** -23) + 1e-38
        err = np.abs(G[b].astype(np.float64) - ref[b].astype(np.float64))
        assert np.all(err <= tol), (b, float((err / tol).max()))


@pytest.mark.parametrize("rows,cols,B", [(64, 128, 16), (1000, 384, 16), (1000, 384, 32),
                                         (777, 336, 16), (20000, 1024, 16), (5, 256, 32),
                                         (1000, 384, 64), (777, 320, 64), (20000, 1024, 64),
                                         (5, 192, 64)])
def test_gram_matches_oracle(mxq, orc, synth, rows, cols, B):
    X = synth.activations(rows, cols, 81, dtype=torch.bfloat16, device=DEV)
    G, h = mxq.mxq_act_block_gram(X, B, with_h=True)
    torch.cuda.synchronize()
    Gn = G.cpu().numpy()
    assert np.isfinite(Gn).all()
    check_gram(orc, X, Gn, B)
    assert np.array_equal(np.diagonal(Gn, axis1=1, axis2=2).reshape(-1), h.cpu().numpy())
    hp = mxq.mxq_act_sqmean(X).cpu().numpy()
    np.testing.assert_allclose(h.cpu().numpy(), hp, rtol=1e-5, atol=0)


def test_gram_strided_and_deterministic(mxq, synth):
    big = synth.activations(3000, 768, 82, dtype=torch.bfloat16, device=DEV)
    X = big[:, 128:640]
    a = mxq.mxq_act_block_gram(X, 16)
    b = mxq.mxq_act_block_gram(X.contiguous(), 16)
    c = mxq.mxq_act_block_gram(X, 16)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(a, c)


def test_gram_rejects_float32_and_bad_blocks(mxq):
    X = torch.zeros(64, 128, dtype=torch.float32, device=DEV)
    with pytest.raises(mxq.MxqError):
        mxq.mxq_act_block_gram(X, 16)
    Xb = torch.zeros(64, 120, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(mxq.MxqError):
        mxq.mxq_act_block_gram(Xb, 16)
    with pytest.raises(mxq.MxqError):
        mxq.mxq_act_block_gram(torch.zeros(64, 128, dtype=torch.bfloat16, device=DEV), 48)
    with pytest.raises(mxq.MxqError):
        mxq.mxq_act_block_gram(torch.zeros(64, 96, dtype=torch.bfloat16, device=DEV), 64)


# ---------------------------------------------------------------------------------------
# block-Hessian search: GPU against the oracle with the same (oracle-computed) G
# ---------------------------------------------------------------------------------------

def correlated_x(synth, rows, cols, seed):
    X = synth.activations(rows, cols, seed, dtype=torch.float32, device="cpu")
    X[:, 1::4] += 0.7 * X[:, 0::4]                   # neighbouring columns correlated
    X[:, 5::16] -= 0.5 * X[:, 3::16]
    return X.to(torch.bfloat16)


def gram_pair(mxq, orc, W, G, fmt, sfmt, B, window=-1):
    p = mxq.params(fmt, "hopt", B, window=window, scale_fmt=sfmt)
    codes, scales = mxq.mxq_quantize_gram(W, p, torch.from_numpy(G).to(DEV))
    torch.cuda.synchronize()
    r = orc.quantize_gram(oracle_view(W), fmt, B, G, window=window, sfmt=sfmt)
    return codes.cpu().numpy(), scales.cpu().numpy(), r


@pytest.mark.parametrize("fmt,sfmt", [("nvfp4", "e4m3"), ("nvfp4", "ue8m0"), ("nvfp4", "ue4m4"),
                                      ("int4", "e4m3"), ("int4", "ue5m3")])
@pytest.mark.parametrize("B,window", [(16, -1), (32, -1), (16, 4)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gram_search_parity(mxq, orc, synth, fmt, sfmt, B, window, dtype):
    n, k = 101, 512
    W = synth.gaussian_weight(n, k, 91, dtype=dtype, device=DEV)
    # Gram blocks of correlated inputs for the first half of the columns (not diagonally
    # dominant: every candidate evaluated) and of 20000 rows of independent unit-variance
    # inputs for the second half (diagonally dominant: the pruned search)
    G1 = orc.block_gram(oracle_view(correlated_x(synth, 400, k, 92)), B)
    X2 = torch.randn(20000, k, generator=torch.Generator().manual_seed(97)).to(torch.bfloat16)
    G2 = orc.block_gram(oracle_view(X2), B)
    G = np.concatenate([G1[:k // B // 2], G2[k // B // 2:]])
    codes, scales, r = gram_pair(mxq, orc, W, G, fmt, sfmt, B, window)
    mism = scales != r.scales
    assert not mism.any(), f"{mism.sum()} scales differ, first {np.argwhere(mism)[:3].tolist()}"
    assert np.array_equal(codes, r.codes)


@pytest.mark.parametrize("B", [16, 32])
def test_gram_search_special_matrices(mxq, orc, synth, B):
    """Zero blocks (every candidate ties), a dead input channel (G_ii = 0: every block goes
    to the exact pass), an indefinite symmetric matrix, and G = diag(h) (= H-optimal)."""
    k = 4 * B
    rng = np.random.default_rng(7)
    W = synth.gaussian_weight(20, k, 93, dtype=torch.bfloat16, device=DEV)
    W[3] = 0
    W[4, :B] = 0
    base = orc.block_gram(oracle_view(correlated_x(synth, 300, k, 94)), B)
    dead = base.copy()
    dead[1, 2, :] = 0
    dead[1, :, 2] = 0
    S = rng.standard_normal((k // B, B, B)).astype(np.float32)
    indef = ((S + np.transpose(S, (0, 2, 1))) / 2).astype(np.float32)
    h = np.exp(rng.normal(0, 1, k)).astype(np.float32)
    diag = np.zeros((k // B, B, B), np.float32)
    for b in range(k // B):
        diag[b] = np.diag(h[b * B:(b + 1) * B])
    for G in (base, dead, indef, diag):
        codes, scales, r = gram_pair(mxq, orc, W, G, "nvfp4", "e4m3", B)
        assert np.array_equal(scales, r.scales) and np.array_equal(codes, r.codes)
    p = mxq.params("nvfp4", "hopt", B)
    c2, s2 = mxq.mxq_quantize(W, p, torch.from_numpy(h).to(DEV))
    c1, s1 = mxq.mxq_quantize_gram(W, p, torch.from_numpy(diag).to(DEV))
    assert torch.equal(s1, s2) and torch.equal(c1, c2)


def test_gpu_gram_feeds_search(mxq, orc, synth):
    """End to end on the GPU (Gram pass, then search with the GPU's G). The GPU pick c_g is
    optimal under the GPU's G_g, so under the oracle's G_o its error is at most the oracle's
    best plus the two picks' sensitivity to the difference of the two matrices:
    e_o(c_g) <= e_o(c_o) + D(c_g) + D(c_o), D(c) = sum_ij |G_g - G_o|_ij |d_i(c)| |d_j(c)|."""
    k, B, n = 512, 16, 40
    Xb = correlated_x(synth, 2000, k, 95)
    W = synth.gaussian_weight(n, k, 96, dtype=torch.bfloat16, device=DEV)
    G = mxq.mxq_act_block_gram(Xb.to(DEV), B)
    p = mxq.params("nvfp4", "hopt", B)
    codes, scales = mxq.mxq_quantize_gram(W, p, G)
    torch.cuda.synchronize()
    Gg = G.cpu().numpy().astype(np.float64)
    Go = orc.block_gram(oracle_view(Xb), B)
    r = orc.quantize_gram(oracle_view(W), "nvfp4", B, Go)
    Wf = orc.to_float(oracle_view(W)).astype(np.float64)

    # the GPU picks decoded by the GPU's own dequant (no GPU output enters the oracle)
    dg = (Wf - mxq.mxq_dequant(codes, scales, p, n, k).cpu().numpy()).reshape(n, k // B, B)
    do = (Wf - orc.dequant(r.codes, r.scales, "nvfp4", B, n, k)).reshape(n, k // B, B)
    A = np.abs(Gg - Go.astype(np.float64))
    e_g = np.einsum("nbi,bij,nbj->nb", dg, Go.astype(np.float64), dg)
    slack = (np.einsum("nbi,bij,nbj->nb", np.abs(dg), A, np.abs(dg)) +
             np.einsum("nbi,bij,nbj->nb", np.abs(do), A, np.abs(do)))
    assert np.all(e_g <= r.best + slack + 1e-12 * np.abs(r.best) + 1e-300)
    assert np.mean(scales.cpu().numpy() == r.scales) > 0.9
