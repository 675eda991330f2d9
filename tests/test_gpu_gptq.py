"""GPU FP8-GPTQ on 64 x 64 tiles ("quantization_algorithms.txt", section 1, the 64x64 tile
scheme) against the oracle.

Bars:
- the sweep (mxq_gptq_tiles) is bit-exact: given the same U and tile scales, every code
  equals the oracle's (both evaluate the definition's float32 steps in its order);
- the factor (mxq_gptq_prepare): both sides compute U in float64 and round it to float32
  once, by different but backward-stable routes (oracle: inverse, then Cholesky; GPU:
  Cholesky of the reversed H, then a triangular inverse). Their float64 values differ by
  a small multiple of cond(H) 2^-53 relative to the block's largest entry -- with the 1%
  damping cond(H) <= 1 + 100 x 64 -- far below a float32 ulp, so an entry differs by one
  float32 rounding step at most, or, near zero, by that float64 error:
  |dU| <= 2^-23 |U| + 2^-30 max|U_b|;
- end to end (Gram, factor, search, sweep, all on the GPU, against the oracle's pipeline
  from the same X and W): codes may differ only where a one-ulp change of U moves a
  propagated weight across an E4M3 rounding boundary -- at most 1e-4 of them -- and the
  output error agrees within 1e-3 relative.
"""
import numpy as np
import pytest
import torch

from gpu_util import output_error_np, oracle_view

pytestmark = pytest.mark.gpu
DEV = "cuda"
T = 64


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


def correlated_x(synth, rows, k, seed, device):
    """Activations with pairwise-correlated channels, so that the propagation matters."""
    X = synth.activations(rows, k, seed, dtype=torch.float32, device=device)
    X[:, 1::2] += 0.8 * X[:, 0::2]
    return X.to(torch.bfloat16)


def oracle_inputs(orc, synth, n, k, seed, dtype):
    W = synth.student_t_weight(n, k, seed, dtype=dtype, device=DEV)
    X = correlated_x(synth, 600, k, seed + 1, DEV)
    Xo = oracle_view(X)
    h = orc.act_sqmean(Xo)
    r = orc.quantize(oracle_view(W), "e4m3", "hopt", T, h=h)
    U = orc.gptq_prepare(orc.block_gram(Xo, T))
    return W, X, r, U


def sweep(mxq, W, U, scales):
    codes = mxq.mxq_gptq_tiles(W, torch.from_numpy(U).to(DEV),
                               torch.from_numpy(np.ascontiguousarray(scales)).to(DEV))
    torch.cuda.synchronize()
    return codes.cpu().numpy()


@pytest.mark.parametrize("n,k", [(64, 64), (128, 192), (320, 256), (64, 1024)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_sweep_bit_exact(mxq, orc, synth, n, k, dtype):
    W, _, r, U = oracle_inputs(orc, synth, n, k, 91, dtype)
    got = sweep(mxq, W, U, r.scales)
    ref = orc.gptq_tiles(oracle_view(W), U, r.scales)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:4].tolist()}"
    assert not np.array_equal(ref, r.codes)        # the propagation changed something


def test_sweep_strided_rows(mxq, orc, synth):
    big = synth.student_t_weight(128, 448, 92, dtype=torch.bfloat16, device=DEV)
    W = big[:, 64:320]                             # ld 448, 128-byte row offset
    X = correlated_x(synth, 400, 256, 93, DEV)
    Xo = oracle_view(X)
    r = orc.quantize(oracle_view(W), "e4m3", "hopt", T, h=orc.act_sqmean(Xo))
    U = orc.gptq_prepare(orc.block_gram(Xo, T))
    got = sweep(mxq, W, U, r.scales)
    assert np.array_equal(got, orc.gptq_tiles(oracle_view(W), U, r.scales))


def test_sweep_special_cases(mxq, orc):
    """Zero tiles (scale 0), signed zeros under propagation, saturation at 448 s, subnormal
    E4M3 codes, a diagonal factor (plain projection) and a strongly coupled one."""
    rng = np.random.default_rng(7)
    n, k = 128, 192
    W = (rng.standard_t(4, (n, k)) * 0.05).astype(np.float32)
    W[:64, :64] = 0.0                               # an all-zero tile
    W[:64, 64:128] = -0.0                           # all negative zeros
    W[5, 64:70] = [-0.0, 0.0, -0.0, 0.0, -0.0, 1e-30]
    W[64:, 128:] *= 1000.0                          # far above 448 s: saturating codes
    W[64:80, :64] = 1e-8                            # 0.01 x the scale: subnormal E4M3 codes
    scales = np.array([[0.0, 1e-3, 2e-4], [1e-6, 3e-4, 5e-5]], np.float32)
    U = np.zeros((k // T, T, T), np.float32)
    U[0] = np.eye(T, dtype=np.float32) * 1.5
    for b in (1, 2):
        A = np.triu(rng.normal(0, 0.6, (T, T))).astype(np.float32)
        A[np.diag_indices(T)] = rng.uniform(0.3, 2.0, T).astype(np.float32)
        U[b] = A
    Wt = torch.from_numpy(W).to(DEV)
    got = sweep(mxq, Wt, U, scales)
    ref = orc.gptq_tiles(W, U, scales)
    assert np.array_equal(got, ref)
    assert np.all(ref[:64, :64] & 0x7F == 0)
    assert np.any(ref[64:, 128:] & 0x7F == 0x7E)
    blk = W[64:, :64]                               # diagonal U: plain projection
    q, _ = orc.project_e4m3_many(float(scales[1, 0]), blk.reshape(-1))
    q = q.reshape(blk.shape) | (np.signbit(blk).astype(np.uint8) << 7)
    assert np.array_equal(got[64:, :64], q)
    assert np.any((q[:16] & 0x7F) > 0) and np.all((q[:16] & 0x7F) < 8)


@pytest.mark.parametrize("u00,u01", [(1.0, 0.5), (2.0, 1.0)])
def test_sweep_worked_example(mxq, u00, u01):
    """w = (1.0625, 0.5), scale 1: column 0 ties to the even code 0x38 (1.0); the residual
    0.0625 / U_00 times U_01 leaves 0.46875, exactly E4M3 0x2F."""
    W = np.zeros((T, T), np.float32)
    W[0, 0], W[0, 1] = 1.0625, 0.5
    U = np.eye(T, dtype=np.float32)[None].copy()
    U[0, 0, 0], U[0, 0, 1] = u00, u01
    got = sweep(mxq, torch.from_numpy(W).to(DEV), U, np.ones((1, 1), np.float32))
    assert got[0, 0] == 0x38 and got[0, 1] == 0x2F
    assert np.all(got[1:] == 0) and np.all(got[0, 2:] == 0)


def check_factor(U_gpu, U_ref):
    assert np.all(np.isfinite(U_gpu))
    assert np.all(np.tril(U_gpu, -1) == 0)
    for b in range(U_ref.shape[0]):
        ref = U_ref[b].astype(np.float64)
        tol = 2.0 ** -23 * np.abs(ref) + 2.0 ** -30 * np.abs(ref).max()
        err = np.abs(U_gpu[b].astype(np.float64) - ref)
        assert np.all(err <= tol), (b, float((err / tol).max()))


@pytest.mark.parametrize("k,rows", [(64, 300), (256, 1000), (1024, 5000)])
def test_prepare_matches_oracle(mxq, orc, synth, k, rows):
    X = correlated_x(synth, rows, k, 95, "cpu")
    G = orc.block_gram(oracle_view(X), T)
    U = mxq.mxq_gptq_prepare(torch.from_numpy(G).to(DEV)).cpu().numpy()
    check_factor(U, orc.gptq_prepare(G))


def test_prepare_degenerate_blocks(mxq, orc):
    """An all-zero block (lambda = 1: U = I), a dead channel, a rank-one block, a diagonal
    block (closed form 1 / sqrt(g + lambda)) and another damping."""
    rng = np.random.default_rng(8)
    G = np.zeros((5, T, T), np.float32)
    A = rng.standard_normal((200, T)).astype(np.float32)
    G[1] = (A.T @ A / 200).astype(np.float32)
    G[1][7, :] = 0.0
    G[1][:, 7] = 0.0
    v = rng.standard_normal(T).astype(np.float32)
    G[2] = np.outer(v, v).astype(np.float32)
    G[3] = np.diag(rng.uniform(0.1, 3.0, T)).astype(np.float32)
    B = rng.standard_normal((100, T)).astype(np.float32)
    G[4] = (B.T @ B / 100).astype(np.float32)
    Gd = torch.from_numpy(G).to(DEV)
    for damp in (0.01, 0.1):
        U = mxq.mxq_gptq_prepare(Gd, damp).cpu().numpy()
        check_factor(U, orc.gptq_prepare(G, damp))
    U = mxq.mxq_gptq_prepare(Gd).cpu().numpy()
    assert np.array_equal(U[0], np.eye(T, dtype=np.float32))


def test_end_to_end_against_oracle_pipeline(mxq, orc, synth):
    n, k, rows = 256, 512, 4096
    W = synth.student_t_weight(n, k, 97, dtype=torch.bfloat16, device=DEV)
    X = correlated_x(synth, rows, k, 98, DEV)
    # GPU: Gram (h = its diagonal), factor, tile-scale search, sweep
    G, h = mxq.mxq_act_block_gram(X, T, with_h=True)
    U = mxq.mxq_gptq_prepare(G)
    p = mxq.params("e4m3", "hopt", T)
    _, scales = mxq.mxq_quantize(W, p, h)
    codes = mxq.mxq_gptq_tiles(W, U, scales)
    torch.cuda.synchronize()
    # oracle from the same inputs
    Xo, Wo = oracle_view(X), oracle_view(W)
    Go = orc.block_gram(Xo, T)
    ho = np.diagonal(Go, axis1=1, axis2=2).reshape(-1).copy()
    r = orc.quantize(Wo, "e4m3", "hopt", T, h=ho)
    ref = orc.gptq_tiles(Wo, orc.gptq_prepare(Go), r.scales)
    cg = codes.cpu().numpy()
    sg = scales.cpu().numpy()
    same = sg == r.scales                          # h from the two Grams: near-ties may differ
    assert np.mean(same) >= 0.9
    mask = np.repeat(np.repeat(same, T, 0), T, 1)
    assert np.mean(cg[mask] != ref[mask]) <= 1e-4
    idx = synth.sample_rows(rows, 512, 99).to(DEV)
    Xs = oracle_view(X[idx])
    # the GPU result measured with its own dequant and plain numpy (no GPU output enters the
    # oracle); the oracle's pipeline and the plain tile search measured by the oracle
    pg = mxq.params("e4m3", "hopt", T)
    What_gpu = mxq.mxq_dequant(codes, scales, pg, n, k).cpu().numpy()
    e_gpu = output_error_np(orc.to_float(Xs), orc.to_float(Wo), What_gpu)
    e_ref = orc.output_error(Xs, Wo, orc.dequant(ref, r.scales, "e4m3", T, n, k))
    e_plain = orc.output_error(Xs, Wo, orc.dequant(r.codes, r.scales, "e4m3", T, n, k))
    assert e_gpu == pytest.approx(e_ref, rel=1e-3)
    assert e_gpu < 0.9 * e_plain


def test_rejections(mxq):
    W = torch.zeros(64, 96, dtype=torch.bfloat16, device=DEV)
    U = torch.zeros(2, T, T, device=DEV)
    s = torch.zeros(1, 2, device=DEV)
    with pytest.raises(mxq.MxqError):
        mxq.mxq_gptq_tiles(W, U, s)                 # k % 64 != 0
    with pytest.raises(mxq.MxqError):
        mxq.mxq_gptq_prepare(torch.zeros(1, T, T, device=DEV), float("nan"))
    with pytest.raises(mxq.MxqError):
        mxq.mxq_gptq_prepare(torch.zeros(1, T, T, device=DEV), -0.5)
