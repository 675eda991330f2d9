"""Output error on the tensor cores against float64 products of the oracle's dequantised
weights (qwantize "Results": ||X_s Wq^T - X_s W^T||_F / ||X_s W^T||_F).

The codes come from the oracle's quantizer (uploaded), so both sides use the same Wq.
Tolerance: the GPU accumulates the bf16 products (exact) in float32 inside the tensor cores
over k terms. That accumulation need not round to nearest (an error biased in one direction
grows like k 2^-23 rather than sqrt(k) 2^-24), so each entry of Y carries up to ~k 2^-24
relative error of sum |x w| in practice: 1e-4 on ||Y||^2 at k <= 10^4, and on the difference
Yq - Y (a few percent of Y) 20x that, 5e-3 on its squared norm (3e-3 on their ratio).
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


def reference_sums(orc, X, W, codes, scales, fmt, block, sfmt):
    n, k = W.shape
    What = orc.dequant(codes, scales, fmt, block, n, k, sfmt=sfmt).astype(np.float64)
    Xf = orc.to_float(oracle_view(X)).astype(np.float64)
    Wf = orc.to_float(oracle_view(W)).astype(np.float64)
    Y = Xf @ Wf.T
    Yq = Xf @ What.T
    return np.array([np.sum((Yq - Y) ** 2), np.sum(Y ** 2)])


@pytest.mark.parametrize("m,n,k", [(256, 128, 512), (200, 100, 544), (128, 64, 64),
                                   (384, 320, 2048)])
@pytest.mark.parametrize("fmt,sfmt,block", [("nvfp4", "e4m3", 16), ("nvfp4", "ue8m0", 32),
                                            ("int4", "e4m3", 16)])
def test_output_error_matches_float64(mxq, orc, synth, m, n, k, fmt, sfmt, block):
    X = synth.activations(m, k, 101, dtype=torch.bfloat16, device=DEV)
    W = synth.gaussian_weight(n, k, 102, dtype=torch.bfloat16, device=DEV)
    h = orc.act_sqmean(oracle_view(X))
    r = orc.quantize(oracle_view(W), fmt, "hopt", block, h=h, sfmt=sfmt)
    p = mxq.params(fmt, "hopt", block, scale_fmt=sfmt)
    sums = mxq.mxq_output_error(X, W, torch.from_numpy(r.codes).to(DEV),
                                torch.from_numpy(r.scales).to(DEV), p).cpu().numpy()
    ref = reference_sums(orc, X, W, r.codes, r.scales, fmt, block, sfmt)
    assert np.isfinite(sums).all()
    np.testing.assert_allclose(sums[0], ref[0], rtol=5e-3)
    np.testing.assert_allclose(sums[1], ref[1], rtol=1e-4)


def test_output_error_zero_for_exact_weights(mxq, orc, synth):
    """Weights that NVFP4 represents exactly (codebook values times E4M3 scales) give a zero
    difference: both products accumulate the same exact terms in the same order."""
    k, n = 256, 64
    rng = np.random.default_rng(3)
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    W = (vals[rng.integers(0, 8, (n, k))] * rng.choice([-1, 1], (n, k))).astype(np.float32)
    W[:, ::16] = 6.0                                  # amax 6 in every block: scale 1.0
    Wt = torch.from_numpy(W).to(torch.bfloat16).to(DEV)
    X = synth.activations(128, k, 104, dtype=torch.bfloat16, device=DEV)
    r = orc.quantize(oracle_view(Wt), "nvfp4", "naive", 16)
    assert np.all(r.scales == 0x38)
    p = mxq.params("nvfp4", "naive", 16)
    sums = mxq.mxq_output_error(X, Wt, torch.from_numpy(r.codes).to(DEV),
                                torch.from_numpy(r.scales).to(DEV), p).cpu().numpy()
    assert sums[0] == 0.0 and sums[1] > 0


@pytest.mark.slow
def test_output_error_full_calibration_shape(mxq, orc, synth):
    """The pages' metric shape: 512 sampled rows of X against W 2560 x 9728, NVFP4 block 16."""
    wl = synth.WORKLOADS["nvfp4_full_calib"]
    W = synth.workload_weight(wl, 0, device=DEV)
    Xs = synth.workload_activations(wl, 0, device=DEV, rows=512)
    h = orc.act_sqmean(oracle_view(Xs))
    r = orc.quantize(oracle_view(W), "nvfp4", "hopt", 16, h=h, n_threads=16)
    p = mxq.params("nvfp4", "hopt", 16)
    sums = mxq.mxq_output_error(Xs, W, torch.from_numpy(r.codes).to(DEV),
                                torch.from_numpy(r.scales).to(DEV), p).cpu().numpy()
    ref = reference_sums(orc, Xs, W, r.codes, r.scales, "nvfp4", 16, "e4m3")
    np.testing.assert_allclose(sums[0], ref[0], rtol=5e-3)
    np.testing.assert_allclose(sums[1], ref[1], rtol=1e-4)
    rel = (sums[0] / sums[1]) ** 0.5
    assert rel == pytest.approx(orc.output_error(oracle_view(Xs), oracle_view(W),
                                                 orc.dequant(r.codes, r.scales, "nvfp4", 16,
                                                             2560, 9728)), rel=3e-3)
