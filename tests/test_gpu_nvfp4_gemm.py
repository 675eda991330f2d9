"""The NVFP4 x NVFP4 product on the block-scaled tensor cores (mxq_nvfp4_gemm) against the
oracle.

The operands are the oracle's own NVFP4 quantization -- E2M1 codes and one E4M3 scale per 16
elements ("Is Finer Better? The Limits of Microscaling Formats in LLMs", sec. 2.1) --
uploaded; their scales go through mxq_swizzle_scales into the 128 x 4 tile layout that the
block-scaled MMA reads. The expected product is the oracle's float64 product of the two
dequantised matrices. Each product of two scaled E2M1 values is exact and the tensor cores
accumulate in float32, so |D - ref| <= (k + 2) 2^-24 (|A^| |B^|^T) entry by entry.

The layout is proven against the hardware, not only against the oracle's restatement of it:
two scales of one row swapped by hand must move that row of the result to the product with
the swapped scales (and away from the original), and row-major scales passed where the
swizzled ones belong must not reproduce the product.
"""
import numpy as np
import pytest
import torch

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


def oracle_nvfp4(orc, W_bits, mode, h=None):
    r = orc.quantize(W_bits, "nvfp4", mode, 16, h=h, n_threads=8)
    return r.codes.view(np.uint8), r.scales.astype(np.uint8)


def gpu_product(mxq, ca, sa, cb, sb, m, n, k):
    sw_a = mxq.mxq_swizzle_scales(torch.from_numpy(np.ascontiguousarray(sa)).to(DEV))
    sw_b = mxq.mxq_swizzle_scales(torch.from_numpy(np.ascontiguousarray(sb)).to(DEV))
    D = mxq.mxq_nvfp4_gemm(torch.from_numpy(ca).to(DEV), sw_a, torch.from_numpy(cb).to(DEV),
                           sw_b, m, n, k)
    torch.cuda.synchronize()
    return D.cpu().numpy().astype(np.float64)


def reference(orc, ca, sa, cb, sb, m, n, k):
    A = orc.dequant(ca, sa, "nvfp4", 16, m, k).astype(np.float64)
    B = orc.dequant(cb, sb, "nvfp4", 16, n, k).astype(np.float64)
    return A @ B.T, (k + 2) * 2.0 ** -24 * (np.abs(A) @ np.abs(B).T) + 1e-30


def operands(orc, synth, m, n, k, seed):
    Wa = synth.gaussian_weight(m, k, seed, dtype=torch.bfloat16)
    Wb = synth.gaussian_weight(n, k, seed + 1, dtype=torch.bfloat16)
    X = synth.activations(256, k, seed + 2, dtype=torch.bfloat16)
    h = orc.act_sqmean(X.view(torch.int16).numpy().view(np.uint16))
    ca, sa = oracle_nvfp4(orc, Wa.view(torch.int16).numpy().view(np.uint16), "naive")
    cb, sb = oracle_nvfp4(orc, Wb.view(torch.int16).numpy().view(np.uint16), "hopt", h)
    return ca, sa, cb, sb


@pytest.mark.parametrize("m,n,k", [(128, 128, 256), (200, 72, 320), (300, 500, 1024),
                                   (33, 17, 64), (129, 257, 576)])
def test_product_matches_oracle(mxq, orc, synth, m, n, k):
    ca, sa, cb, sb = operands(orc, synth, m, n, k, 300 + m)
    D = gpu_product(mxq, ca, sa, cb, sb, m, n, k)
    ref, tol = reference(orc, ca, sa, cb, sb, m, n, k)
    err = np.abs(D - ref)
    assert np.all(err <= tol), float((err / tol).max())


def test_product_full_width(mxq, orc, synth):
    """The full-calibration shapes' inner dimension (k = 9728, 38 stages of 256): 512 rows of
    the activations quantized naively (the activation side of a W4A4 product) times 384 rows
    of the weight quantized H-optimally."""
    wl = synth.WORKLOADS["nvfp4_full_calib"]
    X = synth.workload_activations(wl, 0, rows=16384)
    Xb = X.view(torch.int16).numpy().view(np.uint16)
    h = orc.act_sqmean(Xb)
    W = synth.workload_weight(wl, 0, rows=384)
    ca, sa = oracle_nvfp4(orc, np.ascontiguousarray(Xb[:512]), "naive")
    cb, sb = oracle_nvfp4(orc, W.view(torch.int16).numpy().view(np.uint16), "hopt", h)
    m, n, k = 512, 384, X.shape[1]
    D = gpu_product(mxq, ca, sa, cb, sb, m, n, k)
    ref, tol = reference(orc, ca, sa, cb, sb, m, n, k)
    err = np.abs(D - ref)
    assert np.all(err <= tol), float((err / tol).max())
    print(f"NVFP4 product 512 x 384 x {k}: largest error / bound {float((err / tol).max()):.3g}")


def test_scale_positions_are_read_where_the_swizzle_puts_them(mxq, orc, synth):
    m, n, k = 200, 72, 320
    ca, sa, cb, sb = operands(orc, synth, m, n, k, 400)
    ref, tol = reference(orc, ca, sa, cb, sb, m, n, k)
    # two different scales of A's row 37 (second 32-row group of the tile), swapped
    r = 37
    c1 = 0
    c2 = int(np.nonzero(sa[r] != sa[r, c1])[0][0])
    sa2 = sa.copy()
    sa2[r, c1], sa2[r, c2] = sa[r, c2], sa[r, c1]
    D2 = gpu_product(mxq, ca, sa2, cb, sb, m, n, k)
    ref2, tol2 = reference(orc, ca, sa2, cb, sb, m, n, k)
    assert np.all(np.abs(D2 - ref2) <= tol2)
    assert np.any(np.abs(D2[r] - ref[r]) > tol[r])           # the swap moved row r ...
    others = np.arange(m) != r
    assert np.all(np.abs(D2[others] - ref[others]) <= tol[others])   # ... and nothing else
    # row-major scale bytes where the swizzled ones belong: not the product
    flat = np.zeros(mxq.mxq_swizzle_scales(torch.from_numpy(sa).to(DEV)).numel(), np.uint8)
    flat[:sa.size] = sa.reshape(-1)
    sw_b = mxq.mxq_swizzle_scales(torch.from_numpy(sb).to(DEV))
    D3 = mxq.mxq_nvfp4_gemm(torch.from_numpy(ca).to(DEV), torch.from_numpy(flat).to(DEV),
                            torch.from_numpy(cb).to(DEV), sw_b, m, n, k).cpu().numpy()
    assert np.any(np.abs(D3.astype(np.float64) - ref) > tol)


def test_repeatable(mxq, orc, synth):
    m, n, k = 300, 500, 1024
    ca, sa, cb, sb = operands(orc, synth, m, n, k, 500)
    a = gpu_product(mxq, ca, sa, cb, sb, m, n, k)
    b = gpu_product(mxq, ca, sa, cb, sb, m, n, k)
    assert np.array_equal(a, b)
