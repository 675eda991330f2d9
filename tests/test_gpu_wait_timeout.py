"""The failure path of the tensor-core kernels, exercised on purpose and without a fault.

Every pipeline wait of the four tensor-core kernels (block Gram pass, full Gram matrix,
output error, block-scaled NVFP4 product) is a bounded poll of an mbarrier. Here the bound
is lowered to one poll (mxq_set_wait_polls), so that the first wait that is not already
satisfied runs out: the kernel must then set its error word, let its own copies and MMAs
finish, free its tensor memory and return, and the call's outputs must come back as NaN.
The bound is then restored and the same call, in the same process and context, must give
the normal result bit for bit -- nothing was left allocated, locked or corrupted.
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


def timed_out_then_normal(mxq, call):
    """call() under a one-poll bound, then under the default; both results (host copies)."""
    good = call()
    torch.cuda.synchronize()
    mxq.mxq_set_wait_polls(1)
    try:
        bad = call()
        torch.cuda.synchronize()
    finally:
        mxq.mxq_set_wait_polls(0)
    again = call()
    torch.cuda.synchronize()
    return good.cpu(), bad.cpu(), again.cpu()


def test_block_gram_wait_runs_out(mxq, synth):
    X = synth.activations(4096, 512, 7, dtype=torch.bfloat16, device=DEV)
    good, bad, again = timed_out_then_normal(mxq, lambda: mxq.mxq_act_block_gram(X, 16))
    assert torch.isnan(bad).all()
    assert torch.isfinite(good).all() and torch.equal(again, good)


def test_full_gram_wait_runs_out(mxq, synth):
    X = synth.activations(4096, 1024, 8, dtype=torch.bfloat16, device=DEV)
    good, bad, again = timed_out_then_normal(mxq, lambda: mxq.mxq_act_gram(X))
    assert torch.isnan(bad).all()
    assert torch.isfinite(good).all() and torch.equal(again, good)


def test_output_error_wait_runs_out(mxq, synth):
    X = synth.activations(512, 1024, 9, dtype=torch.bfloat16, device=DEV)
    W = synth.gaussian_weight(256, 1024, 10, dtype=torch.bfloat16, device=DEV)
    p = mxq.params("nvfp4", "naive", 16)
    codes, scales = mxq.mxq_quantize(W, p)
    good, bad, again = timed_out_then_normal(
        mxq, lambda: mxq.mxq_output_error(X, W, codes, scales, p))
    assert torch.isnan(bad).all()
    assert torch.isfinite(good).all() and torch.equal(again, good)


def test_nvfp4_product_wait_runs_out(mxq, synth):
    A = synth.gaussian_weight(256, 2048, 11, dtype=torch.bfloat16, device=DEV)
    Bm = synth.gaussian_weight(256, 2048, 12, dtype=torch.bfloat16, device=DEV)
    p = mxq.params("nvfp4", "naive", 16)
    ca, sa = mxq.mxq_quantize(A, p)
    cb, sb = mxq.mxq_quantize(Bm, p)
    swa, swb = mxq.mxq_swizzle_scales(sa), mxq.mxq_swizzle_scales(sb)
    good, bad, again = timed_out_then_normal(
        mxq, lambda: mxq.mxq_nvfp4_gemm(ca, swa, cb, swb, 256, 256, 2048))
    assert torch.isnan(bad).all()
    assert torch.isfinite(good).all() and torch.equal(again, good)
    # the default bound is back: a larger product is still correct afterwards
    assert np.isfinite(mxq.mxq_nvfp4_gemm(ca, swa, cb, swb, 256, 256, 2048).cpu().numpy()).all()
