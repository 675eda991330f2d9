"""GPU parity for E2M1 and INT4 elements on the other block-scale grids: MXFP4 (UE8M0),
NVINT4 (INT4 on E4M3), UE4M4 and UE5M3 -- the CUDA path through the C-ABI against the CPU
oracle, on the same bytes.

Bars: element projection, codes, scales and dequantised values bit-exact; picks bit-exact
in every block, near-ties included (flagged blocks are re-scored in the definition's order);
error sums within 1e-5 relative.
"""
import numpy as np
import pytest
import torch

from gpu_util import all_positive_bf16_f32, oracle_view

pytestmark = pytest.mark.gpu
DEV = "cuda"

COMBOS = [("nvfp4", "ue8m0"), ("nvfp4", "ue4m4"), ("nvfp4", "ue5m3"), ("int4", "e4m3"),
          ("int4", "ue4m4"), ("int4", "ue5m3")]


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


@pytest.mark.parametrize("fmt,sfmt", COMBOS)
def test_project_every_bf16(mxq, orc, fmt, sfmt):
    """Every finite positive bf16 value at every 5th scale code plus both ends."""
    w = all_positive_bf16_f32(DEV)
    wc = w.cpu().numpy()
    tab = orc.scale_table(sfmt)
    first = 0 if sfmt == "ue8m0" else 1
    codes = sorted(set(range(first, len(tab), 5)) | {first, first + 1, len(tab) - 1})
    for c in codes:
        g = mxq.mxq_project(w, fmt, float(tab[c]), scale_fmt=sfmt).cpu().numpy()
        r, _ = orc.project_many(fmt, c, wc, sfmt=sfmt)
        bad = np.nonzero(g != r)[0]
        assert bad.size == 0, f"{sfmt} code {c}: {bad.size} mismatches, e.g. w={wc[bad[:4]]}"


def run_pair(mxq, orc, W, fmt, sfmt, mode, block, h=None, window=-1):
    p = mxq.params(fmt, mode, block, window=window, scale_fmt=sfmt)
    hd = None if h is None else torch.from_numpy(h).to(DEV)
    codes, scales = mxq.mxq_quantize(W, p, hd)
    torch.cuda.synchronize()
    r = orc.quantize(oracle_view(W), fmt, mode, block, h=h, window=window, sfmt=sfmt)
    return codes.cpu().numpy(), scales.cpu().numpy(), r


def assert_equal(codes, scales, r, tag):
    mism = scales != r.scales
    assert not mism.any(), (f"{tag}: {mism.sum()} of {mism.size} scales differ, first at "
                            f"{np.argwhere(mism)[:3].tolist()}")
    assert np.array_equal(codes, r.codes), f"{tag}: codes differ"


@pytest.mark.parametrize("fmt,sfmt", COMBOS)
@pytest.mark.parametrize("block,window", [(16, -1), (32, -1), (16, 3)])
@pytest.mark.parametrize("mode", ["naive", "sse", "hopt"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_parity(mxq, orc, synth, fmt, sfmt, block, window, mode, dtype):
    n, k = 37, 1024                          # ragged row count, several blocks per row
    W = synth.gaussian_weight(n, k, 61, dtype=dtype, device=DEV)
    h = None
    if mode == "hopt":
        X = synth.activations(300, k, 62, dtype=torch.bfloat16, device="cpu")
        h = orc.act_sqmean(oracle_view(X))
    codes, scales, r = run_pair(mxq, orc, W, fmt, sfmt, mode, block, h, window)
    assert_equal(codes, scales, r, f"{fmt}/{sfmt} b{block} w{window} {mode}")


def special_blocks(B):
    rows = [np.zeros(B), -np.zeros(B), np.ones(B), np.full(B, 1e-5), np.full(B, -3e-7),
            np.r_[6.0, np.zeros(B - 1)], np.r_[np.zeros(B - 1), -448.0 * 6],
            np.r_[3e38, np.ones(B - 1)], np.full(B, 2.0 ** -133),
            np.r_[1e-38, -1e-39, np.zeros(B - 2)], np.full(B, 3 * 2.0 ** -128),
            np.linspace(-1, 1, B), np.full(B, 0.5) * (-1) ** np.arange(B),
            np.r_[100.0, np.full(B - 1, 0.7)], np.full(B, 1000.0), np.full(B, 2.0),
            np.full(B, 7.0), np.full(B, 2.0 ** 120)]
    return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("fmt,sfmt", COMBOS)
@pytest.mark.parametrize("block", [16, 32])
@pytest.mark.parametrize("mode", ["naive", "sse", "hopt"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_special_blocks(mxq, orc, fmt, sfmt, block, mode, dtype):
    """Zeros, signed zeros, zero naive scales, saturation, huge, tiny and subnormal values
    (scales down to 2^-127 on UE8M0), exact ties between candidate scales."""
    W = torch.from_numpy(special_blocks(block)).to(dtype).to(DEV)
    h = np.exp(np.random.default_rng(5).normal(0, 1, block)).astype(np.float32) \
        if mode == "hopt" else None
    for window in (-1, 2):
        codes, scales, r = run_pair(mxq, orc, W, fmt, sfmt, mode, block, h, window)
        assert_equal(codes, scales, r, f"special {fmt}/{sfmt} b{block} {mode} w{window}")


@pytest.mark.parametrize("fmt,sfmt", COMBOS)
def test_dequant_and_error_parity(mxq, orc, synth, fmt, sfmt):
    n, k = 45, 512
    W = synth.gaussian_weight(n, k, 71, dtype=torch.bfloat16, device=DEV)
    X = synth.activations(256, k, 72, dtype=torch.bfloat16, device="cpu")
    h = orc.act_sqmean(oracle_view(X))
    hd = torch.from_numpy(h).to(DEV)
    p = mxq.params(fmt, "hopt", 16, scale_fmt=sfmt)
    # the oracle's quantization, uploaded: both sides decode and measure the same codes
    r = orc.quantize(oracle_view(W), fmt, "hopt", 16, h=h, sfmt=sfmt)
    codes, scales = torch.from_numpy(r.codes).to(DEV), torch.from_numpy(r.scales).to(DEV)
    What = mxq.mxq_dequant(codes, scales, p, n, k)
    sums = mxq.mxq_error(W, codes, scales, p, hd)
    torch.cuda.synchronize()
    ref = orc.dequant(r.codes, r.scales, fmt, 16, n, k, sfmt=sfmt)
    assert np.array_equal(What.cpu().numpy(), ref)
    rs = orc.error_sums(oracle_view(W), ref, h)
    np.testing.assert_allclose(sums.cpu().numpy(), rs, rtol=1e-5)


def test_ue8m0_nan_scale_decodes_to_nan(mxq):
    p = mxq.params("nvfp4", "naive", 16, scale_fmt="ue8m0")
    codes = torch.full((1, 8), 0x22, dtype=torch.uint8, device=DEV)
    scales = torch.tensor([[255]], dtype=torch.uint8, device=DEV)
    out = mxq.mxq_dequant(codes, scales, p, 1, 16).cpu()
    assert torch.isnan(out).all()


@pytest.mark.parametrize("n,kb", [(300, 10), (128, 4), (2560, 608), (37, 2)])
def test_swizzle_scales_matches_oracle(mxq, orc, n, kb):
    s = torch.randint(0, 256, (n, kb), dtype=torch.uint8, device=DEV)
    out = mxq.mxq_swizzle_scales(s).cpu().numpy()
    assert np.array_equal(out, orc.swizzle_scales(s.cpu().numpy()))
