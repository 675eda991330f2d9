"""GPU parity: the CUDA path through the C-ABI against the CPU oracle, on the same bytes.

Bars (stated with each check):
 * element projection, codes, scales, dequantised values: bit-exact;
 * NVFP4 and INT8 picks: bit-exact in every block, near-ties included (the library
   re-scores near-ties in the definition's order); blocks whose two best candidate
   errors differ by < 1e-6 relative are also counted and reported;
 * E4M3 tile picks: bit-exact wherever the two best tile errors differ by >= 1e-6;
 * h: within 1e-5 relative; error sums: within 1e-5 relative.
"""
import os

import numpy as np
import pytest
import torch

from gpu_util import all_positive_bf16_f32, near_tie_mask, oracle_view

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


def e4m3_values(orc):
    return orc.e4m3_table()


# ---------------------------------------------------------------------------------------
# exhaustive element projection
# ---------------------------------------------------------------------------------------

def test_project_nvfp4_every_bf16_every_scale(mxq, orc):
    w = all_positive_bf16_f32(DEV)
    wc = w.cpu().numpy()
    tab = e4m3_values(orc)
    for c in range(1, 127):
        g = mxq.mxq_project(w, "nvfp4", float(tab[c])).cpu().numpy()
        r, _ = orc.project_many("nvfp4", c, wc)
        bad = np.nonzero(g != r)[0]
        assert bad.size == 0, f"scale code {c}: {bad.size} mismatches, e.g. w={wc[bad[:4]]}"
    g = mxq.mxq_project(-w, "nvfp4", 1.0).cpu().numpy()          # sign ignored
    assert np.array_equal(g, orc.project_many("nvfp4", 0x38, wc)[0])


def _near(values, ulps=3):
    v = np.asarray(values, np.float32)
    out = [v]
    lo, hi = v.copy(), v.copy()
    for _ in range(ulps):
        lo = np.nextafter(lo, np.float32(0))
        hi = np.nextafter(hi, np.float32(np.inf))
        out += [lo, hi]
    return np.concatenate(out)


def test_project_nvfp4_float32_near_every_boundary(mxq, orc):
    """float32 weights within 3 ulps of s * midpoint and s * grid value, every scale."""
    tab = e4m3_values(orc)
    pts = np.array([0.25, 0.5, 0.75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 6.5, 7],
                   np.float32)
    rng = np.random.default_rng(0)
    for c in range(1, 127):
        s = tab[c]
        base = (pts * s).astype(np.float32)
        rnd = (rng.random(4096) * 7 * s).astype(np.float32)
        wc = np.concatenate([_near(base), rnd])
        g = mxq.mxq_project(torch.from_numpy(wc).to(DEV), "nvfp4", float(s)).cpu().numpy()
        r, _ = orc.project_many("nvfp4", c, wc)
        assert np.array_equal(g, r), f"scale code {c}"


def test_project_int8_every_bf16_every_scale(mxq, orc):
    w = all_positive_bf16_f32(DEV)
    wc = w.cpu().numpy()
    tab = e4m3_values(orc)
    rng = np.random.default_rng(1)
    for c in range(1, 127):
        g = mxq.mxq_project(w, "int8", float(tab[c])).cpu().numpy()
        r, _ = orc.project_many("int8", c, wc)
        assert np.array_equal(g, r), f"scale code {c}"
        s_eff = np.float32(tab[c]) / np.float32(127)
        half = ((np.arange(128, dtype=np.float32) + np.float32(0.5)) * s_eff).astype(np.float32)
        wf = np.concatenate([_near(half), (rng.random(2048) * 130 * s_eff).astype(np.float32)])
        g = mxq.mxq_project(torch.from_numpy(wf).to(DEV), "int8", float(tab[c])).cpu().numpy()
        assert np.array_equal(g, orc.project_many("int8", c, wf)[0]), f"fp32, scale code {c}"


def test_project_e4m3_every_bf16(mxq, orc):
    w = all_positive_bf16_f32(DEV)
    wc = w.cpu().numpy()
    g64 = orc.log_grid(64, -2.0, 2.0)
    for amax in (1.0, 0.0371, 3.3e-3, 17.5):
        base = np.float32(amax) / np.float32(448)
        for p in range(0, 64, 3):
            s = np.float32(base * g64[p])
            g = mxq.mxq_project(w, "e4m3", float(s)).cpu().numpy()
            r, _ = orc.project_e4m3_many(float(s), wc)
            assert np.array_equal(g, r), f"amax {amax} point {p}"


# ---------------------------------------------------------------------------------------
# h pass
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols,dtype", [(512, 256, torch.float32), (1000, 264, torch.bfloat16),
                                             (3, 8, torch.bfloat16), (1, 4, torch.float32),
                                             (4133, 1544, torch.bfloat16), (257, 9728, torch.bfloat16)])
def test_act_sqmean_parity(mxq, orc, synth, rows, cols, dtype):
    X = synth.activations(rows, cols, 7, dtype=dtype, device=DEV)
    h = mxq.mxq_act_sqmean(X)
    ref = orc.act_sqmean(oracle_view(X))
    np.testing.assert_allclose(h.cpu().numpy(), ref, rtol=1e-5, atol=0)


def test_act_sqmean_strided_and_sharded(mxq, orc, synth):
    big = synth.activations(2000, 640, 8, dtype=torch.bfloat16, device=DEV)
    X = big[:, 64:576]                      # ld = 640 > cols = 512
    h = mxq.mxq_act_sqmean(X)
    ref = orc.act_sqmean(oracle_view(X))
    np.testing.assert_allclose(h.cpu().numpy(), ref, rtol=1e-5)
    parts = torch.stack([mxq.mxq_act_sqsum(X[:700]), mxq.mxq_act_sqsum(X[700:1333]),
                         mxq.mxq_act_sqsum(X[1333:])])
    h2 = mxq.mxq_act_sqmean_finalize(parts, 2000)
    np.testing.assert_allclose(h2.cpu().numpy(), ref, rtol=1e-5)
    refsum = orc.act_sqsum(oracle_view(X[:700]))
    np.testing.assert_allclose(parts[0].cpu().numpy(), refsum, rtol=1e-5)


def test_act_sqmean_deterministic(mxq, synth):
    X = synth.activations(5000, 1024, 9, dtype=torch.bfloat16, device=DEV)
    a = mxq.mxq_act_sqmean(X)
    b = mxq.mxq_act_sqmean(X)
    assert torch.equal(a, b)


# ---------------------------------------------------------------------------------------
# quantization
# ---------------------------------------------------------------------------------------

def run_pair(mxq, orc, W, fmt, mode, block, h=None, window=-1):
    p = mxq.params(fmt, mode, block, window=window)
    hd = None if h is None else torch.from_numpy(h).to(DEV)
    codes, scales = mxq.mxq_quantize(W, p, hd)
    torch.cuda.synchronize()
    r = orc.quantize(oracle_view(W), fmt, mode, block, h=h, window=window)
    return codes.cpu().numpy().view(np.uint8), scales.cpu().numpy(), r, p


def assert_blocks_equal(fmt, block, codes, scales, r, allow_near_tie=False, tag=""):
    n = scales.shape[0] if fmt != "e4m3" else scales.shape[0] * block
    near = near_tie_mask(r.best, r.second)
    if fmt == "e4m3":
        bad = scales != r.scales
        if allow_near_tie:
            bad &= ~near
        assert not bad.any(), f"{tag}: {bad.sum()} tiles differ"
        ok_tiles = ~(scales != r.scales)
        cg = codes.reshape(n // block, block, -1, block)
        co = r.codes.reshape(n // block, block, -1, block)
        tile_codes_equal = (cg == co).all(axis=(1, 3))
        assert tile_codes_equal[ok_tiles].all(), f"{tag}: codes differ in matching tiles"
        return int(near.sum())
    mism = scales != r.scales
    assert not mism.any(), (f"{tag}: {mism.sum()} of {mism.size} block scales differ "
                            f"({(mism & near).sum()} near ties), first at "
                            f"{np.argwhere(mism)[:3].tolist()}")
    assert np.array_equal(codes, r.codes.view(np.uint8)), f"{tag}: codes differ"
    return int(near.sum())


@pytest.mark.parametrize("mode", ["naive", "sse", "hopt"])
def test_quantize_tiny_workload(mxq, orc, synth, mode):
    """The tiny NVFP4 workload (W 64x256 fp32, X 512x256 fp32, block 16, all 126 scales)."""
    wl = synth.WORKLOADS["tiny_nvfp4"]
    W = synth.workload_weight(wl, 0, device=DEV)
    X = synth.workload_activations(wl, 0, device="cpu")
    h = orc.act_sqmean(oracle_view(X)) if mode == "hopt" else None
    codes, scales, r, _ = run_pair(mxq, orc, W, "nvfp4", mode, 16, h)
    assert_blocks_equal("nvfp4", 16, codes, scales, r, tag=f"tiny {mode}")


CASES = [("nvfp4", 16, -1), ("nvfp4", 32, -1), ("nvfp4", 16, 8), ("nvfp4", 32, 0),
         ("nvfp4", 16, 2), ("int8", 32, 8), ("int8", 64, 8), ("int8", 128, 8), ("int8", 256, 8),
         ("int8", 32, -1), ("int8", 64, 0)]


@pytest.mark.parametrize("fmt,block,window", CASES)
@pytest.mark.parametrize("mode", ["naive", "sse", "hopt"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_parity(mxq, orc, synth, fmt, block, window, mode, dtype):
    n, k = 37, 1024                          # ragged row count, several blocks per row
    W = synth.gaussian_weight(n, k, 21, dtype=dtype, device=DEV)
    h = None
    if mode == "hopt":
        X = synth.activations(300, k, 22, dtype=torch.bfloat16, device="cpu")
        h = orc.act_sqmean(oracle_view(X))
    codes, scales, r, _ = run_pair(mxq, orc, W, fmt, mode, block, h, window)
    assert_blocks_equal(fmt, block, codes, scales, r, tag=f"{fmt}{block} w{window} {mode}")


@pytest.mark.parametrize("mode", ["naive", "sse", "hopt"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_e4m3_tiles_parity(mxq, orc, synth, mode, dtype):
    W = synth.student_t_weight(192, 256, 31, dtype=dtype, device=DEV)   # 3 x 4 tiles
    h = None
    if mode == "hopt":
        X = synth.activations(500, 256, 32, dtype=torch.bfloat16, device="cpu", n_outlier=0)
        h = orc.act_sqmean(oracle_view(X))
    codes, scales, r, _ = run_pair(mxq, orc, W, "e4m3", mode, 64, h)
    near = assert_blocks_equal("e4m3", 64, codes, scales, r, allow_near_tie=True,
                               tag=f"e4m3 {mode}")
    print(f"e4m3 tiles {mode}: {near} near-tie tiles of {scales.size}")


def special_blocks(B):
    rows = [np.zeros(B), -np.zeros(B), np.ones(B), np.full(B, 1e-5), np.full(B, -3e-7),
            np.r_[6.0, np.zeros(B - 1)], np.r_[np.zeros(B - 1), -448.0 * 6],
            np.r_[3e38, np.ones(B - 1)], np.full(B, 2.0 ** -133), np.r_[1e-38, -1e-39, np.zeros(B - 2)],
            np.linspace(-1, 1, B), np.full(B, 0.5) * (-1) ** np.arange(B),
            np.r_[100.0, np.full(B - 1, 0.7)], np.full(B, 1000.0), np.full(B, 2.0 ** -10 * 6)]
    return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("fmt,block", [("nvfp4", 16), ("nvfp4", 32), ("int8", 32), ("int8", 64)])
@pytest.mark.parametrize("mode", ["naive", "sse", "hopt"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_special_blocks(mxq, orc, fmt, block, mode, dtype):
    """Zeros, signed zeros, a zero naive scale, saturation, huge and subnormal values,
    exact ties between candidate scales."""
    Wn = special_blocks(block)
    W = torch.from_numpy(Wn).to(dtype).to(DEV)
    h = np.exp(np.random.default_rng(5).normal(0, 1, block)).astype(np.float32) \
        if mode == "hopt" else None
    for window in (-1, 8):
        codes, scales, r, _ = run_pair(mxq, orc, W, fmt, mode, block, h, window)
        assert_blocks_equal(fmt, block, codes, scales, r, tag=f"special {fmt}{block} {mode}")


def test_quantize_strided_input(mxq, orc, synth):
    big = synth.gaussian_weight(40, 1536, 41, dtype=torch.bfloat16, device=DEV)
    W = big[:, 256:1280]
    Wc = W.contiguous()
    p = mxq.params("nvfp4", "sse", 16)
    a = mxq.mxq_quantize(W, p)
    b = mxq.mxq_quantize(Wc, p)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_quantize_empty(mxq):
    W = torch.empty(0, 256, dtype=torch.bfloat16, device=DEV)
    codes, scales = mxq.mxq_quantize(W, mxq.params("nvfp4", "sse", 16))
    assert codes.numel() == 0 and scales.numel() == 0


# ---------------------------------------------------------------------------------------
# dequant and error metrics
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("fmt,block,mode", [("nvfp4", 16, "hopt"), ("nvfp4", 32, "sse"),
                                            ("int8", 64, "hopt"), ("int8", 256, "naive"),
                                            ("e4m3", 64, "hopt")])
def test_dequant_and_error_parity(mxq, orc, synth, fmt, block, mode):
    n, k = (128, 512) if fmt == "e4m3" else (45, 512)
    W = synth.gaussian_weight(n, k, 51, dtype=torch.bfloat16, device=DEV)
    X = synth.activations(256, k, 52, dtype=torch.bfloat16, device="cpu")
    h = orc.act_sqmean(oracle_view(X))
    hd = torch.from_numpy(h).to(DEV)
    p = mxq.params(fmt, mode, block)
    # the oracle's quantization, uploaded: both sides decode and measure the same codes
    r = orc.quantize(oracle_view(W), fmt, mode, block, h=h if mode == "hopt" else None)
    c_np, s_np = r.codes, r.scales
    codes, scales = torch.from_numpy(c_np).to(DEV), torch.from_numpy(s_np).to(DEV)
    What = mxq.mxq_dequant(codes, scales, p, n, k)
    sums = mxq.mxq_error(W, codes, scales, p, hd)
    torch.cuda.synchronize()
    ref = orc.dequant(c_np, s_np, fmt, block, n, k)
    assert np.array_equal(What.cpu().numpy(), ref)
    rs = orc.error_sums(oracle_view(W), ref, h)
    np.testing.assert_allclose(sums.cpu().numpy(), rs, rtol=1e-5)
    m = mxq.mxq_metrics_from_sums(sums.cpu())
    mo = orc.metrics(rs)
    assert m["weight_rel"] == pytest.approx(mo["weight_rel"], rel=1e-5)
    assert m["h_rel"] == pytest.approx(mo["h_rel"], rel=1e-5)
    sums0 = mxq.mxq_error(W, codes, scales, p, None).cpu().numpy()
    assert sums0[2] == 0 and sums0[3] == 0
    np.testing.assert_allclose(sums0[:2], rs[:2], rtol=1e-5)


@pytest.mark.parametrize("fmt,block,mode,with_h", [("nvfp4", 16, "hopt", True),
                                                   ("nvfp4", 32, "hopt", True),
                                                   ("nvfp4", 16, "sse", True),
                                                   ("nvfp4", 32, "sse", False),
                                                   ("nvfp4", 16, "naive", True),
                                                   ("int8", 64, "hopt", True),
                                                   ("e4m3", 64, "hopt", True)])
def test_quantize_with_error_sums(mxq, orc, synth, fmt, block, mode, with_h):
    """mxq_quantize_err: the same codes and scales as mxq_quantize, bit for bit, and the
    error sums of the oracle's quantization (equal to the GPU's, checked first) at 1e-5; the
    NVFP4 searches add the sums inside the search (ragged row count: 77 rows)."""
    n, k = (128, 512) if fmt == "e4m3" else (77, 1024)
    W = synth.gaussian_weight(n, k, 81, dtype=torch.bfloat16, device=DEV)
    X = synth.activations(256, k, 82, dtype=torch.bfloat16, device="cpu")
    h = orc.act_sqmean(oracle_view(X))
    hd = torch.from_numpy(h).to(DEV) if with_h else None
    p = mxq.params(fmt, mode, block)
    c1, s1 = mxq.mxq_quantize(W, p, hd)
    c2, s2, sums = mxq.mxq_quantize_err(W, p, hd)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2)
    r = orc.quantize(oracle_view(W), fmt, mode, block, h=h if mode == "hopt" else None)
    if fmt != "e4m3":              # (tiles are bit-exact outside near ties: tested elsewhere)
        assert np.array_equal(c2.cpu().numpy().view(np.uint8), r.codes.view(np.uint8))
        assert np.array_equal(s2.cpu().numpy(), r.scales)
    What = orc.dequant(r.codes, r.scales, fmt, block, n, k)
    ref = orc.error_sums(oracle_view(W), What, h if with_h else None)
    np.testing.assert_allclose(sums.cpu().numpy(), ref, rtol=1e-5, atol=0)
    again = mxq.mxq_quantize_err(W, p, hd)[2]
    assert torch.equal(sums, again)                     # deterministic


@pytest.mark.parametrize("B,mode", [(16, "hopt"), (32, "hopt"), (32, "sse")])
def test_search_occupancy_setting(mxq, orc, synth, B, mode):
    """ctas_per_sm limits the NVFP4 search's persistent grid (room for a concurrent h pass):
    the codes and scales are the same for every setting, and the fused error sums agree with
    the oracle's (they group the blocks by CTA, so only the last bits may move)."""
    n, k = 300, 2048
    W = synth.gaussian_weight(n, k, 91, dtype=torch.bfloat16, device=DEV)
    X = synth.activations(256, k, 92, dtype=torch.bfloat16, device="cpu")
    h = orc.act_sqmean(oracle_view(X))
    hd = torch.from_numpy(h).to(DEV)
    r = orc.quantize(oracle_view(W), "nvfp4", mode, B, h=h if mode == "hopt" else None)
    ref = orc.error_sums(oracle_view(W), orc.dequant(r.codes, r.scales, "nvfp4", B, n, k),
                         h if mode == "hopt" else None)
    for cps in (0, 1, 2, 3, 9):
        p = mxq.params("nvfp4", mode, B, ctas_per_sm=cps)
        c, s, sums = mxq.mxq_quantize_err(W, p, hd if mode == "hopt" else None)
        assert np.array_equal(c.cpu().numpy(), r.codes) and np.array_equal(s.cpu().numpy(), r.scales)
        np.testing.assert_allclose(sums.cpu().numpy(), ref, rtol=1e-5)


def test_error_deterministic(mxq, synth):
    W = synth.gaussian_weight(512, 4096, 61, dtype=torch.bfloat16, device=DEV)
    p = mxq.params("nvfp4", "naive", 16)
    codes, scales = mxq.mxq_quantize(W, p)
    a = mxq.mxq_error(W, codes, scales, p).cpu()
    b = mxq.mxq_error(W, codes, scales, p).cpu()
    assert torch.equal(a, b)
