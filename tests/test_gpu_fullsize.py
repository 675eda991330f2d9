"""Full-size parity: every workload at its full shape on the GPU (the launch shapes the
benchmark times), checked against the oracle on seeded samples of rows (the oracle computes
those outputs one block at a time) and, for h, on the whole activation matrix.

The oracle receives only its own inputs: h for the quantizer comparisons is the oracle's h
(uploaded to the GPU), so the search is compared in isolation; the h pass is compared on its
own; and one end-to-end check runs each side on its own h.
"""
import os

import numpy as np
import pytest
import torch

from gpu_util import near_tie_mask, oracle_view, order_with_ties

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"
NT = os.cpu_count() or 1


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


def sampled_parity(mxq, orc, W, fmt, block, mode, h_np, window, rows, tag, sfmt="e4m3"):
    """Quantize all of W on the GPU; compare `rows` with the oracle; return near-tie count."""
    p = mxq.params(fmt, mode, block, window=window, scale_fmt=sfmt)
    hd = None if h_np is None else torch.from_numpy(h_np).to(DEV)
    codes, scales = mxq.mxq_quantize(W, p, hd)
    torch.cuda.synchronize()
    Ws = oracle_view(W[torch.as_tensor(rows, device=W.device)])
    r = orc.quantize(Ws, fmt, mode, block, h=h_np, window=window, n_threads=NT, sfmt=sfmt)
    if fmt == "e4m3":
        raise AssertionError("use tile_parity for e4m3")
    g_codes = codes[torch.as_tensor(rows, device=W.device)].cpu().numpy().view(np.uint8)
    g_scales = scales[torch.as_tensor(rows, device=W.device)].cpu().numpy()
    bad = g_scales != r.scales
    near = near_tie_mask(r.best, r.second)
    assert not bad.any(), f"{tag}: {bad.sum()} of {bad.size} sampled blocks differ " \
                          f"({(bad & near).sum()} in near ties)"
    assert np.array_equal(g_codes, r.codes.view(np.uint8)), f"{tag}: codes differ"
    return int(near.sum()), int(near.size)


def test_nvfp4_full_calibration(mxq, orc, synth):
    wl = synth.WORKLOADS["nvfp4_full_calib"]
    (_, n, k), (R, _) = wl.weights[0], wl.x_shapes[0]
    X = synth.workload_activations(wl, 0, device=DEV)               # 4.76 GB
    h_gpu = mxq.mxq_act_sqmean(X)
    torch.cuda.synchronize()
    Xh = oracle_view(X)
    del X
    torch.cuda.empty_cache()
    h_orc = orc.act_sqmean(Xh, n_threads=NT)
    del Xh
    np.testing.assert_allclose(h_gpu.cpu().numpy(), h_orc, rtol=1e-5)
    W = synth.workload_weight(wl, 0, device=DEV)
    rows = synth.sample_rows(n, 48, wl.seed).numpy()
    for block in (16, 32):
        for mode in ("naive", "sse", "hopt"):
            near, tot = sampled_parity(mxq, orc, W, "nvfp4", block, mode,
                                       h_orc if mode == "hopt" else None, -1, rows,
                                       f"nvfp4 bs{block} {mode}")
            print(f"nvfp4 bs{block} {mode}: {tot} sampled blocks bit-exact, {near} near ties")
    # end to end: each side on its own h; picks may differ only where the h difference
    # (<= ~2e-6 relative) can move a block whose two best errors are within 1e-5
    p = mxq.params("nvfp4", "hopt", 16)
    codes, scales = mxq.mxq_quantize(W, p, h_gpu)
    r = orc.quantize(oracle_view(W[torch.as_tensor(rows, device=DEV)]), "nvfp4", "hopt", 16,
                     h=h_orc, n_threads=NT)
    g = scales[torch.as_tensor(rows, device=DEV)].cpu().numpy()
    bad = g != r.scales
    assert not (bad & ~near_tie_mask(r.best, r.second, rel=1e-5)).any()


@pytest.mark.parametrize("block", [32, 64, 128, 256])
def test_int8_e4m3_scales(mxq, orc, synth, block):
    wl = synth.WORKLOADS["int8_e4m3scale"]
    (_, n, k), _ = wl.weights[0], wl.x_shapes[0]
    X = synth.workload_activations(wl, 0, device=DEV)
    h_gpu = mxq.mxq_act_sqmean(X)
    h_orc = orc.act_sqmean(oracle_view(X), n_threads=NT)
    np.testing.assert_allclose(h_gpu.cpu().numpy(), h_orc, rtol=1e-5)
    W = synth.workload_weight(wl, 0, device=DEV)
    rows = synth.sample_rows(n, 24, wl.seed + block).numpy()
    for mode in ("naive", "sse", "hopt"):
        near, tot = sampled_parity(mxq, orc, W, "int8", block, mode,
                                   h_orc if mode == "hopt" else None, 8, rows,
                                   f"int8 bs{block} {mode}")
        print(f"int8 bs{block} {mode}: {tot} sampled blocks bit-exact, {near} near ties")


def test_e4m3_tiles_full(mxq, orc, synth):
    wl = synth.WORKLOADS["e4m3_tiles"]
    (_, n, k), _ = wl.weights[0], wl.x_shapes[0]
    X = synth.workload_activations(wl, 0, device=DEV)
    h_gpu = mxq.mxq_act_sqmean(X)
    h_orc = orc.act_sqmean(oracle_view(X), n_threads=NT)
    np.testing.assert_allclose(h_gpu.cpu().numpy(), h_orc, rtol=1e-5)
    W = synth.workload_weight(wl, 0, device=DEV)
    p = mxq.params("e4m3", "hopt", 64)
    codes, scales = mxq.mxq_quantize(W, p, torch.from_numpy(h_orc).to(DEV))
    torch.cuda.synchronize()
    tile_rows = synth.sample_rows(n // 64, 2, wl.seed).numpy()
    for tr in tile_rows:
        Wt = oracle_view(W[tr * 64:(tr + 1) * 64])
        r = orc.quantize(Wt, "e4m3", "hopt", 64, h=h_orc, n_threads=NT)
        gs = scales[tr].cpu().numpy()
        near = near_tie_mask(r.best, r.second)[0]
        bad = gs != r.scales[0]
        assert not (bad & ~near).any(), f"tile row {tr}: {(bad & ~near).sum()} tiles differ"
        gc = codes[tr * 64:(tr + 1) * 64].cpu().numpy()
        for tj in np.nonzero(~bad)[0]:
            assert np.array_equal(gc[:, tj * 64:(tj + 1) * 64], r.codes[:, tj * 64:(tj + 1) * 64])
        print(f"e4m3 tile row {tr}: {gs.size} tiles, {near.sum()} near ties, "
              f"{bad.sum()} differing (all near ties)")


def test_decoder_layer_back_to_back(mxq, orc, synth):
    wl = synth.WORKLOADS["decoder_layer"]
    hs = {}
    for xi, (R, k) in enumerate(wl.x_shapes):
        X = synth.workload_activations(wl, xi, device=DEV)
        h_gpu = mxq.mxq_act_sqmean(X)
        h_orc = orc.act_sqmean(oracle_view(X), n_threads=NT)
        np.testing.assert_allclose(h_gpu.cpu().numpy(), h_orc, rtol=1e-5)
        hs[k] = h_orc
        del X
        torch.cuda.empty_cache()
    p = mxq.params("nvfp4", "hopt", 16)
    outs = []
    Ws = [synth.workload_weight(wl, i, device=DEV) for i in range(len(wl.weights))]
    stream = torch.cuda.current_stream()
    for W in Ws:                                            # back to back on one stream
        outs.append(mxq.mxq_quantize(W, p, torch.from_numpy(hs[W.shape[1]]).to(DEV),
                                     stream=stream))
    torch.cuda.synchronize()
    for i, (W, (codes, scales)) in enumerate(zip(Ws, outs)):
        name, n, k = wl.weights[i]
        rows = synth.sample_rows(n, 4, wl.seed + i).numpy()
        r = orc.quantize(oracle_view(W[torch.as_tensor(rows, device=DEV)]), "nvfp4", "hopt", 16,
                         h=hs[k], n_threads=NT)
        ri = torch.as_tensor(rows, device=DEV)
        assert np.array_equal(scales[ri].cpu().numpy(), r.scales), name
        assert np.array_equal(codes[ri].cpu().numpy(), r.codes), name


@pytest.mark.parametrize("fmt,sfmt,block", [("nvfp4", "ue8m0", 32), ("int4", "e4m3", 16),
                                            ("nvfp4", "ue4m4", 16)])
def test_scale_grids_full_size(mxq, orc, synth, fmt, sfmt, block):
    """MXFP4, NVINT4 and E2M1-on-UE4M4 on the full-calibration weight (2560 x 9728), H-opt
    over the whole grid, with h from 32768 rows of the full-calibration activations."""
    wl = synth.WORKLOADS["nvfp4_full_calib"]
    W = synth.workload_weight(wl, 0, device=DEV)
    X = synth.workload_activations(wl, 0, device="cpu", rows=32768)
    h = orc.act_sqmean(oracle_view(X), n_threads=NT)
    rows = synth.sample_rows(W.shape[0], 24, wl.seed + 31).tolist()
    near, tot = sampled_parity(mxq, orc, W, fmt, block, "hopt", h, -1, rows,
                               f"{fmt}/{sfmt} bs{block}", sfmt=sfmt)
    print(f"{fmt}/{sfmt} bs{block}: {tot} sampled blocks bit-exact, {near} near ties")


def test_block_hessian_full_size(mxq, orc, synth):
    """Block-Hessian NVFP4 bs16 on the full-calibration weight with the oracle's Gram blocks
    of 16384 activation rows (uploaded): sampled rows bit-exact."""
    wl = synth.WORKLOADS["nvfp4_full_calib"]
    W = synth.workload_weight(wl, 0, device=DEV)
    X = synth.workload_activations(wl, 0, device="cpu", rows=16384)
    G = orc.block_gram(oracle_view(X), 16)
    p = mxq.params("nvfp4", "hopt", 16)
    codes, scales = mxq.mxq_quantize_gram(W, p, torch.from_numpy(G).to(DEV))
    torch.cuda.synchronize()
    rows = synth.sample_rows(W.shape[0], 8, wl.seed + 41).tolist()
    ri = torch.as_tensor(rows, device=DEV)
    r = orc.quantize_gram(oracle_view(W[ri]), "nvfp4", 16, G, n_threads=NT)
    assert np.array_equal(scales[ri].cpu().numpy(), r.scales)
    assert np.array_equal(codes[ri].cpu().numpy(), r.codes)


def test_gptq_ordered_full_size(mxq, orc, synth):
    """Ordered GPTQ with the NVFP4 bs16 H-optimal quantizer on the full-calibration weight
    (2560 x 9728), the Hessian of 8192 activation rows (the oracle's, uploaded): the block
    order equal to the oracle's except where two blocks' float64 losses agree to 1e-12
    relative (the two sides sum a block's loss in different orders), the factor of the full 9728 x 9728 Hessian within one float32 rounding of
    the oracle's, and sampled rows of the sweep bit-exact given the oracle's factor."""
    wl = synth.WORKLOADS["nvfp4_full_calib"]
    W = synth.workload_weight(wl, 0, device=DEV)
    n, k = W.shape
    X = oracle_view(synth.workload_activations(wl, 0, device="cpu", rows=8192))
    H = orc.gram(X)
    h = orc.act_sqmean(X, n_threads=NT)
    p = mxq.params("nvfp4", "hopt", 16)
    hd = torch.from_numpy(h).to(DEV)
    perm = mxq.mxq_gptq_order(W, hd, p)
    Wo = oracle_view(W)
    L = orc.block_losses(Wo, h, "nvfp4", "hopt", 16, n_threads=NT)
    perm_ref = orc.block_order(L)
    ties = order_with_ties(perm.cpu().numpy(), perm_ref, L)
    print(f"block order: {len(perm_ref)} blocks, {ties} adjacent near ties (< 1e-12 relative)")
    # the sweep below follows the GPU's order, which equals the oracle's up to near ties
    perm_ref = perm.cpu().numpy()
    cols = (perm_ref[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    U_ref = orc.gptq_prepare(np.ascontiguousarray(H[np.ix_(cols, cols)])[None])[0]
    U = mxq.mxq_gptq_factor(torch.from_numpy(H).to(DEV), 16, perm).cpu().numpy()
    ref = U_ref.astype(np.float64)
    tol = 2.0 ** -23 * np.abs(ref) + 2.0 ** -28 * np.abs(ref).max()
    err = np.abs(U.astype(np.float64) - ref)
    assert np.all(err <= tol), float((err / tol).max())
    del U, ref, err
    codes, scales = mxq.mxq_gptq(W, torch.from_numpy(U_ref).to(DEV), p, hd, perm)
    torch.cuda.synchronize()
    rows = synth.sample_rows(n, 8, wl.seed + 51).tolist()
    ri = torch.as_tensor(rows, device=DEV)
    r = orc.gptq_blocks(oracle_view(W[ri]), U_ref, h, "nvfp4", "hopt", 16, perm=perm_ref,
                        n_threads=NT)
    assert np.array_equal(scales[ri].cpu().numpy(), r.scales)
    assert np.array_equal(codes[ri].cpu().numpy(), r.codes)


def test_gptq_tiles_full_size(mxq, orc, synth):
    """FP8-GPTQ on the 64 x 64 tiles of the 4096 x 4096 weight: the oracle's Gram blocks of
    all 8192 activation rows, its factors and its tile scales (two sampled tile rows,
    uploaded); those tile rows of the GPU sweep bit-exact, the factors within one float32
    rounding."""
    wl = synth.WORKLOADS["e4m3_tiles"]
    W = synth.workload_weight(wl, 0, device=DEV)
    n, k = W.shape
    X = oracle_view(synth.workload_activations(wl, 0, device="cpu"))
    G = orc.block_gram(X, 64)
    U = orc.gptq_prepare(G)
    Ug = mxq.mxq_gptq_prepare(torch.from_numpy(G).to(DEV)).cpu().numpy()
    tol = 2.0 ** -23 * np.abs(U) + 2.0 ** -30 * np.abs(U).max(axis=(1, 2), keepdims=True)
    assert np.all(np.abs(Ug.astype(np.float64) - U) <= tol)
    h = orc.act_sqmean(X, n_threads=NT)
    scales = np.zeros((n // 64, k // 64), np.float32)
    tile_rows = synth.sample_rows(n // 64, 2, wl.seed + 61).numpy()
    for tr in tile_rows:
        r = orc.quantize(oracle_view(W[tr * 64:(tr + 1) * 64]), "e4m3", "hopt", 64, h=h,
                         n_threads=NT)
        scales[tr] = r.scales[0]
    codes = mxq.mxq_gptq_tiles(W, torch.from_numpy(U).to(DEV),
                               torch.from_numpy(scales).to(DEV)).cpu().numpy()
    for tr in tile_rows:
        ref = orc.gptq_tiles(oracle_view(W[tr * 64:(tr + 1) * 64]), U, scales[tr:tr + 1])
        assert np.array_equal(codes[tr * 64:(tr + 1) * 64], ref), f"tile row {tr}"


@pytest.mark.parametrize("wl_name,wi,fmt,block", [("nvfp4_full_calib", 0, "nvfp4", 16),
                                                  ("decoder_layer", 4, "nvfp4", 16),
                                                  ("int8_e4m3scale", 0, "int8", 32)])
def test_error_sums_full_size(mxq, orc, synth, wl_name, wi, fmt, block):
    """Error sums (sum d^2, sum w^2, sum h d^2, sum h w^2) and the two relative errors of a
    whole weight at its full shape -- the launch configuration the benchmark times (the
    headline 2560 x 9728 weight, the decoder layer's 14336 x 4096 gate projection, the INT8
    workload's weight) -- against the oracle's float64 sums of the same codes, 1e-5
    relative. h from 8192 rows of the workload's activations, and the codes and scales, are
    the oracle's (uploaded), so both sides measure the same quantization."""
    wl = synth.WORKLOADS[wl_name]
    W = synth.workload_weight(wl, wi, device=DEV)
    n, k = W.shape
    X = synth.workload_activations(wl, synth.x_index_for_weight(wl, wi), device="cpu",
                                   rows=8192)
    h = orc.act_sqmean(oracle_view(X), n_threads=NT)
    del X
    hd = torch.from_numpy(h).to(DEV)
    p = mxq.params(fmt, "hopt", block, window=wl.window)
    Wo = oracle_view(W)
    r = orc.quantize(Wo, fmt, "hopt", block, h=h, window=wl.window, n_threads=NT)
    codes, scales = torch.from_numpy(r.codes).to(DEV), torch.from_numpy(r.scales).to(DEV)
    sums = mxq.mxq_error(W, codes, scales, p, hd).cpu().numpy()
    sums0 = mxq.mxq_error(W, codes, scales, p, None).cpu().numpy()
    What = orc.dequant(r.codes, r.scales, fmt, block, n, k)
    ref = orc.error_sums(Wo, What, h)
    np.testing.assert_allclose(sums, ref, rtol=1e-5)
    np.testing.assert_allclose(sums0[:2], ref[:2], rtol=1e-5)
    assert sums0[2] == 0 and sums0[3] == 0
    if fmt == "nvfp4":
        # the fused call (error sums added inside the search) on the whole weight: every
        # block's codes and scale equal the oracle's, and the sums agree
        cf, sf, sumsf = mxq.mxq_quantize_err(W, p, hd)
        torch.cuda.synchronize()
        assert np.array_equal(sf.cpu().numpy(), r.scales)
        assert np.array_equal(cf.cpu().numpy(), r.codes)
        np.testing.assert_allclose(sumsf.cpu().numpy(), ref, rtol=1e-5)
    m, mo = mxq.mxq_metrics_from_sums(sums), orc.metrics(ref)
    assert m["weight_rel"] == pytest.approx(mo["weight_rel"], rel=1e-5)
    assert m["h_rel"] == pytest.approx(mo["h_rel"], rel=1e-5)
    print(f"{wl_name}[{wi}] {fmt} bs{block}: weight error {m['weight_rel']:.4%}, "
          f"h-weighted {m['h_rel']:.4%} (oracle {mo['weight_rel']:.4%}, {mo['h_rel']:.4%})")


def test_gram_full_size_sampled(mxq, orc, synth):
    """The GPTQ Hessian H = X^T X / R of the full-calibration activations (244449 x 9728, the
    launch the GPTQ benchmark times: 380 tiles of 256 x 512 over 74 pairs of SMs, five whole
    waves and ten tiles cut into row chunks), checked entry by entry against the oracle's
    float64 sums on sampled entries: every diagonal entry of a sampled set, random pairs,
    and pairs at the tile edges (rows 255 / 256, columns 511 / 512, the last column)."""
    wl = synth.WORKLOADS["nvfp4_full_calib"]
    X = synth.workload_activations(wl, 0, device=DEV)
    R, K = X.shape
    H = mxq.mxq_act_gram(X)
    torch.cuda.synchronize()
    Xh = oracle_view(X)
    del X
    torch.cuda.empty_cache()
    rng = np.random.default_rng(7)
    edges = [0, 255, 256, 511, 512, 4607, 4608, 9215, 9216, K - 1]
    pairs = np.concatenate([
        np.stack([d := rng.choice(K, 256, replace=False), d], axis=1),
        rng.integers(0, K, (768, 2)),
        np.array([(i, j) for i in edges for j in edges])])
    got = H[torch.as_tensor(pairs[:, 0], device=DEV),
            torch.as_tensor(pairs[:, 1], device=DEV)].cpu().numpy().astype(np.float64)
    sym = H[torch.as_tensor(pairs[:, 1], device=DEV),
            torch.as_tensor(pairs[:, 0], device=DEV)].cpu().numpy().astype(np.float64)
    assert np.array_equal(got, sym)
    ref = orc.gram_entries(Xh, pairs)
    absref = np.zeros(len(pairs))                # (|X|^T |X|)_ij for the bound
    for r0 in range(0, R, 16384):
        c = np.abs(orc.to_float(Xh[r0:r0 + 16384])).astype(np.float64)
        absref += (c[:, pairs[:, 0]] * c[:, pairs[:, 1]]).sum(axis=0)
    tol = (R + 2) * 2.0 ** -24 * absref / R + 1e-38
    err = np.abs(got - ref)
    assert np.all(err <= tol), float((err / tol).max())
    print(f"Gram 244449 x 9728: {len(pairs)} sampled entries within the float32 bound; "
          f"largest error / bound {float((err / tol).max()):.3g}")
