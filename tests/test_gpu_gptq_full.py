"""GPU GPTQ with the block quantizer as its inner step (qwantize "Results", "GPTQ
Quantization"; sequential and ordered) against the oracle, stage by stage.

Bars:
- the sweep (mxq_gptq) is bit-exact: given the oracle's factor U (and block order), every
  scale and code equals the oracle's -- both evaluate the definition's float32 steps in its
  order, and every scale search scores its candidates exactly;
- the block order (mxq_gptq_order) equals the oracle's except where two blocks' losses
  agree to 1e-12 relative: the losses are float64 sums of the same float32 terms in
  different orders, so only such blocks can swap;
- the factor (mxq_gptq_factor): float64 on both sides by different stable routes, rounded
  to float32 once: |dU| <= 2^-23 |U| + 2^-28 max|U| (the float64 difference is a small
  multiple of cond(H) 2^-53 of the largest entry, cond(H) <= 1 + 100 k with the damping);
- the Gram matrix (mxq_act_gram: tensor-core tiles over the upper triangle, accumulating
  bf16 products in float32 over the rows in order -- the last wave's tiles in row chunks
  added in double --, times 1/R, then mirrored):
  |dH| <= (R + 2) 2^-24 (|X|^T |X|)_ij / R, H exactly symmetric and the same on every run;
- end to end (Gram, order, factor and sweep on the GPU against the oracle's pipeline on the
  same X and W): the Gram matrices differ within that bound, which moves U, so codes are
  compared by what is unique: the output error within 1% and below the plain quantizer's.
"""
import numpy as np
import pytest
import torch

from gpu_util import oracle_view, order_with_ties, output_error_np

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


def correlated_x(synth, rows, k, seed, device):
    X = synth.activations(rows, k, seed, dtype=torch.float32, device=device)
    X[:, 1::2] += 0.8 * X[:, 0::2]
    return X.to(torch.bfloat16)


# Tiles of H are 256 x 512 per pair of SMs, 74 pairs on a B200: k <= 4096 gives fewer tiles
# than pairs (every tile cut into row chunks, added in a fixed order); k = 6144 gives 156
# tiles (two whole waves, then 8 tiles in chunks); 208 and 777 rows leave ragged edges in
# both dimensions
@pytest.mark.parametrize("rows,k", [(3000, 256), (777, 208), (20000, 512), (3000, 2048),
                                    (600, 4096), (1000, 6144), (65, 8)])
def test_gram_matches_oracle(mxq, orc, synth, rows, k):
    X = correlated_x(synth, rows, k, 121, DEV)
    H = mxq.mxq_act_gram(X).cpu().numpy()
    assert np.array_equal(H, H.T)
    assert np.array_equal(H, mxq.mxq_act_gram(X).cpu().numpy())       # deterministic
    Xo = oracle_view(X)
    ref = orc.gram(Xo).astype(np.float64)
    A = np.abs(orc.to_float(Xo).astype(np.float64))
    tol = (rows + 2) * 2.0 ** -24 * (A.T @ A) / rows + 1e-38
    assert np.all(np.abs(H - ref) <= tol), float((np.abs(H - ref) / tol).max())


def check_factor(U, ref):
    assert np.all(np.isfinite(U)) and np.all(np.tril(U, -1) == 0)
    ref = ref.astype(np.float64)
    tol = 2.0 ** -23 * np.abs(ref) + 2.0 ** -28 * np.abs(ref).max()
    err = np.abs(U.astype(np.float64) - ref)
    assert np.all(err <= tol), float((err / tol).max())


def block_cols(perm, B):
    return (np.asarray(perm)[:, None] * B + np.arange(B)[None, :]).reshape(-1)


def test_gram_odd_width(mxq, orc, synth):
    """102 columns of a 104-wide matrix: rows of H are not 16-byte multiples, and the last
    column group of every TMA box lies partly beyond the matrix (zero fill)."""
    rows = 1234
    X = correlated_x(synth, rows, 104, 125, DEV)[:, :102]
    H = mxq.mxq_act_gram(X).cpu().numpy()
    assert H.shape == (102, 102) and np.array_equal(H, H.T)
    Xo = oracle_view(X)
    ref = orc.gram(Xo).astype(np.float64)
    A = np.abs(orc.to_float(Xo).astype(np.float64))
    tol = (rows + 2) * 2.0 ** -24 * (A.T @ A) / rows + 1e-38
    assert np.all(np.abs(H - ref) <= tol), float((np.abs(H - ref) / tol).max())


def test_gram_strided_columns(mxq, orc, synth):
    """X a column slice of a wider matrix (ld 2304, 2048 columns starting at column 128): the
    tiles' operand offsets are columns of the slice."""
    rows = 1500
    big = correlated_x(synth, rows, 2304, 123, DEV)
    X = big[:, 128:2176]
    H = mxq.mxq_act_gram(X).cpu().numpy()
    assert np.array_equal(H, H.T)
    Xo = oracle_view(X)
    ref = orc.gram(Xo).astype(np.float64)
    A = np.abs(orc.to_float(Xo).astype(np.float64))
    tol = (rows + 2) * 2.0 ** -24 * (A.T @ A) / rows + 1e-38
    assert np.all(np.abs(H - ref) <= tol), float((np.abs(H - ref) / tol).max())


@pytest.mark.parametrize("k,B,ordered", [(64, 16, False), (256, 16, True), (1024, 32, True),
                                         (208, 16, False), (1008, 16, True), (1088, 16, False),
                                         (1280, 32, True)])
def test_factor_matches_oracle(mxq, orc, synth, k, B, ordered):
    X = correlated_x(synth, 4 * k, k, 122, "cpu")
    H = orc.gram(oracle_view(X))
    perm = np.random.default_rng(k).permutation(k // B).astype(np.int32) if ordered else None
    Hp = H if perm is None else H[np.ix_(block_cols(perm, B), block_cols(perm, B))]
    ref = orc.gptq_prepare(np.ascontiguousarray(Hp)[None])[0]
    pd = None if perm is None else torch.from_numpy(perm).to(DEV)
    U = mxq.mxq_gptq_factor(torch.from_numpy(H).to(DEV), B, pd).cpu().numpy()
    check_factor(U, ref)


def test_factor_and_sweep_enqueued_ahead(mxq, orc, synth):
    """Several factor + sweep calls enqueued back to back with no synchronisation (the host
    runs far ahead of the GPU, and the library's ring of events wraps around more than
    once): every call's outputs equal those of a call made alone."""
    n, k, B = 40, 1024, 16
    W, h, U0, _ = sweep_case(orc, synth, n, k, B, 141, torch.bfloat16, False)
    X = correlated_x(synth, 4 * k, k, 142, "cpu")
    H = torch.from_numpy(orc.gram(oracle_view(X))).to(DEV)
    hd = torch.from_numpy(h).to(DEV)
    p = mxq.params("nvfp4", "hopt", B)
    U_ref = mxq.mxq_gptq_factor(H, B)
    c_ref, s_ref = mxq.mxq_gptq(W, U_ref, p, hd)
    torch.cuda.synchronize()
    outs = []
    for _ in range(6):
        U = mxq.mxq_gptq_factor(H, B)
        outs.append((U,) + tuple(mxq.mxq_gptq(W, U, p, hd)))
    torch.cuda.synchronize()
    for U, c, s in outs:
        assert torch.equal(U, U_ref)
        assert torch.equal(c, c_ref) and torch.equal(s, s_ref)


def test_factor_degenerate(mxq, orc):
    """An all-zero H (lambda = 1: U = I), a dead channel and a rank-one H."""
    k = 128
    Z = np.zeros((k, k), np.float32)
    U = mxq.mxq_gptq_factor(torch.from_numpy(Z).to(DEV), 16).cpu().numpy()
    assert np.array_equal(U, np.eye(k, dtype=np.float32))
    rng = np.random.default_rng(5)
    A = rng.standard_normal((300, k)).astype(np.float32)
    H = (A.T @ A / 300).astype(np.float32)
    H[9, :] = 0.0
    H[:, 9] = 0.0
    for Hx in (H, np.outer(A[0], A[0]).astype(np.float32)):
        U = mxq.mxq_gptq_factor(torch.from_numpy(Hx).to(DEV), 16, damp=0.05).cpu().numpy()
        check_factor(U, orc.gptq_prepare(Hx[None], 0.05)[0])


def sweep_case(orc, synth, n, k, B, seed, dtype, ordered):
    W = synth.student_t_weight(n, k, seed, dtype=dtype, device=DEV)
    X = correlated_x(synth, 3 * k, k, seed + 1, "cpu")
    Xo = oracle_view(X)
    H = orc.gram(Xo)
    h = orc.act_sqmean(Xo)
    perm = np.random.default_rng(seed).permutation(k // B).astype(np.int32) if ordered else None
    cols = block_cols(perm, B) if ordered else np.arange(k)
    U = orc.gptq_prepare(np.ascontiguousarray(H[np.ix_(cols, cols)])[None])[0]
    return W, h, U, perm


COMBOS = [("nvfp4", "e4m3", 16), ("nvfp4", "e4m3", 32), ("nvfp4", "ue8m0", 32),
          ("int4", "e4m3", 16), ("nvfp4", "ue4m4", 16)]


@pytest.mark.parametrize("fmt,sfmt,B", COMBOS)
@pytest.mark.parametrize("mode", ["naive", "sse", "hopt"])
@pytest.mark.parametrize("ordered", [False, True])
def test_sweep_bit_exact(mxq, orc, synth, fmt, sfmt, B, mode, ordered):
    n, k = 37, 224                       # ragged rows; three full panels and a partial one
    W, h, U, perm = sweep_case(orc, synth, n, k, B, 131, torch.bfloat16, ordered)
    p = mxq.params(fmt, mode, B, scale_fmt=sfmt)
    pd = None if perm is None else torch.from_numpy(perm).to(DEV)
    codes, scales = mxq.mxq_gptq(W, torch.from_numpy(U).to(DEV), p, torch.from_numpy(h).to(DEV),
                                 pd)
    torch.cuda.synchronize()
    r = orc.gptq_blocks(oracle_view(W), U, h, fmt, mode, B, sfmt=sfmt, perm=perm)
    sc = scales.cpu().numpy()
    bad = np.argwhere(sc != r.scales)
    assert bad.size == 0, f"{len(bad)} scales differ, first at {bad[:3].tolist()}"
    assert np.array_equal(codes.cpu().numpy(), r.codes)


@pytest.mark.parametrize("n,k,B,dtype", [(64, 1024, 16, torch.float32), (130, 512, 32, torch.bfloat16),
                                         (300, 256, 16, torch.bfloat16)])
def test_sweep_bit_exact_larger(mxq, orc, synth, n, k, B, dtype):
    W, h, U, perm = sweep_case(orc, synth, n, k, B, 132, dtype, True)
    p = mxq.params("nvfp4", "hopt", B)
    codes, scales = mxq.mxq_gptq(W, torch.from_numpy(U).to(DEV), p, torch.from_numpy(h).to(DEV),
                                 torch.from_numpy(perm).to(DEV))
    torch.cuda.synchronize()
    r = orc.gptq_blocks(oracle_view(W), U, h, "nvfp4", "hopt", B, perm=perm, n_threads=8)
    assert np.array_equal(scales.cpu().numpy(), r.scales)
    assert np.array_equal(codes.cpu().numpy(), r.codes)


@pytest.mark.parametrize("n,k,B,mode", [(1, 16, 16, "hopt"), (2, 32, 32, "sse"), (3, 48, 16, "hopt"),
                                        (5, 96, 32, "hopt"), (6, 16, 16, "naive")])
def test_sweep_small_shapes(mxq, orc, synth, n, k, B, mode):
    """Rows that leave half-warps and whole warps of the panel kernel without a row (the
    kernel takes one half-warp per row, four rows per CTA), and inputs narrower than one
    panel of 64 positions (a single partial panel, no trailing update)."""
    W, h, U, perm = sweep_case(orc, synth, n, k, B, 133 + n, torch.bfloat16, False)
    p = mxq.params("nvfp4", mode, B)
    codes, scales = mxq.mxq_gptq(W, torch.from_numpy(U).to(DEV), p, torch.from_numpy(h).to(DEV))
    torch.cuda.synchronize()
    r = orc.gptq_blocks(oracle_view(W), U, h, "nvfp4", mode, B)
    assert np.array_equal(scales.cpu().numpy(), r.scales)
    assert np.array_equal(codes.cpu().numpy(), r.codes)


def test_sweep_worked_examples(mxq):
    """The oracle's hand-derived cases: the residual changes the next block's scale
    (0x33, not 0x35) and an in-block code; one product per block past the block."""
    k = 32
    W = np.zeros((1, k), np.float32)
    W[0, [0, 1, 2, 16]] = [1.25, 5.0625, 6.0, 5.0]
    U = np.eye(k, dtype=np.float32)
    U[0, 1], U[0, 16] = 0.5, 4.0
    p = mxq.params("nvfp4", "naive", 16)
    c, s = mxq.mxq_gptq(torch.from_numpy(W).to(DEV), torch.from_numpy(U).to(DEV), p)
    assert s.cpu().numpy()[0].tolist() == [0x38, 0x33]
    c = c.cpu().numpy()[0]
    assert c[0] == 0x62 and c[1] == 0x07 and c[8] == 0x07
    W = np.zeros((1, k), np.float32)
    W[0, [0, 1, 2, 16, 17]] = [1.25, 1.25, 6.0, 1.75, 3.0]
    U = np.eye(k, dtype=np.float32)
    U[0, 16] = U[1, 16] = 2.0 ** -22
    c, s = mxq.mxq_gptq(torch.from_numpy(W).to(DEV), torch.from_numpy(U).to(DEV), p)
    assert s.cpu().numpy()[0].tolist() == [0x38, 0x30] and c.cpu().numpy()[0, 8] == 0x75


@pytest.mark.parametrize("fmt,sfmt,B,mode", [("nvfp4", "e4m3", 16, "hopt"),
                                             ("nvfp4", "ue8m0", 32, "sse"),
                                             ("int4", "e4m3", 16, "naive")])
def test_order_matches_oracle(mxq, orc, synth, fmt, sfmt, B, mode):
    n, k = 200, 1024
    W = synth.student_t_weight(n, k, 141, dtype=torch.bfloat16, device=DEV)
    X = synth.activations(500, k, 142, dtype=torch.bfloat16, device="cpu")
    h = orc.act_sqmean(oracle_view(X))
    p = mxq.params(fmt, mode, B, scale_fmt=sfmt)
    perm = mxq.mxq_gptq_order(W, torch.from_numpy(h).to(DEV), p).cpu().numpy()
    L = orc.block_losses(oracle_view(W), h, fmt, mode, B, sfmt=sfmt)
    ref = orc.block_order(L)
    order_with_ties(perm, ref, L)


def test_end_to_end_against_oracle_pipeline(mxq, orc, synth):
    n, k, rows, B = 128, 512, 4096, 16
    W = synth.student_t_weight(n, k, 151, dtype=torch.bfloat16, device=DEV)
    X = correlated_x(synth, rows, k, 152, DEV)
    p = mxq.params("nvfp4", "hopt", B)
    h = mxq.mxq_act_sqmean(X)
    H = mxq.mxq_act_gram(X)
    perm = mxq.mxq_gptq_order(W, h, p)
    U = mxq.mxq_gptq_factor(H, B, perm)
    codes, scales = mxq.mxq_gptq(W, U, p, h, perm)
    torch.cuda.synchronize()
    Xo, Wo = oracle_view(X), oracle_view(W)
    Ho = orc.gram(Xo)
    ho = orc.act_sqmean(Xo)
    r = orc.gptq(Wo, Ho, ho, "nvfp4", "hopt", B, ordered=True)
    plain = orc.quantize(Wo, "nvfp4", "hopt", B, h=ho)
    idx = np.sort(np.random.default_rng(0).choice(rows, 512, replace=False))
    Xs = Xo[idx]

    def out_err(c, s):
        return orc.output_error(Xs, Wo, orc.dequant(c, s, "nvfp4", B, n, k))
    # the GPU result measured with its own dequant and plain numpy (no GPU output enters the
    # oracle)
    What_gpu = mxq.mxq_dequant(codes, scales, p, n, k).cpu().numpy()
    e_gpu = output_error_np(orc.to_float(Xs), orc.to_float(Wo), What_gpu)
    e_ref = out_err(r.codes, r.scales)
    assert e_gpu == pytest.approx(e_ref, rel=1e-2)
    assert e_gpu < 0.95 * out_err(plain.codes, plain.scales)


def test_rejections(mxq):
    W = torch.zeros(16, 64, dtype=torch.bfloat16, device=DEV)
    U = torch.eye(64, device=DEV)
    with pytest.raises(mxq.MxqError):
        mxq.mxq_gptq(W, U, mxq.params("int8", "hopt", 32), torch.ones(64, device=DEV))
    with pytest.raises(mxq.MxqError):
        mxq.mxq_gptq(W, U, mxq.params("nvfp4", "hopt", 16))          # H-optimal needs h
    with pytest.raises(mxq.MxqError):
        mxq.mxq_gptq_factor(torch.zeros(64, 64, device=DEV), 64)
    with pytest.raises(mxq.MxqError):
        mxq.mxq_gptq_factor(torch.zeros(64, 64, device=DEV), 16, damp=float("inf"))
    with pytest.raises(mxq.MxqError):
        mxq.mxq_act_gram(torch.zeros(8, 64, device=DEV))              # float32 X


@pytest.mark.parametrize("fmt,sfmt,B,mode", [("nvfp4", "e4m3", 16, "hopt"), ("nvfp4", "ue8m0", 32, "sse"),
                                             ("int4", "e4m3", 16, "naive"),
                                             ("nvfp4", "ue5m3", 16, "hopt")])
def test_sweep_special_values(mxq, orc, fmt, sfmt, B, mode):
    """All-zero and negative-zero blocks (every candidate ties at zero error), saturating and
    subnormal-scale blocks, a dead input channel (h = 0), and a factor with negative and
    zero couplings -- bit-exact with the oracle on the same factor."""
    rng = np.random.default_rng(17)
    n, k = 12, 128
    W = (rng.standard_t(4, (n, k)) * 0.05).astype(np.float32)
    W[0, :] = 0.0
    W[1, :] = -0.0
    W[2, :B] = 1e30                                    # far above every scale's range
    W[3, :] *= 1e-30                                   # scales in the subnormal corner
    W[4, ::7] = 0.0
    W[5, B:2 * B] = -W[5, :B]
    h = np.exp(rng.normal(0, 1, k)).astype(np.float32)
    h[5] = 0.0
    A = rng.standard_normal((300, k)).astype(np.float32)
    A[:, 1::2] -= 0.7 * A[:, 0::2]
    H = (A.T @ A / 300).astype(np.float32)
    U = orc.gptq_prepare(H[None])[0]
    U[0, 1:5] = 0.0
    p = mxq.params(fmt, mode, B, scale_fmt=sfmt)
    Wt = torch.from_numpy(W).to(DEV)
    codes, scales = mxq.mxq_gptq(Wt, torch.from_numpy(U).to(DEV), p, torch.from_numpy(h).to(DEV))
    torch.cuda.synchronize()
    r = orc.gptq_blocks(W, U, h, fmt, mode, B, sfmt=sfmt)
    assert np.array_equal(scales.cpu().numpy(), r.scales)
    assert np.array_equal(codes.cpu().numpy(), r.codes)
