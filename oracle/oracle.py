"""ctypes + numpy front end of the CPU oracle.

TEST INFRASTRUCTURE ONLY: a plain, slow, obviously correct restatement of block-scaled
weight quantization with a searched E4M3 block scale (see ``oracle.c`` for the sources and
readings). Only the tests, the smoke check and the benchmark's CPU-baseline leg import it;
the CUDA library never does, and the two share no code.

The output error, ``||X_s W^T - X_s Wq^T||_F / ||X_s W^T||_F`` on sampled rows of X
(qwantize "Results", metric definitions), is computed here with numpy float64 matrix
products.
"""
from __future__ import annotations

import ctypes
import os
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# MXQ_ORACLE_LIB lets a test load a deliberately broken build (planted-mistake checks).
_LIB_PATH = os.environ.get("MXQ_ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

F32, BF16 = 0, 1
NVFP4, INT8, E4M3, INT4 = 0, 1, 2, 3
NAIVE, SSE, HOPT = 0, 1, 2
FMTS = {"nvfp4": NVFP4, "int8": INT8, "e4m3": E4M3, "int4": INT4}
# block-scale grids (sfmt): "mxfp4" is E2M1 elements ("nvfp4") on the "ue8m0" grid
SFMTS = {"e4m3": 0, "ue4m4": 1, "ue5m3": 2, "ue8m0": 3}
MODES = {"naive": NAIVE, "sse": SSE, "hopt": HOPT}

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_D = ctypes.c_double


def lib():
    """Load (building on first use if needed) the compiled oracle."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.environ.get("MXQ_ORACLE_LIB") and (not os.path.exists(_LIB_PATH) or (
                    os.path.getmtime(_LIB_PATH) < os.path.getmtime(os.path.join(_HERE, "oracle.c")))):
                from oracle.build_oracle import build
                build()
            L = ctypes.CDLL(_LIB_PATH)
            L.orc_e4m3_value.restype = _D
            L.orc_e4m3_value.argtypes = [_I]
            L.orc_e2m1_value.restype = _D
            L.orc_e2m1_value.argtypes = [_I]
            for f in ("orc_ue4m4_value", "orc_ue5m3_value", "orc_ue8m0_value"):
                getattr(L, f).restype = _D
                getattr(L, f).argtypes = [_I]
            L.orc_scale_table.restype = _I
            L.orc_scale_table.argtypes = [_I, _P]
            L.orc_e4m3_table.argtypes = [_P]
            L.orc_e2m1_table.argtypes = [_P]
            for f in ("orc_e4m3_rne_code", "orc_e2m1_rne_code", "orc_int127_rne"):
                getattr(L, f).restype = _I
                getattr(L, f).argtypes = [ctypes.c_float]
            L.orc_project.restype = _I
            L.orc_project.argtypes = [_I, _I, _I, ctypes.c_float, ctypes.POINTER(ctypes.c_float)]
            L.orc_project_e4m3.restype = _I
            L.orc_project_e4m3.argtypes = [ctypes.c_float, ctypes.c_float,
                                           ctypes.POINTER(ctypes.c_float)]
            L.orc_project_many.argtypes = [_I, _I, _I, _P, _I64, _P, _P]
            L.orc_project_e4m3_many.argtypes = [ctypes.c_float, _P, _I64, _P, _P]
            L.orc_naive_code.restype = _I
            L.orc_naive_code.argtypes = [_I, _I, ctypes.c_float]
            L.orc_act_sqsum.argtypes = [_P, _I, _I64, _I64, _I64, _I64, _I64, _P]
            L.orc_act_sqmean.argtypes = [_P, _I, _I64, _I64, _I64, _P]
            L.orc_quantize_blocks.restype = _I
            L.orc_quantize_blocks.argtypes = [_P, _I, _I64, _I64, _I64, _P, _I, _I, _I, _I, _I,
                                              _I64, _I64, _P, _P, _P, _P, _P]
            L.orc_block_gram.restype = _I
            L.orc_block_gram.argtypes = [_P, _I, _I64, _I64, _I64, _I, _P]
            L.orc_quantize_blocks_gram.restype = _I
            L.orc_quantize_blocks_gram.argtypes = [_P, _I, _I64, _I64, _I64, _P, _I, _I, _I, _I,
                                                   _I64, _I64, _P, _P, _P, _P, _P]
            L.orc_swizzle_scales.argtypes = [_P, _I64, _I64, _P]
            L.orc_gptq_blocks.restype = _I
            L.orc_gptq_blocks.argtypes = [_P, _I, _I64, _I64, _I64, _P, _I, _I, _I, _I, _I, _P,
                                          _P, _I64, _I64, _P, _P]
            L.orc_gptq_tiles.restype = _I
            L.orc_gptq_tiles.argtypes = [_P, _I, _I64, _I64, _I64, _P, _P, _P, _P]
            L.orc_log_grid.argtypes = [_I, _D, _D, _P]
            L.orc_quantize_tiles.restype = _I
            L.orc_quantize_tiles.argtypes = [_P, _I, _I64, _I64, _I64, _P, _I, _I, _I, _D, _D,
                                             _I64, _I64, _P, _P, _P, _P, _P]
            L.orc_dequant.restype = _I
            L.orc_dequant.argtypes = [_P, _P, _I, _I, _I, _I64, _I64, _P]
            L.orc_error_sums.argtypes = [_P, _I, _I64, _I64, _I64, _P, _P, _P]
            _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _as_input(W):
    """(array, dtype code): float32 stays float32; bf16 is held as its uint16 bits."""
    W = np.ascontiguousarray(W)
    if W.dtype == np.float32:
        return W, F32
    if W.dtype == np.uint16:
        return W, BF16
    raise TypeError("oracle inputs are float32 arrays or bf16 bit patterns (uint16)")


def _threads(n_threads):
    return max(1, int(n_threads or 1))


# --------------------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------------------

def e4m3_table() -> np.ndarray:
    t = np.zeros(127, np.float32)
    lib().orc_e4m3_table(_ptr(t))
    return t


def e2m1_table() -> np.ndarray:
    t = np.zeros(8, np.float32)
    lib().orc_e2m1_table(_ptr(t))
    return t


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(int(code))


def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def scale_value(sfmt: str, code: int) -> float:
    """Value of a scale code, decoded from its bit fields (E4M3, UE4M4, UE5M3, UE8M0)."""
    if sfmt == "e4m3":
        return e4m3_value(code)
    return getattr(lib(), f"orc_{sfmt}_value")(int(code))


def scale_table(sfmt: str) -> np.ndarray:
    """The sorted table of a scale grid, indexed by code."""
    t = np.zeros(256, np.float32)
    n = lib().orc_scale_table(SFMTS[sfmt], _ptr(t))
    return t[:n].copy()


def naive_code(fmt: str, amax: float, sfmt: str = "e4m3") -> int:
    return lib().orc_naive_code(FMTS[fmt], SFMTS[sfmt], float(amax))


def project(fmt: str, code: int, w: float, sfmt: str = "e4m3"):
    """(magnitude code, |w^|) of one element at scale code ``code`` (NVFP4 / INT4 / INT8)."""
    out = ctypes.c_float()
    q = lib().orc_project(FMTS[fmt], SFMTS[sfmt], int(code), float(w), ctypes.byref(out))
    return q, out.value


def project_e4m3(w: float, s: float):
    out = ctypes.c_float()
    q = lib().orc_project_e4m3(float(w), float(s), ctypes.byref(out))
    return q, out.value


def project_many(fmt: str, code: int, w, sfmt: str = "e4m3"):
    """Vector form of :func:`project`: (codes uint8, |w^| float32) for float32 ``w``."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    q = np.zeros(w.shape, np.uint8)
    wq = np.zeros(w.shape, np.float32)
    lib().orc_project_many(FMTS[fmt], SFMTS[sfmt], int(code), _ptr(w), w.size, _ptr(q),
                           _ptr(wq))
    return q, wq


def project_e4m3_many(s: float, w):
    w = np.ascontiguousarray(w, dtype=np.float32)
    q = np.zeros(w.shape, np.uint8)
    wq = np.zeros(w.shape, np.float32)
    lib().orc_project_e4m3_many(float(s), _ptr(w), w.size, _ptr(q), _ptr(wq))
    return q, wq


def log_grid(points: int = 64, lo: float = -2.0, hi: float = 2.0) -> np.ndarray:
    g = np.zeros(points, np.float32)
    lib().orc_log_grid(points, lo, hi, _ptr(g))
    return g


# --------------------------------------------------------------------------------------
# h = E[x^2]
# --------------------------------------------------------------------------------------

def act_sqsum(X, row0=0, row1=None) -> np.ndarray:
    """Column sums of squares (float64) over rows [row0, row1)."""
    X, dt = _as_input(X)
    R, K = X.shape
    row1 = R if row1 is None else row1
    out = np.zeros(K, np.float64)
    lib().orc_act_sqsum(_ptr(X), dt, R, K, K, row0, row1, _ptr(out))
    return out


def act_sqmean(X, n_threads=1) -> np.ndarray:
    """h_j = fl32(sum_r x_rj^2 / R) (float32 [K]); row ranges summed on threads, then
    combined in double in ascending row-range order when n_threads > 1."""
    X, dt = _as_input(X)
    R, K = X.shape
    nt = _threads(n_threads)
    if nt == 1:
        h = np.zeros(K, np.float32)
        lib().orc_act_sqmean(_ptr(X), dt, R, K, K, _ptr(h))
        return h
    bounds = np.linspace(0, R, nt + 1).astype(np.int64)
    with ThreadPoolExecutor(nt) as ex:
        parts = list(ex.map(lambda i: act_sqsum(X, int(bounds[i]), int(bounds[i + 1])),
                            range(nt)))
    tot = np.zeros(K, np.float64)
    for p in parts:
        tot += p
    return (tot / R).astype(np.float32) if R else np.zeros(K, np.float32)


# --------------------------------------------------------------------------------------
# quantization
# --------------------------------------------------------------------------------------

class Result(dict):
    """codes, scales, best, second (candidate errors), naive (naive code / grid index)."""
    __getattr__ = dict.__getitem__


def quantize(W, fmt: str, mode: str, block: int, *, h=None, window: int = -1,
             rows=None, n_threads=1, points=64, lo=-2.0, hi=2.0, sfmt: str = "e4m3") -> Result:
    """Quantize W [n, k] (float32 or bf16 bits). ``rows``: optional (row0, row1) --
    only those rows (tile rows for E4M3) are computed; other outputs stay zero/NaN.
    ``sfmt``: the block-scale grid of NVFP4 / INT4 elements."""
    W, dt = _as_input(W)
    n, k = W.shape
    f, m = FMTS[fmt], MODES[mode]
    hp = None
    if h is not None:
        h = np.ascontiguousarray(h, dtype=np.float32)
        hp = h
    if m == HOPT and h is None:
        raise ValueError("H-optimal needs h")
    nt = _threads(n_threads)
    if f == E4M3:
        T = block
        tn, tk = n // T, k // T
        codes = np.zeros((n, k), np.uint8)
        scales = np.zeros((tn, tk), np.float32)
        best = np.full((tn, tk), np.nan)
        second = np.full((tn, tk), np.nan)
        gidx = np.full((tn, tk), -2, np.int32)
        r0, r1 = (0, tn) if rows is None else rows

        def run(a, b):
            rc = lib().orc_quantize_tiles(_ptr(W), dt, n, k, k, _ptr(hp), m, T, points, lo, hi,
                                          a, b, _ptr(codes), _ptr(scales), _ptr(best),
                                          _ptr(second), _ptr(gidx))
            if rc != 0:
                raise ValueError("oracle rejected the arguments")
        _run_ranges(run, r0, r1, nt)
        return Result(codes=codes, scales=scales, best=best, second=second, naive=gidx)
    kb = k // block
    codes = np.zeros((n, k // 2) if f in (NVFP4, INT4) else (n, k), np.uint8)
    scales = np.zeros((n, kb), np.uint8)
    best = np.full((n, kb), np.nan)
    second = np.full((n, kb), np.nan)
    naive = np.full((n, kb), -1, np.int32)
    r0, r1 = (0, n) if rows is None else rows

    def run(a, b):
        rc = lib().orc_quantize_blocks(_ptr(W), dt, n, k, k, _ptr(hp), f, SFMTS[sfmt], m, block,
                                       window, a, b, _ptr(codes), _ptr(scales), _ptr(best),
                                       _ptr(second), _ptr(naive))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
    _run_ranges(run, r0, r1, nt)
    return Result(codes=codes, scales=scales, best=best, second=second, naive=naive)


def block_gram(X, B: int) -> np.ndarray:
    """G[b] = fl32(X_b^T X_b / R) for every column block b: float32 [cols/B, B, B]."""
    X, dt = _as_input(X)
    R, K = X.shape
    G = np.zeros((K // B, B, B), np.float32)
    if lib().orc_block_gram(_ptr(X), dt, R, K, K, B, _ptr(G)) != 0:
        raise ValueError("oracle rejected the arguments")
    return G


def quantize_gram(W, fmt: str, block: int, G, *, window: int = -1, rows=None, n_threads=1,
                  sfmt: str = "e4m3") -> Result:
    """Block-Hessian H-optimal search of W [n, k] with the Gram blocks G [k/B, B, B]."""
    W, dt = _as_input(W)
    n, k = W.shape
    G = np.ascontiguousarray(G, dtype=np.float32)
    if G.shape != (k // block, block, block):
        raise ValueError("G must be [k/B, B, B]")
    f = FMTS[fmt]
    kb = k // block
    codes = np.zeros((n, k // 2) if f in (NVFP4, INT4) else (n, k), np.uint8)
    scales = np.zeros((n, kb), np.uint8)
    best = np.full((n, kb), np.nan)
    second = np.full((n, kb), np.nan)
    naive = np.full((n, kb), -1, np.int32)
    r0, r1 = (0, n) if rows is None else rows

    def run(a, b):
        rc = lib().orc_quantize_blocks_gram(_ptr(W), dt, n, k, k, _ptr(G), f, SFMTS[sfmt],
                                            block, window, a, b, _ptr(codes), _ptr(scales),
                                            _ptr(best), _ptr(second), _ptr(naive))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
    _run_ranges(run, r0, r1, _threads(n_threads))
    return Result(codes=codes, scales=scales, best=best, second=second, naive=naive)


def _run_ranges(fn, r0, r1, nt):
    if nt == 1 or r1 - r0 <= 1:
        fn(r0, r1)
        return
    bounds = np.linspace(r0, r1, min(nt, r1 - r0) + 1).astype(np.int64)
    with ThreadPoolExecutor(len(bounds) - 1) as ex:
        list(ex.map(lambda i: fn(int(bounds[i]), int(bounds[i + 1])), range(len(bounds) - 1)))


def dequant(codes, scales, fmt: str, block: int, n: int, k: int,
            sfmt: str = "e4m3") -> np.ndarray:
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    out = np.zeros((n, k), np.float32)
    rc = lib().orc_dequant(_ptr(codes), _ptr(scales), FMTS[fmt], SFMTS[sfmt], block, n, k,
                           _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def gptq_prepare(G, damp: float = 0.01) -> np.ndarray:
    """U [k/64, 64, 64] float32 for FP8-GPTQ on 64 x 64 tiles ("quantization_algorithms.txt",
    sec. 1): per column block H = G + lambda I with lambda = damp * mean(diag G) (1 when that
    mean is 0 -- an all-zero block), H^-1, and U its upper Cholesky factor (H^-1 = U^T U),
    all in float64, rounded to float32 once. G: the Gram blocks (block_gram(X, 64))."""
    G = np.asarray(G, dtype=np.float64)
    U = np.zeros(G.shape, np.float32)
    for b in range(G.shape[0]):
        lam = damp * float(np.mean(np.diag(G[b])))
        H = G[b] + (lam if lam > 0 else 1.0) * np.eye(G.shape[1])
        Hinv = np.linalg.inv(H)
        U[b] = np.linalg.cholesky((Hinv + Hinv.T) / 2).T.astype(np.float32)
    return U


def gptq_tiles(W, U, scales, want_prop=False):
    """E4M3 codes [n, k] of the tile GPTQ sweep with fixed tile scales; optionally the
    propagated weights (float32 [n, k]) at the moment each column was quantised."""
    W, dt = _as_input(W)
    n, k = W.shape
    U = np.ascontiguousarray(U, dtype=np.float32)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    codes = np.zeros((n, k), np.uint8)
    prop = np.zeros((n, k), np.float32) if want_prop else None
    if lib().orc_gptq_tiles(_ptr(W), dt, n, k, k, _ptr(U), _ptr(scales), _ptr(codes),
                            _ptr(prop)) != 0:
        raise ValueError("oracle rejected the arguments")
    return (codes, prop) if want_prop else codes


def gram(X) -> np.ndarray:
    """The full K x K Gram matrix H = fl32(X^T X / R) of X [R, K] (float64 product)."""
    Xf = to_float(X).astype(np.float64)
    R = Xf.shape[0]
    return (Xf.T @ Xf / R).astype(np.float32) if R else np.zeros((Xf.shape[1],) * 2, np.float32)


def gram_entries(X, pairs, chunk_rows: int = 16384) -> np.ndarray:
    """Entries (i, j) of the Gram matrix H = X^T X / R of X [R, K] (float64 sums of the exact
    products, then / R; float64 result) for pairs [P, 2] of column indices -- the same
    definition as ``gram`` for matrices too large to multiply out on the host."""
    Xin, _ = _as_input(X)
    R = Xin.shape[0]
    pairs = np.asarray(pairs, np.int64)
    cols, inv = np.unique(pairs.reshape(-1), return_inverse=True)
    a, b = inv.reshape(-1, 2).T
    acc = np.zeros(len(pairs))
    for r0 in range(0, R, chunk_rows):
        Xc = to_float(Xin[r0:r0 + chunk_rows])[:, cols].astype(np.float64)
        acc += (Xc[:, a] * Xc[:, b]).sum(axis=0)
    return acc / R if R else acc


def block_losses(W, h, fmt: str, mode: str, block: int, *, sfmt: str = "e4m3",
                 window: int = -1, n_threads=1) -> np.ndarray:
    """Hessian-weighted quantization loss of each column block: sum over rows and the
    block's columns of h_j (w_ij - w^_ij)^2 (float64; each row's block summed, then the rows
    in ascending order) for the block quantizer's own (uncompensated) result.

    The qwantize "GPTQ Quantization" section orders blocks by this loss but fixes no
    summation order; rows outer, a block's columns inner, is the reading taken here. A
    device that sums in another order can swap two blocks whose losses agree to ~1e-15, so
    block orders are compared under a 1e-12 relative tie rule."""
    W, _ = _as_input(W)
    n, k = W.shape
    r = quantize(W, fmt, mode, block, h=h if mode == "hopt" else None, window=window,
                 sfmt=sfmt, n_threads=n_threads)
    What = dequant(r.codes, r.scales, fmt, block, n, k, sfmt=sfmt).astype(np.float64)
    d = to_float(W).astype(np.float64) - What
    e = (d * d) * np.asarray(h, np.float64)[None, :]
    per_row = e.reshape(n, k // block, block).sum(axis=2)
    loss = np.zeros(k // block)
    for i in range(n):
        loss += per_row[i]
    return loss


def block_order(losses) -> np.ndarray:
    """Ordered GPTQ's block sequence: descending loss, the lower block first on equal loss."""
    losses = np.asarray(losses, np.float64)
    return np.array(sorted(range(len(losses)), key=lambda b: (-losses[b], b)), np.int32)


def gptq_blocks(W, U, h, fmt: str, mode: str, block: int, *, sfmt: str = "e4m3",
                window: int = -1, perm=None, rows=None, n_threads=1) -> Result:
    """GPTQ with the block quantizer as its inner step (orc_gptq_blocks): codes and scales
    in the layouts of ``quantize``. U [k, k]: the factor of the damped H^-1 in sweep order;
    perm: the block visited at each sweep position (None: natural order)."""
    W, dt = _as_input(W)
    n, k = W.shape
    f, m = FMTS[fmt], MODES[mode]
    if f == E4M3:
        raise ValueError("E4M3 elements: gptq_tiles")
    hp = None if h is None else np.ascontiguousarray(h, dtype=np.float32)
    if m == HOPT and hp is None:
        raise ValueError("H-optimal needs h")
    U = np.ascontiguousarray(U, dtype=np.float32)
    pp = None if perm is None else np.ascontiguousarray(perm, dtype=np.int32)
    codes = np.zeros((n, k // 2) if f in (NVFP4, INT4) else (n, k), np.uint8)
    scales = np.zeros((n, k // block), np.uint8)
    r0, r1 = (0, n) if rows is None else rows

    def run(a, b):
        if lib().orc_gptq_blocks(_ptr(W), dt, n, k, k, _ptr(hp), f, SFMTS[sfmt], m, block,
                                 window, _ptr(U), _ptr(pp), a, b, _ptr(codes),
                                 _ptr(scales)) != 0:
            raise ValueError("oracle rejected the arguments")
    _run_ranges(run, r0, r1, _threads(n_threads))
    return Result(codes=codes, scales=scales, best=None, second=None, naive=None)


def gptq(W, H, h, fmt: str, mode: str, block: int, *, ordered: bool = False,
         damp: float = 0.01, sfmt: str = "e4m3", window: int = -1, rows=None,
         n_threads=1) -> Result:
    """Sequential (natural block order) or ordered (descending block loss) GPTQ of W [n, k]
    with Hessian H [k, k] (e.g. gram(X)) and h = diag(H) for the H-optimal search. Returns
    codes and scales in the original column order; ``naive`` holds the block order used."""
    k = np.asarray(H).shape[0]
    perm = block_order(block_losses(W, h, fmt, mode, block, sfmt=sfmt, window=window)) \
        if ordered else np.arange(k // block, dtype=np.int32)
    cols = (perm[:, None] * block + np.arange(block)[None, :]).reshape(-1)
    Hp = np.asarray(H, np.float32)[np.ix_(cols, cols)]
    U = gptq_prepare(Hp[None], damp)[0]
    r = gptq_blocks(W, U, h, fmt, mode, block, sfmt=sfmt, window=window,
                    perm=perm if ordered else None, rows=rows, n_threads=n_threads)
    r["naive"] = perm
    return r


def swizzle_scales(scales) -> np.ndarray:
    """Scale bytes [n, kb] in the 128 x 4 tile layout of sm_100 block-scaled MMA (flat)."""
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    n, kb = scales.shape
    out = np.zeros(((n + 127) // 128) * 128 * ((kb + 3) // 4) * 4, np.uint8)
    lib().orc_swizzle_scales(_ptr(scales), n, kb, _ptr(out))
    return out


def error_sums(W, What, h=None) -> np.ndarray:
    """[sum d^2, sum w^2, sum h d^2, sum h w^2] in float64."""
    W, dt = _as_input(W)
    n, k = W.shape
    What = np.ascontiguousarray(What, dtype=np.float32)
    hh = None if h is None else np.ascontiguousarray(h, dtype=np.float32)
    out = np.zeros(4, np.float64)
    lib().orc_error_sums(_ptr(W), dt, n, k, k, _ptr(What), _ptr(hh), _ptr(out))
    return out


def metrics(sums) -> dict:
    """Relative weight error and relative h-weighted error from the four sums."""
    s = [float(x) for x in sums]
    return {"sse": s[0], "w_sq": s[1], "hsse": s[2], "hw_sq": s[3],
            "weight_rel": (s[0] / s[1]) ** 0.5 if s[1] > 0 else 0.0,
            "h_rel": (s[2] / s[3]) ** 0.5 if s[3] > 0 else 0.0}


def to_float(W) -> np.ndarray:
    """float32 image of an oracle input (bf16 bits widened exactly)."""
    W, dt = _as_input(W)
    if dt == F32:
        return W
    return (W.astype(np.uint32) << 16).view(np.float32)


def output_error(X_rows, W, What) -> float:
    """||X_s What^T - X_s W^T||_F / ||X_s W^T||_F in float64 (X_s: the sampled rows)."""
    Xs = to_float(X_rows).astype(np.float64)
    Wf = to_float(W).astype(np.float64)
    Y = Xs @ Wf.T
    Yq = Xs @ np.asarray(What, np.float64).T
    den = np.linalg.norm(Y)
    return float(np.linalg.norm(Yq - Y) / den) if den > 0 else 0.0


def near_tie(best, second, rel=1e-6) -> np.ndarray:
    """Blocks whose two best candidate errors differ by less than ``rel`` relative."""
    best = np.asarray(best)
    second = np.asarray(second)
    with np.errstate(invalid="ignore", divide="ignore"):
        return ((second - best) < rel * best) | ((best == 0) & (second == 0))
