"""Thin ctypes binding of ``libmxq.so`` (declared in ``include/mxq.h``).

Argument marshalling only: every step of the path runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream. The functions keep the C names;
outputs that are not given are allocated with torch on the input's device.

The binding never falls back to another implementation: if the shared library is
missing it raises ``ImportError`` at import time (build it with
``python -m block_scaled_weight_b200.build`` or ``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmxq.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libmxq.so not built ({_LIB_PATH}); run block_scaled_weight_b200.build")
_lib = ctypes.CDLL(_LIB_PATH)

MXQ_OK = 0
STATUS = {0: "MXQ_OK", 1: "MXQ_ERR_INVALID_ARG", 2: "MXQ_ERR_SHAPE", 3: "MXQ_ERR_DTYPE",
          4: "MXQ_ERR_ALIGN", 5: "MXQ_ERR_UNSUPPORTED", 6: "MXQ_ERR_CUDA",
          7: "MXQ_ERR_WORKSPACE"}
F32, BF16 = 0, 1
FMT = {"nvfp4": 0, "int8": 1, "e4m3": 2, "int4": 3}
MODE = {"naive": 0, "sse": 1, "hopt": 2}
# block-scale grids; MXFP4 is fmt "nvfp4" (E2M1 elements) with scale_fmt "ue8m0"
SCALE = {"e4m3": 0, "ue4m4": 1, "ue5m3": 2, "ue8m0": 3}

EXPORTS = ("mxq_act_sqmean_workspace", "mxq_act_sqmean", "mxq_act_sqmean_noalloc",
           "mxq_act_sqsum", "mxq_act_block_gram_workspace", "mxq_act_block_gram",
           "mxq_act_sqmean_finalize", "mxq_quantize", "mxq_quantize_gram", "mxq_project",
           "mxq_swizzled_scales_bytes", "mxq_swizzle_scales", "mxq_nvfp4_gemm_workspace",
           "mxq_nvfp4_gemm", "mxq_output_error_workspace",
           "mxq_output_error", "mxq_gptq_prepare", "mxq_gptq_tiles", "mxq_act_gram_workspace",
           "mxq_act_gram",
           "mxq_gptq_factor_workspace", "mxq_gptq_factor", "mxq_gptq_order_workspace",
           "mxq_gptq_order", "mxq_gptq_workspace", "mxq_gptq", "mxq_dequant",
           "mxq_error_workspace", "mxq_quantize_err_workspace", "mxq_quantize_err",
           "mxq_error", "mxq_metrics_from_sums", "mxq_status_string", "mxq_last_error",
           "mxq_set_wait_polls")


class MxqParams(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("mode", ctypes.c_int32), ("block", ctypes.c_int32),
                ("tile_rows", ctypes.c_int32), ("window", ctypes.c_int32),
                ("log_points", ctypes.c_int32), ("log_lo_exp2", ctypes.c_float),
                ("log_hi_exp2", ctypes.c_float), ("scale_fmt", ctypes.c_int32),
                ("ctas_per_sm", ctypes.c_int32)]


class MxqMetrics(ctypes.Structure):
    _fields_ = [(n, ctypes.c_double) for n in ("sse", "w_sq", "hsse", "hw_sq", "weight_rel",
                                               "h_rel")]


_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_sig = {
    "mxq_act_sqmean_workspace": (_SZ, [_I64, _I64]),
    "mxq_act_sqmean": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "mxq_act_sqmean_noalloc": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, _P]),
    "mxq_act_sqsum": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "mxq_act_sqmean_finalize": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P]),
    "mxq_act_block_gram_workspace": (_SZ, [_I64, _I64, _I32]),
    "mxq_act_block_gram": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _I32, _P, _P, _P, _SZ,
                                          _P]),
    "mxq_quantize": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, ctypes.POINTER(MxqParams),
                                    _P, _P, _P]),
    "mxq_quantize_gram": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P,
                                         ctypes.POINTER(MxqParams), _P, _P, _P]),
    "mxq_project": (ctypes.c_int, [_P, _I64, _I32, _I32, ctypes.c_float, _P, _P]),
    "mxq_swizzled_scales_bytes": (_SZ, [_I64, _I64]),
    "mxq_output_error_workspace": (_SZ, [_I64, _I64]),
    "mxq_output_error": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _I64, _I64, _P, _P,
                                        ctypes.POINTER(MxqParams), _P, _P, _SZ, _P]),
    "mxq_swizzle_scales": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "mxq_nvfp4_gemm_workspace": (_SZ, []),
    "mxq_nvfp4_gemm": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "mxq_gptq_prepare": (ctypes.c_int, [_P, _I64, ctypes.c_double, _P, _P]),
    "mxq_gptq_tiles": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _P]),
    "mxq_act_gram_workspace": (_SZ, [_I64, _I64]),
    "mxq_act_gram": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "mxq_gptq_factor_workspace": (_SZ, [_I64]),
    "mxq_gptq_factor": (ctypes.c_int, [_P, _I64, _I32, _P, ctypes.c_double, _P, _P, _SZ, _P]),
    "mxq_gptq_order_workspace": (_SZ, [_I64, _I64, ctypes.POINTER(MxqParams)]),
    "mxq_gptq_order": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, ctypes.POINTER(MxqParams),
                                      _P, _P, _SZ, _P]),
    "mxq_gptq_workspace": (_SZ, [_I64, _I64]),
    "mxq_gptq": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, _P, _P,
                                ctypes.POINTER(MxqParams), _P, _P, _P, _SZ, _P]),
    "mxq_dequant": (ctypes.c_int, [_P, _P, ctypes.POINTER(MxqParams), _I64, _I64, _P, _P]),
    "mxq_error_workspace": (_SZ, [_I64, _I64]),
    "mxq_quantize_err_workspace": (_SZ, [_I64, _I64, ctypes.POINTER(MxqParams)]),
    "mxq_quantize_err": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, ctypes.POINTER(MxqParams),
                                        _P, _P, _P, _P, _SZ, _P]),
    "mxq_error": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, _P, _P,
                                 ctypes.POINTER(MxqParams), _P, _P, _SZ, _P]),
    "mxq_metrics_from_sums": (ctypes.c_int, [_P, ctypes.POINTER(MxqMetrics)]),
    "mxq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mxq_last_error": (ctypes.c_char_p, []),
    "mxq_set_wait_polls": (None, [ctypes.c_uint32]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class MxqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.mxq_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


def _check(status: int, where: str):
    if status != MXQ_OK:
        raise MxqError(status, where)


def lib_path() -> str:
    return _LIB_PATH


def params(fmt="nvfp4", mode="hopt", block=16, *, window=-1, tile_rows=None, log_points=64,
           log_lo_exp2=-2.0, log_hi_exp2=2.0, scale_fmt="e4m3", ctas_per_sm=0) -> MxqParams:
    f = FMT[fmt] if isinstance(fmt, str) else int(fmt)
    sf = SCALE[scale_fmt] if isinstance(scale_fmt, str) else int(scale_fmt)
    m = MODE[mode] if isinstance(mode, str) else int(mode)
    if tile_rows is None:
        tile_rows = block if f == FMT["e4m3"] else 1
    return MxqParams(f, m, block, tile_rows, window, log_points, log_lo_exp2, log_hi_exp2, sf,
                     ctas_per_sm)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    return 99  # rejected by the library with MXQ_ERR_DTYPE


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return t.stride(0)


def mxq_act_sqmean_workspace(rows: int, cols: int) -> int:
    return int(_lib.mxq_act_sqmean_workspace(rows, cols))


def mxq_error_workspace(n: int, k: int) -> int:
    return int(_lib.mxq_error_workspace(n, k))


def _workspace(nbytes, device, ws):
    if ws is not None:
        return ws
    return torch.empty(max(int(nbytes), 8), dtype=torch.uint8, device=device)


def mxq_act_sqmean(X: torch.Tensor, h: torch.Tensor | None = None, *, workspace=None,
                   stream=None) -> torch.Tensor:
    """h_j = mean_r X[r, j]^2 (float32 [cols])."""
    R, K = X.shape
    if h is None:
        h = torch.empty(K, dtype=torch.float32, device=X.device)
    ws = _workspace(mxq_act_sqmean_workspace(R, K), X.device, workspace)
    _check(_lib.mxq_act_sqmean(_ptr(X), _dtype(X), R, K, _ld(X), _ptr(h), _ptr(ws), ws.numel(),
                               _stream(stream, X.device)), "mxq_act_sqmean")
    return h


def mxq_act_sqmean_noalloc(X: torch.Tensor, h: torch.Tensor | None = None, *,
                           stream=None) -> torch.Tensor:
    """h_j = mean_r X[r, j]^2 without a workspace: the library's static 1 MiB device scratch
    is used instead (for callers that must not allocate device memory; widths up to 131072
    columns). Calls that overlap on the GPU share that scratch and must be ordered."""
    R, K = X.shape
    if h is None:
        h = torch.empty(K, dtype=torch.float32, device=X.device)
    _check(_lib.mxq_act_sqmean_noalloc(_ptr(X), _dtype(X), R, K, _ld(X), _ptr(h),
                                       _stream(stream, X.device)), "mxq_act_sqmean_noalloc")
    return h


def mxq_act_sqsum(X: torch.Tensor, colsum: torch.Tensor | None = None, *, workspace=None,
                  stream=None) -> torch.Tensor:
    """sum_r X[r, j]^2 over this shard's rows (float64 [cols])."""
    R, K = X.shape
    if colsum is None:
        colsum = torch.empty(K, dtype=torch.float64, device=X.device)
    ws = _workspace(mxq_act_sqmean_workspace(R, K), X.device, workspace)
    _check(_lib.mxq_act_sqsum(_ptr(X), _dtype(X), R, K, _ld(X), _ptr(colsum), _ptr(ws),
                              ws.numel(), _stream(stream, X.device)), "mxq_act_sqsum")
    return colsum


def mxq_act_block_gram_workspace(rows: int, cols: int, block: int) -> int:
    return int(_lib.mxq_act_block_gram_workspace(rows, cols, block))


def mxq_act_block_gram(X: torch.Tensor, block: int = 16, G: torch.Tensor | None = None,
                       h: torch.Tensor | None = None, *, with_h=False, workspace=None,
                       stream=None):
    """Gram blocks G [cols/B, B, B] = fl32(X_b^T X_b / R) of bf16 X (tensor cores); with
    ``with_h`` (or ``h`` given) also h = diag(G). Returns G, or (G, h)."""
    R, K = X.shape
    if G is None:
        G = torch.empty(K // block, block, block, dtype=torch.float32, device=X.device)
    if with_h and h is None:
        h = torch.empty(K, dtype=torch.float32, device=X.device)
    ws = _workspace(mxq_act_block_gram_workspace(R, K, block), X.device, workspace)
    _check(_lib.mxq_act_block_gram(_ptr(X), _dtype(X), R, K, _ld(X), block, _ptr(G), _ptr(h),
                                   _ptr(ws), ws.numel(), _stream(stream, X.device)),
           "mxq_act_block_gram")
    return (G, h) if h is not None else G


def mxq_act_sqmean_finalize(partials: torch.Tensor, total_rows: int,
                            h: torch.Tensor | None = None, *, stream=None) -> torch.Tensor:
    """h from gathered per-shard column sums ``partials`` [parts, cols] (float64)."""
    parts, K = partials.shape
    if h is None:
        h = torch.empty(K, dtype=torch.float32, device=partials.device)
    _check(_lib.mxq_act_sqmean_finalize(_ptr(partials.contiguous()), parts, K, int(total_rows),
                                        _ptr(h), _stream(stream, partials.device)),
           "mxq_act_sqmean_finalize")
    return h


def output_shapes(p: MxqParams, n: int, k: int):
    """(codes shape, codes dtype, scales shape, scales dtype) for a quantization."""
    if p.fmt in (FMT["nvfp4"], FMT["int4"]):
        return (n, k // 2), torch.uint8, (n, k // p.block), torch.uint8
    if p.fmt == FMT["int8"]:
        return (n, k), torch.int8, (n, k // p.block), torch.uint8
    return (n, k), torch.uint8, (n // p.block, k // p.block), torch.float32


def mxq_quantize(W: torch.Tensor, p: MxqParams, h: torch.Tensor | None = None, *, codes=None,
                 scales=None, stream=None):
    """(codes, scales) of W [n, k] under settings ``p`` (see ``params``)."""
    n, k = W.shape
    cs, cd, ss, sd = output_shapes(p, n, k)
    if codes is None:
        codes = torch.empty(cs, dtype=cd, device=W.device)
    if scales is None:
        scales = torch.empty(ss, dtype=sd, device=W.device)
    _check(_lib.mxq_quantize(_ptr(W), _dtype(W), n, k, _ld(W), _ptr(h), ctypes.byref(p),
                             _ptr(codes), _ptr(scales), _stream(stream, W.device)),
           "mxq_quantize")
    return codes, scales


def mxq_quantize_gram(W: torch.Tensor, p: MxqParams, G: torch.Tensor, *, codes=None,
                      scales=None, stream=None):
    """(codes, scales) of W [n, k] minimising d^T G_b d per block (G [k/B, B, B] float)."""
    n, k = W.shape
    cs, cd, ss, sd = output_shapes(p, n, k)
    if codes is None:
        codes = torch.empty(cs, dtype=cd, device=W.device)
    if scales is None:
        scales = torch.empty(ss, dtype=sd, device=W.device)
    _check(_lib.mxq_quantize_gram(_ptr(W), _dtype(W), n, k, _ld(W), _ptr(G), ctypes.byref(p),
                                  _ptr(codes), _ptr(scales), _stream(stream, W.device)),
           "mxq_quantize_gram")
    return codes, scales


def mxq_project(w: torch.Tensor, fmt: str, scale: float, *, scale_fmt="e4m3", q=None,
                stream=None) -> torch.Tensor:
    """Magnitude codes of float32 ``w`` at one fixed scale (the search's element step);
    ``scale`` is a value of the grid ``scale_fmt`` (NVFP4 / INT4 / INT8)."""
    w = w.contiguous()
    if q is None:
        q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    _check(_lib.mxq_project(_ptr(w), w.numel(), FMT[fmt], SCALE[scale_fmt], float(scale),
                            _ptr(q), _stream(stream, w.device)), "mxq_project")
    return q


def mxq_gptq_prepare(G: torch.Tensor, damp: float = 0.01, *, U=None, stream=None) -> torch.Tensor:
    """U [nb, 64, 64] float32: the upper Cholesky factor of the inverse of each damped Gram
    block G [nb, 64, 64] (float32, from mxq_act_block_gram with block 64)."""
    nb = G.shape[0]
    if U is None:
        U = torch.empty((nb, 64, 64), dtype=torch.float32, device=G.device)
    _check(_lib.mxq_gptq_prepare(_ptr(G), nb, float(damp), _ptr(U), _stream(stream, G.device)),
           "mxq_gptq_prepare")
    return U


def mxq_gptq_tiles(W: torch.Tensor, U: torch.Tensor, scales: torch.Tensor, *, codes=None,
                   stream=None) -> torch.Tensor:
    """E4M3 codes [n, k] (uint8, sign << 7 | code) of the tile GPTQ sweep of W [n, k] at the
    tile scales [n/64, k/64] (float32) with the factors U [k/64, 64, 64]."""
    n, k = W.shape
    if codes is None:
        codes = torch.empty((n, k), dtype=torch.uint8, device=W.device)
    _check(_lib.mxq_gptq_tiles(_ptr(W), _dtype(W), n, k, _ld(W), _ptr(U), _ptr(scales),
                               _ptr(codes), _stream(stream, W.device)), "mxq_gptq_tiles")
    return codes


def mxq_act_gram_workspace(rows: int, cols: int) -> int:
    return int(_lib.mxq_act_gram_workspace(rows, cols))


def mxq_act_gram(X: torch.Tensor, H: torch.Tensor | None = None, *, workspace=None,
                 stream=None) -> torch.Tensor:
    """H = X^T X / R [K, K] float32 of bf16 X [R, K] (GPTQ's Hessian up to a factor)."""
    R, K = X.shape
    if H is None:
        H = torch.empty(K, K, dtype=torch.float32, device=X.device)
    ws = _workspace(mxq_act_gram_workspace(R, K), X.device, workspace)
    _check(_lib.mxq_act_gram(_ptr(X), _dtype(X), R, K, _ld(X), _ptr(H), _ptr(ws), ws.numel(),
                             _stream(stream, X.device)), "mxq_act_gram")
    return H


def mxq_gptq_factor_workspace(k: int) -> int:
    return int(_lib.mxq_gptq_factor_workspace(k))


def mxq_gptq_order_workspace(n: int, k: int, p: MxqParams) -> int:
    return int(_lib.mxq_gptq_order_workspace(n, k, ctypes.byref(p)))


def mxq_gptq_workspace(n: int, k: int) -> int:
    return int(_lib.mxq_gptq_workspace(n, k))


def mxq_gptq_factor(H: torch.Tensor, block: int, perm: torch.Tensor | None = None,
                    damp: float = 0.01, *, U=None, workspace=None, stream=None) -> torch.Tensor:
    """U [K, K] float32: the upper Cholesky factor of the damped H^-1 in sweep order."""
    K = H.shape[0]
    if U is None:
        U = torch.empty(K, K, dtype=torch.float32, device=H.device)
    ws = _workspace(mxq_gptq_factor_workspace(K), H.device, workspace)
    _check(_lib.mxq_gptq_factor(_ptr(H), K, block, _ptr(perm), float(damp), _ptr(U), _ptr(ws),
                                ws.numel(), _stream(stream, H.device)), "mxq_gptq_factor")
    return U


def mxq_gptq_order(W: torch.Tensor, h: torch.Tensor, p: MxqParams, *, perm=None,
                   workspace=None, stream=None) -> torch.Tensor:
    """Ordered GPTQ's block sequence (int32 [k / block]): descending Hessian-weighted loss."""
    n, k = W.shape
    if perm is None:
        perm = torch.empty(k // p.block, dtype=torch.int32, device=W.device)
    ws = _workspace(mxq_gptq_order_workspace(n, k, p), W.device, workspace)
    _check(_lib.mxq_gptq_order(_ptr(W), _dtype(W), n, k, _ld(W), _ptr(h), ctypes.byref(p),
                               _ptr(perm), _ptr(ws), ws.numel(), _stream(stream, W.device)),
           "mxq_gptq_order")
    return perm


def mxq_gptq(W: torch.Tensor, U: torch.Tensor, p: MxqParams, h: torch.Tensor | None = None,
             perm: torch.Tensor | None = None, *, codes=None, scales=None, workspace=None,
             stream=None):
    """(codes, scales) of the GPTQ sweep of W [n, k] (layouts of mxq_quantize)."""
    n, k = W.shape
    cs, cd, ss, sd = output_shapes(p, n, k)
    if codes is None:
        codes = torch.empty(cs, dtype=cd, device=W.device)
    if scales is None:
        scales = torch.empty(ss, dtype=sd, device=W.device)
    ws = _workspace(mxq_gptq_workspace(n, k), W.device, workspace)
    _check(_lib.mxq_gptq(_ptr(W), _dtype(W), n, k, _ld(W), _ptr(h), _ptr(U), _ptr(perm),
                         ctypes.byref(p), _ptr(codes), _ptr(scales), _ptr(ws), ws.numel(),
                         _stream(stream, W.device)), "mxq_gptq")
    return codes, scales


def mxq_output_error(X: torch.Tensor, W: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                     p: MxqParams, *, sums=None, workspace=None, stream=None) -> torch.Tensor:
    """[sum (X Wq^T - X W^T)^2, sum (X W^T)^2] (float64, device) for bf16 X [m, k], W [n, k]."""
    m, k = X.shape
    n = W.shape[0]
    if sums is None:
        sums = torch.empty(2, dtype=torch.float64, device=X.device)
    ws = _workspace(int(_lib.mxq_output_error_workspace(m, n)), X.device, workspace)
    _check(_lib.mxq_output_error(_ptr(X), m, k, _ld(X), _ptr(W), n, _ld(W), _ptr(codes),
                                 _ptr(scales), ctypes.byref(p), _ptr(sums), _ptr(ws), ws.numel(),
                                 _stream(stream, X.device)), "mxq_output_error")
    return sums


def mxq_swizzle_scales(scales: torch.Tensor, *, out=None, stream=None) -> torch.Tensor:
    """Row-major scale bytes [n, kb] -> the 128 x 4 tile layout of block-scaled MMA (flat)."""
    scales = scales.contiguous()
    n, kb = scales.shape
    if out is None:
        out = torch.empty(int(_lib.mxq_swizzled_scales_bytes(n, kb)), dtype=torch.uint8,
                          device=scales.device)
    _check(_lib.mxq_swizzle_scales(_ptr(scales), n, kb, _ptr(out), _stream(stream, scales.device)),
           "mxq_swizzle_scales")
    return out


def mxq_nvfp4_gemm(a_codes: torch.Tensor, a_scales_sw: torch.Tensor, b_codes: torch.Tensor,
                   b_scales_sw: torch.Tensor, m: int, n: int, k: int, *, D=None, workspace=None,
                   stream=None) -> torch.Tensor:
    """D = dequant(A) dequant(B)^T [m, n] float32 on the block-scaled tensor cores, from NVFP4
    codes [rows, k/2] and scales already in the swizzled layout (mxq_swizzle_scales)."""
    if D is None:
        D = torch.empty(m, n, dtype=torch.float32, device=a_codes.device)
    ws = _workspace(int(_lib.mxq_nvfp4_gemm_workspace()), a_codes.device, workspace)
    _check(_lib.mxq_nvfp4_gemm(_ptr(a_codes), _ptr(a_scales_sw), _ptr(b_codes), _ptr(b_scales_sw),
                               m, n, k, _ptr(D), _ptr(ws), ws.numel(),
                               _stream(stream, a_codes.device)), "mxq_nvfp4_gemm")
    return D


def mxq_dequant(codes: torch.Tensor, scales: torch.Tensor, p: MxqParams, n: int, k: int, *,
                out=None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(n, k, dtype=torch.float32, device=codes.device)
    _check(_lib.mxq_dequant(_ptr(codes), _ptr(scales), ctypes.byref(p), n, k, _ptr(out),
                            _stream(stream, codes.device)), "mxq_dequant")
    return out


def mxq_error(W: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, p: MxqParams,
              h: torch.Tensor | None = None, *, sums=None, workspace=None,
              stream=None) -> torch.Tensor:
    """Device float64 [4]: sum d^2, sum w^2, sum h d^2, sum h w^2."""
    n, k = W.shape
    if sums is None:
        sums = torch.empty(4, dtype=torch.float64, device=W.device)
    ws = _workspace(mxq_error_workspace(n, k), W.device, workspace)
    _check(_lib.mxq_error(_ptr(W), _dtype(W), n, k, _ld(W), _ptr(codes), _ptr(scales), _ptr(h),
                          ctypes.byref(p), _ptr(sums), _ptr(ws), ws.numel(),
                          _stream(stream, W.device)), "mxq_error")
    return sums


def mxq_quantize_err_workspace(n: int, k: int, p: MxqParams) -> int:
    return int(_lib.mxq_quantize_err_workspace(n, k, ctypes.byref(p)))


def mxq_quantize_err(W: torch.Tensor, p: MxqParams, h: torch.Tensor | None = None, *,
                     codes=None, scales=None, sums=None, workspace=None, stream=None):
    """mxq_quantize and mxq_error in one call: (codes, scales, device float64 [4] sums)."""
    n, k = W.shape
    if codes is None or scales is None:
        cs, cd, ss, sd = output_shapes(p, n, k)
        codes = torch.empty(cs, dtype=cd, device=W.device) if codes is None else codes
        scales = torch.empty(ss, dtype=sd, device=W.device) if scales is None else scales
    if sums is None:
        sums = torch.empty(4, dtype=torch.float64, device=W.device)
    ws = _workspace(mxq_quantize_err_workspace(n, k, p), W.device, workspace)
    _check(_lib.mxq_quantize_err(_ptr(W), _dtype(W), n, k, _ld(W), _ptr(h), ctypes.byref(p),
                                 _ptr(codes), _ptr(scales), _ptr(sums), _ptr(ws), ws.numel(),
                                 _stream(stream, W.device)), "mxq_quantize_err")
    return codes, scales, sums


def mxq_metrics_from_sums(sums) -> dict:
    """Metrics from four host doubles (a CPU tensor, a list or a numpy array)."""
    arr = (ctypes.c_double * 4)(*[float(x) for x in list(sums)])
    m = MxqMetrics()
    _check(_lib.mxq_metrics_from_sums(ctypes.cast(arr, ctypes.c_void_p), ctypes.byref(m)),
           "mxq_metrics_from_sums")
    return {name: getattr(m, name) for name, _ in MxqMetrics._fields_}


def mxq_set_wait_polls(polls: int) -> None:
    """Bound of the tensor-core kernels' pipeline waits for later launches (0: the default)."""
    _lib.mxq_set_wait_polls(int(polls))
