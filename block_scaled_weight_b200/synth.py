"""Seeded synthetic inputs for block-scaled weight quantization.

This module only draws random numbers. It holds none of the quantization method's
arithmetic, so both the CUDA path and the CPU oracle can consume what it produces.

The shapes and statistics stand in for the workload on the qwantize results page
("Results", benchmark note): the ``down_proj`` weight of a Qwen3-4B decoder layer
(W 2560x9728 bf16) and calibration activations collected on WikiText-2
(X 244449x9728 bf16). Neither the model nor the dataset is used; the matrices below
take their shapes and a heavy-tailed, outlier-carrying statistic instead:

* weights: ``w_ij ~ N(0, sigma_i^2)``, ``sigma_i = exp(mu + s*z_i)`` (per output row
  lognormal), with a few input columns multiplied by a large factor (outliers);
* activations: ``x_rj ~ N(0, tau_j^2)``, ``tau_j = exp(z_j)`` (per input channel
  lognormal), with a few channels multiplied by a large factor;
* the E4M3-element workload draws Student-t (nu = 4) entries times a per-row
  lognormal scale.

Every draw is fp32 from a ``torch.Generator`` seeded by (config seed, stream id);
bf16 tensors are the round-to-nearest-even cast of those fp32 draws. Outlier columns
are the first ``n`` entries of a seeded permutation. Draws on a CUDA device use the
CUDA generator, so the same seed gives different (equally valid) numbers on CPU and
GPU: a parity check always feeds both sides the same bytes.
"""
from __future__ import annotations

import dataclasses

import torch

# Stream ids keep independent draws independent of generation order.
_S_ROW_STD, _S_W, _S_W_OUT, _S_CH_STD, _S_X, _S_X_OUT, _S_SAMPLE = range(7)


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed) * 1_000_003 + int(stream) * 7_919 + 17)
    return g


def _cast(t: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    return t if t.dtype == dtype else t.to(dtype)


def lognormal(n: int, mu: float, s: float, gen: torch.Generator, device) -> torch.Tensor:
    """``exp(mu + s*z)`` for ``n`` standard normal draws ``z`` (fp32)."""
    z = torch.randn(n, generator=gen, device=device, dtype=torch.float32)
    return torch.exp(mu + s * z)


def outlier_columns(k: int, count: int, gen: torch.Generator, device) -> torch.Tensor:
    """The first ``count`` entries of a seeded permutation of ``range(k)``."""
    if count <= 0:
        return torch.empty(0, dtype=torch.long, device=device)
    return torch.randperm(k, generator=gen, device=device)[:count]


def gaussian_weight(n: int, k: int, seed: int, *, dtype=torch.bfloat16, device="cpu",
                    mu: float = -3.0, s: float = 0.5, n_outlier_cols: int = 2,
                    outlier_factor: float = 20.0, stream_base: int = 0) -> torch.Tensor:
    """W [n, k]: row-lognormal Gaussian entries with a few outlier input columns."""
    sig = lognormal(n, mu, s, _gen(seed, stream_base + _S_ROW_STD, device), device)
    w = torch.randn(n, k, generator=_gen(seed, stream_base + _S_W, device), device=device,
                    dtype=torch.float32)
    w.mul_(sig[:, None])
    cols = outlier_columns(k, n_outlier_cols, _gen(seed, stream_base + _S_W_OUT, device), device)
    if cols.numel():
        w[:, cols] *= outlier_factor
    return _cast(w, dtype)


def student_t_weight(n: int, k: int, seed: int, *, nu: int = 4, dtype=torch.bfloat16,
                     device="cpu", mu: float = -3.0, s: float = 0.7,
                     stream_base: int = 0) -> torch.Tensor:
    """W [n, k] = Student-t(nu) entries times a per-row ``exp(mu + s*z)`` scale.

    Student-t(nu) is drawn as ``z0 / sqrt(chi2_nu / nu)`` with ``chi2_nu`` the sum of
    ``nu`` squared standard normals.
    """
    sig = lognormal(n, mu, s, _gen(seed, stream_base + _S_ROW_STD, device), device)
    g = _gen(seed, stream_base + _S_W, device)
    z0 = torch.randn(n, k, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(n, k, device=device, dtype=torch.float32)
    for _ in range(nu):
        zi = torch.randn(n, k, generator=g, device=device, dtype=torch.float32)
        chi2.addcmul_(zi, zi)
    w = z0 / torch.sqrt(chi2 / nu)
    w.mul_(sig[:, None])
    return _cast(w, dtype)


def activations(r: int, k: int, seed: int, *, dtype=torch.bfloat16, device="cpu",
                mu: float = 0.0, s: float = 1.0, n_outlier: int = 3,
                outlier_factor: float = 50.0, chunk_rows: int = 16384,
                stream_base: int = 0, out: torch.Tensor | None = None) -> torch.Tensor:
    """X [r, k]: channel-lognormal Gaussian activations with a few outlier channels.

    Rows are drawn in chunks of ``chunk_rows`` so a multi-GB bf16 matrix never needs its
    fp32 image in memory at once. ``out`` may be a preallocated [r, k] tensor.
    """
    tau = lognormal(k, mu, s, _gen(seed, stream_base + _S_CH_STD, device), device)
    cols = outlier_columns(k, n_outlier, _gen(seed, stream_base + _S_X_OUT, device), device)
    if cols.numel():
        tau[cols] *= outlier_factor
    if out is None:
        out = torch.empty(r, k, dtype=dtype, device=device)
    g = _gen(seed, stream_base + _S_X, device)
    for r0 in range(0, r, chunk_rows):
        r1 = min(r, r0 + chunk_rows)
        x = torch.randn(r1 - r0, k, generator=g, device=device, dtype=torch.float32)
        x.mul_(tau[None, :])
        out[r0:r1].copy_(x)
    return out


def sample_rows(total: int, count: int, seed: int) -> torch.Tensor:
    """``count`` distinct row indices of ``range(total)`` (sorted), seeded; CPU int64."""
    count = min(count, total)
    g = _gen(seed, _S_SAMPLE, "cpu")
    idx = torch.randperm(total, generator=g)[:count]
    return torch.sort(idx).values


@dataclasses.dataclass(frozen=True)
class Workload:
    """One named synthetic workload: weights, activations and the quantizer settings."""
    name: str
    seed: int
    weights: tuple          # ((name, n, k), ...)
    x_shapes: tuple         # ((rows, k), ...) activation matrices
    w_dtype: torch.dtype
    fmt: str                # "nvfp4" | "int8" | "e4m3"
    blocks: tuple           # block sizes along K (e4m3: tile edge)
    modes: tuple
    window: int             # -1: all 126 E4M3 scales
    x_outliers: int = 3
    x_outlier_factor: float = 50.0
    w_kind: str = "gaussian"


# Named synthetic workloads (shapes, statistics, quantizer settings).
WORKLOADS = {
    "tiny_nvfp4": Workload("tiny_nvfp4", 0, (("w", 64, 256),), ((512, 256),), torch.float32,
                           "nvfp4", (16,), ("naive", "sse", "hopt"), -1),
    "int8_e4m3scale": Workload("int8_e4m3scale", 1, (("w", 2560, 9728),), ((4096, 9728),),
                               torch.bfloat16, "int8", (32, 64, 128, 256),
                               ("naive", "sse", "hopt"), 8),
    "nvfp4_full_calib": Workload("nvfp4_full_calib", 2, (("down_proj", 2560, 9728),),
                                 ((244449, 9728),), torch.bfloat16, "nvfp4", (16, 32),
                                 ("naive", "sse", "hopt"), -1, x_outliers=16,
                                 x_outlier_factor=100.0),
    "e4m3_tiles": Workload("e4m3_tiles", 3, (("w", 4096, 4096),), ((8192, 4096),),
                           torch.bfloat16, "e4m3", (64,), ("hopt",), -1, x_outliers=0,
                           w_kind="student_t"),
    "decoder_layer": Workload("decoder_layer", 4,
                              (("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096),
                               ("o", 4096, 4096), ("gate", 14336, 4096), ("up", 14336, 4096),
                               ("down", 4096, 14336)),
                              ((65536, 4096), (65536, 14336)), torch.bfloat16, "nvfp4", (16,),
                              ("hopt",), -1),
}


def workload_weight(wl: Workload, index: int, *, device="cpu", rows: int | None = None,
                    dtype=None) -> torch.Tensor:
    """The ``index``-th weight matrix of a workload (optionally only its first ``rows``)."""
    _, n, k = wl.weights[index]
    n = n if rows is None else min(n, rows)
    dtype = wl.w_dtype if dtype is None else dtype
    if wl.w_kind == "student_t":
        return student_t_weight(n, k, wl.seed, dtype=dtype, device=device,
                                stream_base=100 * index)
    return gaussian_weight(n, k, wl.seed, dtype=dtype, device=device, stream_base=100 * index)


def workload_activations(wl: Workload, index: int, *, device="cpu", rows: int | None = None,
                         dtype=None, out=None) -> torch.Tensor:
    """The ``index``-th activation matrix of a workload (optionally its first ``rows``)."""
    r, k = wl.x_shapes[index]
    r = r if rows is None else min(r, rows)
    dtype = wl.w_dtype if dtype is None else dtype
    return activations(r, k, wl.seed, dtype=dtype, device=device, n_outlier=wl.x_outliers,
                       outlier_factor=wl.x_outlier_factor, stream_base=50 + 100 * index,
                       out=out)


def x_index_for_weight(wl: Workload, index: int) -> int:
    """Which activation matrix feeds weight ``index``: the one whose width is its K."""
    k = wl.weights[index][2]
    for i, (_, kx) in enumerate(wl.x_shapes):
        if kx == k:
            return i
    raise ValueError(f"no activation matrix of width {k} in {wl.name}")
