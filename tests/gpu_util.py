"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch


def oracle_view(t: torch.Tensor) -> np.ndarray:
    """A CPU copy of a float32 or bf16 tensor in the oracle's input form (bf16 as bits)."""
    c = t.detach().to("cpu").contiguous()
    if c.dtype == torch.bfloat16:
        return c.view(torch.int16).numpy().view(np.uint16)
    return c.numpy().astype(np.float32, copy=False)


def all_positive_bf16_f32(device) -> torch.Tensor:
    bits = torch.arange(0, 0x7F80, dtype=torch.int32)
    return (bits << 16).view(torch.float32).to(device)


def near_tie_mask(best, second, rel=1e-6):
    best = np.asarray(best)
    second = np.asarray(second)
    with np.errstate(invalid="ignore"):
        return ((second - best) < rel * best) | ((best == 0) & (second == 0))


def sample_oracle_rows(W_np, rows):
    """Rows of W (oracle form) gathered into a dense matrix."""
    return np.ascontiguousarray(W_np[np.asarray(rows)])


def order_with_ties(perm, perm_ref, losses, rel=1e-12):
    """Check a block order against the oracle's under the tie rule: perm must be a
    permutation, and at every position its block's oracle loss must equal that of the
    oracle's block there to within `rel` relative (the two sides sum each block's float64
    loss in different orders, so blocks whose losses agree to ~1e-15 may swap; the lower
    block first on exactly equal losses is the oracle's own rule). Returns the number of
    adjacent pairs in the oracle order whose losses are that close (the near ties)."""
    perm = np.asarray(perm)
    perm_ref = np.asarray(perm_ref)
    L = np.asarray(losses, np.float64)
    assert np.array_equal(np.sort(perm), np.arange(len(L))), "not a permutation"
    a, b = L[perm], L[perm_ref]
    bad = np.abs(a - b) > rel * np.maximum(np.abs(a), np.abs(b))
    assert not bad.any(), f"{int(bad.sum())} positions differ beyond the tie rule"
    s = L[perm_ref]
    return int((np.abs(s[1:] - s[:-1]) <= rel * np.abs(s[:-1])).sum())


def output_error_np(Xs, W, What) -> float:
    """||X_s What^T - X_s W^T||_F / ||X_s W^T||_F in float64 with plain numpy (a measurement
    of a GPU result in the test itself, so that no GPU output becomes an oracle input)."""
    Xs = np.asarray(Xs, np.float64)
    Y = Xs @ np.asarray(W, np.float64).T
    Yq = Xs @ np.asarray(What, np.float64).T
    den = np.linalg.norm(Y)
    return float(np.linalg.norm(Yq - Y) / den) if den > 0 else 0.0
