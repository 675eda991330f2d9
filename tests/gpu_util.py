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
