"""Small conversions shared by the tests (no layer arithmetic here)."""
import numpy as np
import torch


def raw(t: torch.Tensor) -> np.ndarray:
    """A tensor's bytes as numpy: bf16 -> uint16 bit patterns, others as is."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


def as_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Raw stored values -> float64 (dtype one of f32/bf16)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def max_abs_rel(got: np.ndarray, ref: np.ndarray) -> float:
    """max_i |g_i - r_i| / max_i |r_i| over one output tensor."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    denom = np.max(np.abs(ref)) if ref.size else 0.0
    if denom == 0.0:
        return float(np.max(np.abs(got))) if got.size else 0.0
    return float(np.max(np.abs(got - ref)) / denom)
