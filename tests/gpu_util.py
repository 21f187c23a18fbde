"""Helpers shared by the GPU parity tests (comparison rules and conversions)."""

import numpy as np
import torch

# Tolerance for floating-point outputs against the fp64 oracle evaluated on
# the same dequantised weights: relative L2 error and max abs error relative
# to the largest reference magnitude.
REL_L2 = 5e-3
MAX_ABS_REL = 1e-2


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (host numpy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def from_bits(b: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(device)


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = max(np.linalg.norm(ref), 1e-300)
    rel = np.linalg.norm(got - ref) / den
    mx = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300) if ref.size else 0.0
    return rel, mx


def assert_close(got, ref, name=""):
    rel, mx = errors(got, ref)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    assert rel <= REL_L2 and mx <= MAX_ABS_REL, f"{name}: rel_l2={rel:.3e} max_abs_rel={mx:.3e}"
    return rel, mx
