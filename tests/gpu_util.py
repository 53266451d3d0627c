"""Helpers of the GPU parity tests: move seeded samples to the device and back, and
the tolerances of the parity bar.

Tolerances (the bar stated for this path):
  * fp32 I/O          : max |err| <= 1e-5 * max |ref|
  * bf16 I/O, fp32 acc: |err| <= 2e-2 * rms(ref) for every element
"""
import numpy as np
import torch

from synthetic import bf16_bits_to_f64

FP32_TOL = 1e-5
BF16_TOL = 2e-2


def to_device(sample_or_array, dtype: str) -> torch.Tensor:
    a = getattr(sample_or_array, "stored", sample_or_array)
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    raise ValueError(dtype)


def to_host_f64(t: torch.Tensor) -> np.ndarray:
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.cpu().numpy().astype(np.float64)


def assert_parity(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = "") -> float:
    """Checks the bar for `dtype` and returns the error in units of the bar (<= 1 passes)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if dtype == "f32":
        bound = FP32_TOL * np.abs(ref).max()
        ratio = err.max() / bound if bound > 0 else float(err.max() > 0)
    else:
        bound = BF16_TOL * np.sqrt(np.mean(ref * ref))
        ratio = err.max() / bound if bound > 0 else float(err.max() > 0)
    assert ratio <= 1.0, f"{what}: error {err.max():.3e} is {ratio:.2f}x the {dtype} bound {bound:.3e}"
    return ratio
