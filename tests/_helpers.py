"""Shared helpers of the parity tests: raw-bit views and the comparison
rules of the contract (bit-exact integers and bytes; combine within one
half-precision ulp, or 1e-5 relative to sum_j |w_j y_j| for fp32)."""

import numpy as np
import torch

TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw storage of a CPU/GPU tensor as a numpy array (uint16 for 16-bit
    floats, float32 for fp32, uint8 for bytes)."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def ordered_int16(a: np.ndarray) -> np.ndarray:
    """Map half-precision bit patterns to integers ordered like the values
    (+0 and -0 both map to 0), so that |a - b| counts representable steps."""
    a = a.astype(np.int32)
    mag = a & 0x7FFF
    return np.where(a & 0x8000, -mag, mag)


def assert_half_within_one_ulp(got_bits: np.ndarray, ref_bits: np.ndarray):
    d = np.abs(ordered_int16(got_bits) - ordered_int16(ref_bits))
    assert d.max(initial=0) <= 1, f"max distance {d.max()} steps"


def assert_f32_within_rel(got: np.ndarray, ref: np.ndarray, mag: np.ndarray, rel=1e-5):
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert (err <= rel * mag + 1e-30).all(), f"max err/mag {np.max(err / np.maximum(mag, 1e-30))}"


def combine_magnitude(y_rows_f64: np.ndarray, w: np.ndarray) -> np.ndarray:
    """sum_j |w_j| |y_j| per output element; y_rows_f64 is [T, k, H]."""
    return np.einsum("tk,tkh->th", np.abs(w.astype(np.float64)), np.abs(y_rows_f64))
