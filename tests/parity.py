"""Comparison helpers shared by the GPU parity tests and the smoke check.

Tolerances (the stated bar for this operation):
  * fp32 output: normwise relative error per (b, n, h) row of length d at most
    1e-4 against the fp64 oracle; a row whose oracle value is exactly 0 (phi(Q)
    = 0) must be exactly 0.
  * bf16 output: elementwise |err| <= 2^-7 |ref| + 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

FP32_ROW_RTOL = 1e-4
BF16_RTOL = 2.0 ** -7
BF16_ATOL = 1e-3


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def check_output(O_gpu: torch.Tensor, O_ref: np.ndarray, what: str = ""):
    """Raise AssertionError unless O_gpu meets the tolerance for its dtype."""
    got = to_f64(O_gpu)
    assert got.shape == O_ref.shape, (got.shape, O_ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    zero = np.linalg.norm(O_ref, axis=-1) == 0
    if O_gpu.dtype == torch.float32:
        err = np.linalg.norm(got - O_ref, axis=-1)
        ref = np.linalg.norm(O_ref, axis=-1)
        rel = np.where(zero, 0.0, err / np.where(zero, 1.0, ref))
        worst = np.unravel_index(np.argmax(rel), rel.shape)
        assert rel.max() <= FP32_ROW_RTOL, \
            f"{what}: max row rel err {rel.max():.3e} at {worst} > {FP32_ROW_RTOL}"
    else:
        bound = BF16_RTOL * np.abs(O_ref) + BF16_ATOL
        excess = np.abs(got - O_ref) - bound
        worst = np.unravel_index(np.argmax(excess), excess.shape)
        assert excess.max() <= 0, \
            f"{what}: bf16 error exceeds bound by {excess.max():.3e} at {worst}"
    assert np.all(got[zero] == 0.0), f"{what}: rows with phi(Q)=0 are not exactly 0"


def head_slice(t: torch.Tensor, heads) -> np.ndarray:
    """(B, N, len(heads), d) fp64 copy of the given heads."""
    return to_f64(t[:, :, list(heads), :].contiguous())
