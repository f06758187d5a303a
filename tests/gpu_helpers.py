"""Shared helpers for the GPU parity tests (CUDA path vs. the fp64 oracle)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

# Tolerances on bf16 outputs against the fp64 oracle, over all outputs of a call.
MAX_ABS_TOL = 2e-2
MEAN_ABS_TOL = 2e-3

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


def device_qkv(bits: np.ndarray) -> torch.Tensor:
    """Upload packed bf16 bit patterns as a contiguous bf16 CUDA tensor (same bytes)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to("cuda").view(torch.bfloat16)


def run_cuda(bits: np.ndarray, scale: float) -> np.ndarray:
    import vit_self_attention_b200 as vab
    qkv = device_qkv(bits)
    out = vab.attention(qkv, scale)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, want: np.ndarray) -> tuple[float, float]:
    diff = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(want, dtype=np.float64))
    return float(diff.max()), float(diff.mean())


def assert_parity(got: np.ndarray, want: np.ndarray, what: str,
                  max_tol: float = MAX_ABS_TOL, mean_tol: float = MEAN_ABS_TOL) -> None:
    assert got.shape == want.shape, f"{what}: shape {got.shape} vs {want.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite outputs"
    mx, mean = errors(got, want)
    assert mx <= max_tol and mean <= mean_tol, (
        f"{what}: max|err| {mx:.3e} (tol {max_tol:.0e}), mean|err| {mean:.3e} (tol {mean_tol:.0e})")


def assert_close_bf16(got: np.ndarray, want: np.ndarray, what: str, mag=None) -> None:
    """Tolerance of a bf16 output layer derived from its arithmetic (LayerNorm, linear):
    the result is formed in fp32 (fp32 accumulation of the dot products, then bias, GELU
    and residual in the same fp32 epilogue) and rounded to bf16 once, nearest even, which
    is off by at most 2^-9 of the magnitude it rounds.  Elementwise
    |err| <= 2^-8 mag + 2^-10 (twice the rounding bound, plus a floor for outputs near
    zero where the fp32 accumulation error of up to a few thousand products is what
    remains), with mag = |want| or, with a residual, the sum of the magnitudes of the two
    terms; the mean error at most 2^-9 of the mean magnitude (plus 1e-4)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, f"{what}: shape {got.shape} vs {want.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite outputs"
    err = np.abs(got - want)
    mag = np.abs(want) if mag is None else np.asarray(mag, dtype=np.float64)
    bound = 2.0 ** -8 * mag + 2.0 ** -10
    worst = float(np.max(err - bound))
    mean_err, mean_mag = float(err.mean()), float(mag.mean())
    assert worst <= 0.0, f"{what}: an element exceeds 2^-8|y| + 2^-10 by {worst:.3e}"
    assert mean_err <= 2.0 ** -9 * mean_mag + 1e-4, (
        f"{what}: mean|err| {mean_err:.3e} vs mean|y| {mean_mag:.3e}")
