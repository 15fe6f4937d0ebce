"""Shared helpers of the GPU parity tests: oracle calls, tolerances, sigma band.

Tolerance rule (derived from the arithmetic; the numbers behind it are in the
design notes): fp32 compute must match the fp64 oracle within 1e-4 relative
Frobenius error.  bf16/fp16 compute must match within 2e-2, or within 1.25 x the
error that the oracle's own storage-rounding emulation shows on the same input
when that floor is above 1.6e-2 (ill-conditioned spectra, where any 16-bit
execution mixes singular vectors of nearly equal singular values); and in both
cases every output singular value must lie within 0.05 of the value the
iteration maps the matching input singular value to (the sigma band).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

Q5 = [oracle.QUINTIC] * 5
FP32_TOL = 1e-4
BF16_TOL = 2e-2
SIGMA_BAND = 0.05


def rel(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def emulated_output(U: np.ndarray, coeffs, mode: str, restart_after=2, gram_fmt="fp16", x_fmt="bf16"):
    """(exact, emulated) oriented outputs: the iteration in fp64 and with every
    stored matrix rounded to its 16-bit storage type (oracle emulation)."""
    X, _ = oracle.orient(U)
    X0 = oracle.frobenius_normalize(X)
    exact = oracle.ns_standard(X0, coeffs)
    if mode == "standard":
        emu = oracle.ns_standard(oracle.round_to(X0, x_fmt), coeffs, emulate=x_fmt)
    else:
        x_fmt = gram_fmt  # the Gram chain stores X0 and the restart X in the Gram type too
        ra = 0 if mode == "gram" else restart_after
        emu = oracle.ns_gram(oracle.round_to(X0, x_fmt), coeffs, ra, emulate_gram=gram_fmt, emulate_x=x_fmt)
    return exact, emu


def emulated_floor(U: np.ndarray, coeffs, mode: str, restart_after=2, gram_fmt="fp16", x_fmt="bf16") -> float:
    """Relative error of a 16-bit-storage execution of the iteration (oracle emulation)."""
    exact, emu = emulated_output(U, coeffs, mode, restart_after, gram_fmt, x_fmt)
    return rel(emu, exact) if np.all(np.isfinite(emu)) else math.inf


def emulated_band_holds(U: np.ndarray, coeffs, mode: str, restart_after=2, gram_fmt="fp16") -> bool:
    """Whether the 16-bit execution itself keeps the sigma band on this input
    (the naive Gram form does not on ill-conditioned spectra: the write-up's
    float16 instability)."""
    _, emu = emulated_output(U, coeffs, mode, restart_after, gram_fmt)
    if not np.all(np.isfinite(emu)):
        return False
    Xo, tr = oracle.orient(U)
    return sigma_band_error(Xo, emu, coeffs) < SIGMA_BAND


def tolerance(compute: str, floor: float | None = None) -> float:
    if compute == "fp32":
        return FP32_TOL
    if floor is None or floor <= BF16_TOL / 1.25:
        return BF16_TOL
    return 1.25 * floor


def sigma_band_error(U: np.ndarray | torch.Tensor, O: np.ndarray | torch.Tensor, coeffs, eps=1e-7) -> float:
    """max |sigma_i(O) - f^K(sigma_i(U) / (||U||_F + eps))| over sorted singular values.

    Accepts numpy (LAPACK SVD on the host) or CUDA tensors (torch SVD on the
    device, fp64 for n <= 2048 else fp32) so it can run at any size."""
    if isinstance(U, torch.Tensor):
        dt = torch.float64 if min(U.shape) <= 2048 else torch.float32
        su = torch.linalg.svdvals(U.to(dt))
        so = torch.linalg.svdvals(O.to(dt))
        t = (su / (torch.sqrt(torch.sum(su.double() ** 2)).to(dt) + eps)).double().cpu().numpy()
        so = so.double().cpu().numpy()
    else:
        su = np.linalg.svd(U, compute_uv=False)
        so = np.linalg.svd(O, compute_uv=False)
        t = su / (math.sqrt(float(np.sum(su * su))) + eps)
    pred = np.sort(oracle.singular_value_map(t, coeffs))
    return float(np.max(np.abs(np.sort(so) - pred)))
