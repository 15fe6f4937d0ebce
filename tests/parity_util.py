"""Shared helpers of the GPU parity tests: oracle calls, tolerances, sigma band.

Tolerances: fp32 compute must match the fp64 oracle within 1e-4 relative
Frobenius error, 16-bit compute within 2e-2, and every output singular value
must lie within 0.05 of the value the iteration maps the matching input
singular value to (the sigma band).

One exception, used only where a test says so: on ill-conditioned spectra no
16-bit execution of some forms can reach 2e-2 (bf16 storage of the standard
form; the naive fp16 Gram form, which the write-up calls unstable).  There the
bound is 1.25 x the error of the oracle's stored-precision iteration on the
same input (``oracle.ns_standard_stored`` / ``ns_gram_stored``, pinned in
test_oracle_pins.py), i.e. the GPU may add at most a quarter of what the
storage type's own rounding already costs.
"""
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


def emulated_output(U: np.ndarray, coeffs, mode: str, restart_after=2, chain="fp16", eps=1e-7):
    """(exact, stored) oriented outputs for the input U: the fp64 iteration, and
    the iteration with every product stored in ``chain`` (the chain's 16-bit
    type: compute_dtype for the standard form, gram_dtype for the Gram forms).
    As in the kernels, a bf16 chain starts from the raw U rounded to bf16 and
    applies f = 1 / (||U||_F + eps) inside the first products, and an fp16 chain
    starts from X0 = f U rounded once to fp16."""
    X, _ = oracle.orient(U)
    f = 1.0 / (oracle.frobenius_norm(X) + eps)
    exact_in = X * f
    exact = oracle.ns_standard(exact_in, coeffs) if mode == "standard" else oracle.ns_gram(
        exact_in, coeffs, 0 if mode == "gram" else restart_after)
    if chain == "bf16":
        start, prescale = oracle.round_to(X, "bf16"), f
    else:
        start, prescale = oracle.round_to(exact_in, chain), None
    if mode == "standard":
        emu = oracle.ns_standard_stored(start, coeffs, chain, prescale=prescale)
    else:
        ra = 0 if mode == "gram" else restart_after
        emu = oracle.ns_gram_stored(start, coeffs, chain, ra, prescale=prescale)
    return exact, emu


def emulated_floor(U: np.ndarray, coeffs, mode: str, restart_after=2, chain="fp16") -> float:
    """Relative error of a 16-bit-storage execution of the iteration on U."""
    exact, emu = emulated_output(U, coeffs, mode, restart_after, chain)
    return rel(emu, exact) if np.all(np.isfinite(emu)) else math.inf


def emulated_band_holds(U: np.ndarray, coeffs, mode: str, restart_after=2, chain="fp16") -> bool:
    """Whether the 16-bit execution itself keeps the sigma band on this input
    (the naive Gram form does not on ill-conditioned spectra: the write-up's
    float16 instability)."""
    _, emu = emulated_output(U, coeffs, mode, restart_after, chain)
    if not np.all(np.isfinite(emu)):
        return False
    Xo, tr = oracle.orient(U)
    return sigma_band_error(Xo, emu, coeffs) < SIGMA_BAND


def tolerance(compute: str, floor: float | None = None) -> float:
    """The stated bar for ``compute``; with ``floor`` (only where a test opts
    into the exception above) max(2e-2, 1.25 x floor)."""
    if compute == "fp32":
        return FP32_TOL
    if floor is None or floor <= BF16_TOL / 1.25:
        return BF16_TOL
    return 1.25 * floor


def chain_of(mode: str, compute: str = "fp16", gram_dtype: str = "fp16") -> str:
    """The storage type of a 16-bit chain (what ``emulated_floor`` takes)."""
    return compute if mode == "standard" else gram_dtype


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
