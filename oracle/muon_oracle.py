"""fp64 CPU oracle for the Muon optimizer step with Newton-Schulz orthogonalisation.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain, obviously correct
statement of what the CUDA library computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it.  The product path (``newton_schulz_matrix_b200``)
never imports, calls or links anything here, and this module shares no code with
it: the only thing both sides take is the seeded input arrays from ``synth/``.

Everything is float64 NumPy.  ``numpy.matmul`` is used as the one library
primitive (a dense product); there is no blocking, fusion or reordering beyond
the steps written out below, in the order the pages give them.

Sources (web pages, cited by title and section):

* [Moonlight] "Moonlight 16B Guide: Scalable MoE & Muon Optimizer" (aifetchly blog):
  box "Scalable Muon Optimizer Step" (steps 1-4), section "The Newton-Schulz
  Iteration for Matrix Orthogonalization", "Innovation 1: Decoupled Weight Decay
  in Muon" (update equation), "Innovation 2: Per-Parameter Update Scale
  Alignment" (s(W) = sqrt(max(d_out, d_in))), and the listing in "End-to-End
  PyTorch Implementation" (orientation m <= n, XX^T on the short side, EMA
  momentum, decay-then-step order).
* [GramNS] "Gram Newton-Schulz" news write-up (Machine Heart, m.web578.cn):
  paragraph on the standard iteration's three products (XX^T: 2mn^2, A^2: 2n^3,
  BX: 2mn^2), the Gram rewrite paragraph (iterate on the n x n matrix XX^T,
  "any odd polynomial can be written as ..."), and the stabilised variant
  paragraph (float16 Gram iteration, restart after step 2, re-initialise the
  Gram matrix).

Readings where the pages are silent or garbled:

* Normalisation is X0 = U / (||U||_F + eps) without the listing's extra sqrt(m)
  factor (the listing's cubic form needs it, the quintic coefficients do not).
* The Gram identity whose formulas were lost is read as
  a X + b (XX^T) X + c (XX^T)^2 X = (a I + b R + c R^2) X with R = XX^T, so
  X_k = Q_k X_{k-1}, R_k = Q_k R_{k-1} Q_k and X_K = (Q_K ... Q_1) X_0.
* The accumulated product is formed by left multiplication Q_acc <- Q_k Q_acc.
* "Restart after step 2" is one restart after iteration ``restart_after``
  (default 2): X <- Q_acc X0, R <- X X^T, Q_acc <- I, then continue.  The
  periodic reading ("re-initialise the Gram matrix" every few steps) is the
  option ``restart_every`` = e > 0: restarts after iterations restart_after,
  restart_after + e, restart_after + 2e, ... while they are before the last.
* Nesterov (not on the pages) is U = (1 - mu) G + mu M_new.

Parity pins: every function below is pinned by ``tests/test_oracle_pins.py``
against closed forms, an SVD routine, exact algebraic identities or values the
pages print; see that file.  The Gram FLOP counters are pinned to the products
the Gram iteration below executes (an instrumented run counts them), not to the
pages: their complexity table was lost, and only its 42-58 % band survives, as a
plausibility check.
"""
from __future__ import annotations

import math
from typing import Iterable, Sequence

import numpy as np

STANDARD = "standard"
GRAM = "gram"
GRAM_STABILIZED = "gram_stabilized"
MODES = (STANDARD, GRAM, GRAM_STABILIZED)

# The quintic coefficients every configuration uses; the cubic one is the
# listing's 1/2 X (3 I - X X^T) = 1.5 X - 0.5 (X X^T) X  [Moonlight, NS section].
QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# Storage rounding (used by the stored-precision iteration further down)
# ---------------------------------------------------------------------------
def round_to(x: np.ndarray, fmt: str | None) -> np.ndarray:
    """Round ``x`` to a storage format and back to float64.

    ``fmt`` is None (no rounding), "fp32", "bf16" (round-to-nearest-even on the
    float32 bit pattern, top 16 bits kept) or "fp16" (IEEE binary16, overflow to
    inf).
    """
    if fmt is None:
        return x
    if fmt == "fp32":
        return x.astype(np.float32).astype(np.float64)
    if fmt == "fp16":
        with np.errstate(over="ignore"):
            return x.astype(np.float16).astype(np.float64)
    if fmt == "bf16":
        f = np.ascontiguousarray(x, dtype=np.float32)
        u = f.view(np.uint32).astype(np.uint64)
        nan = np.isnan(f)
        lsb = (u >> 16) & 1
        r = ((u + 0x7FFF + lsb) >> 16) << 16
        out = (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
        out[nan] = np.nan
        return out
    raise ValueError(f"unknown format {fmt!r}")


# ---------------------------------------------------------------------------
# Step a1/a2: momentum and Nesterov blend   [Moonlight, box step 1; listing]
# ---------------------------------------------------------------------------
def momentum_update(M: np.ndarray, G: np.ndarray, mu: float) -> np.ndarray:
    """M_t = mu * M_{t-1} + (1 - mu) * G  (exponential moving average)."""
    return mu * _f64(M) + (1.0 - mu) * _f64(G)


def nesterov_blend(G: np.ndarray, M_new: np.ndarray, mu: float, nesterov: bool) -> np.ndarray:
    """The matrix that gets orthogonalised: U = (1-mu) G + mu M_new, or M_new."""
    if nesterov:
        return (1.0 - mu) * _f64(G) + mu * _f64(M_new)
    return _f64(M_new)


# ---------------------------------------------------------------------------
# Step a4: orientation   [Moonlight listing: "ensure m <= n"; GramNS: X in R^{n x m}]
# ---------------------------------------------------------------------------
def orient(U: np.ndarray) -> tuple[np.ndarray, bool]:
    """Return (X, transposed) with X short-side-first (rows <= cols)."""
    U = _f64(U)
    if U.shape[0] > U.shape[1]:
        return U.T.copy(), True
    return U.copy(), False


def unorient(X: np.ndarray, transposed: bool) -> np.ndarray:
    return X.T.copy() if transposed else X


# ---------------------------------------------------------------------------
# Step a3: Frobenius normalisation   [Moonlight, NS section step 1; listing]
# ---------------------------------------------------------------------------
def frobenius_norm(X: np.ndarray) -> float:
    X = _f64(X)
    return math.sqrt(float(np.sum(X * X)))


def frobenius_normalize(X: np.ndarray, eps: float = 1e-7) -> np.ndarray:
    """X0 = X / (||X||_F + eps)."""
    return _f64(X) / (frobenius_norm(X) + eps)


# ---------------------------------------------------------------------------
# Step a5: standard odd-polynomial Newton-Schulz   [GramNS, standard iteration]
# ---------------------------------------------------------------------------
def ns_standard(X0: np.ndarray, coeffs: Sequence[Sequence[float]]) -> np.ndarray:
    """Iterate X <- a X + (b A + c A A) X with A = X X^T, once per (a, b, c)."""
    X = _f64(X0)
    for a, b, c in coeffs:
        A = X @ X.T                 # n x n, 2 m n^2 flops
        B = b * A + c * (A @ A)     # n x n, 2 n^3 flops
        X = a * X + B @ X           # n x m, 2 m n^2 flops
    return X


# ---------------------------------------------------------------------------
# Steps a6/a7: Gram Newton-Schulz, naive and stabilised   [GramNS, Gram rewrite]
# ---------------------------------------------------------------------------
def is_restart(k: int, iters: int, restart_after: int, restart_every: int = 0) -> bool:
    """Whether the stabilised Gram iteration restarts after iteration k (1-based)."""
    if not restart_after or k >= iters or k < restart_after:
        return False
    if k == restart_after:
        return True
    return restart_every > 0 and (k - restart_after) % restart_every == 0


def ns_gram(
    X0: np.ndarray,
    coeffs: Sequence[Sequence[float]],
    restart_after: int = 0,
    trace: list | None = None,
    restart_every: int = 0,
) -> np.ndarray:
    """Gram form of the same iteration.

    R = X0 X0^T; for k = 1..K: Q = a I + b R + c R R; Q_acc <- Q Q_acc;
    if k == restart_after (and k < K): X0 <- Q_acc X0, R <- X0 X0^T, Q_acc <- I;
    elif k < K: R <- Q R Q.  Finally X = Q_acc X0.

    ``restart_after = 0`` is the naive variant, 2 the stabilised one;
    ``restart_every`` > 0 repeats the restart (see ``is_restart``).
    If ``trace`` is a list, (k, R, Q_acc, X0) is appended after each iteration
    k, with R the Gram matrix the next iteration will use.
    """
    X = _f64(X0)
    n = X.shape[0]
    eye = np.eye(n)
    R = X @ X.T
    Qacc = eye.copy()
    K = len(coeffs)
    for k, (a, b, c) in enumerate(coeffs, start=1):
        Q = a * eye + b * R + c * (R @ R)
        Qacc = Q @ Qacc
        if k == K:
            break
        if is_restart(k, K, restart_after, restart_every):
            X = Qacc @ X
            R = X @ X.T
            Qacc = eye.copy()
        else:
            R = (Q @ R) @ Q
        if trace is not None:
            trace.append((k, R.copy(), Qacc.copy(), X.copy()))
    return Qacc @ X


# ---------------------------------------------------------------------------
# The orthogonalisation as one call (orient -> normalise -> iterate -> unorient)
# ---------------------------------------------------------------------------
def newton_schulz(
    U: np.ndarray,
    coeffs: Sequence[Sequence[float]],
    mode: str = STANDARD,
    restart_after: int = 2,
    eps: float = 1e-7,
    restart_every: int = 0,
) -> np.ndarray:
    """Orthogonalise one 2-D matrix; the result has U's storage shape."""
    if mode not in MODES:
        raise ValueError(f"mode must be one of {MODES}")
    U = _f64(U)
    if U.ndim != 2:
        raise ValueError("Newton-Schulz needs a 2-D matrix")
    X, transposed = orient(U)
    X0 = frobenius_normalize(X, eps)
    if mode == STANDARD:
        X = ns_standard(X0, coeffs)
    elif mode == GRAM:
        X = ns_gram(X0, coeffs, restart_after=0)
    else:
        X = ns_gram(X0, coeffs, restart_after=restart_after, restart_every=restart_every)
    return unorient(X, transposed)


# ---------------------------------------------------------------------------
# The same iterations with 16-bit storage between the products
# ---------------------------------------------------------------------------
# The pages fix no storage precision beyond "float16" for the stabilised Gram
# variant [GramNS].  A 16-bit execution computes every product exactly enough
# (fp32 accumulation) and rounds it once, to nearest-even, when it stores it.
# The two functions below state that execution in fp64 with the rounding at
# those store points, so that the error such an execution cannot avoid on a
# given input (its floor) can be measured.  They are not the oracle the GPU
# results are graded against: ``ns_standard`` / ``ns_gram`` are.
#
# Store points, per product (f = prescale applies only while X is the raw U):
#   standard:  A = f^2 X X^T (symmetric);  B = c A A^T + b A (symmetric, only
#              if c != 0);  X = f (a X + B X), or f (a X + b (A X)) if c == 0
#   Gram:      R = f^2 X X^T (symmetric);  Q = c R R^T + b R + a I (symmetric);
#              Q_acc = Q (first after a start) or Q Q_acc;  T = Q R;
#              R = T Q (symmetric);  restart: X = f Q_acc X, R = X X^T;
#              result f Q_acc X
# A symmetric product is stored as its upper triangle mirrored onto the lower
# one (the GPU computes only that triangle).  ``fmt`` "fp64" keeps every
# product unrounded but otherwise runs the same steps.
def _stored(x: np.ndarray, fmt: str, symmetric: bool = False) -> np.ndarray:
    if symmetric:
        x = np.triu(x) + np.triu(x, 1).T
    return x if fmt == "fp64" else round_to(x, fmt)


def ns_standard_stored(X: np.ndarray, coeffs: Sequence[Sequence[float]], fmt: str,
                       prescale: float | None = None) -> np.ndarray:
    """Standard iteration with every product stored in ``fmt``.

    ``X`` is the stored input: either X0 already normalised (``prescale``
    None) or the raw oriented U, in which case the first iteration applies
    f = ``prescale`` = 1 / (||U||_F + eps) inside its stores.
    """
    X = _f64(X)
    f = 1.0 if prescale is None else float(prescale)
    for a, b, c in coeffs:
        A = _stored(f * f * (X @ X.T), fmt, symmetric=True)
        if c != 0.0:
            B = _stored(c * (A @ A.T) + b * A, fmt, symmetric=True)
            X = _stored(f * (a * X + B @ X), fmt)
        else:
            X = _stored(f * (a * X + b * (A @ X)), fmt)
        f = 1.0
    return X


def ns_gram_stored(X: np.ndarray, coeffs: Sequence[Sequence[float]], fmt: str, restart_after: int = 0,
                   prescale: float | None = None, trace: list | None = None, restart_every: int = 0) -> np.ndarray:
    """Gram iteration (naive: ``restart_after`` 0) with every product stored in
    ``fmt``; ``X`` and ``prescale`` as in ``ns_standard_stored``.  ``trace`` gets
    (k, R, Q_acc, X) after each iteration k < K, as in ``ns_gram``."""
    X = _f64(X)
    n = X.shape[0]
    eye = np.eye(n)
    f = 1.0 if prescale is None else float(prescale)
    R = _stored(f * f * (X @ X.T), fmt, symmetric=True)
    Qacc = None  # identity
    K = len(coeffs)
    for k, (a, b, c) in enumerate(coeffs, start=1):
        Q = _stored(c * (R @ R.T) + b * R + a * eye, fmt, symmetric=True)
        Qacc = Q if Qacc is None else _stored(Q @ Qacc, fmt)
        if k == K:
            break
        if is_restart(k, K, restart_after, restart_every):
            X = _stored(f * (Qacc @ X), fmt)
            f = 1.0
            R = _stored(X @ X.T, fmt, symmetric=True)
            Qacc = None
        else:
            T = _stored(Q @ R, fmt)
            R = _stored(T @ Q, fmt, symmetric=True)
        if trace is not None:
            trace.append((k, R.copy(), eye.copy() if Qacc is None else Qacc.copy(), X.copy()))
    return _stored(f * (Qacc @ X), fmt)


# ---------------------------------------------------------------------------
# Step a8: update scale and decoupled weight decay   [Moonlight, Innovations 1-2]
# ---------------------------------------------------------------------------
def update_scale(rows: int, cols: int, scale_coef: float) -> float:
    """s(W) = scale_coef * sqrt(max(d_out, d_in))."""
    return scale_coef * math.sqrt(max(rows, cols))


def apply_update(W: np.ndarray, O: np.ndarray, lr: float, weight_decay: float, scale: float) -> np.ndarray:
    """W <- (1 - lr * wd) * W - lr * scale * O   (decay first, as the listing does)."""
    return (1.0 - lr * weight_decay) * _f64(W) - lr * scale * _f64(O)


def muon_step(
    W: np.ndarray,
    G: np.ndarray,
    M: np.ndarray,
    *,
    lr: float,
    momentum: float,
    nesterov: bool,
    weight_decay: float,
    scale_coef: float,
    eps: float,
    coeffs: Sequence[Sequence[float]],
    mode: str = STANDARD,
    restart_after: int = 2,
    restart_every: int = 0,
) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One Muon step for one parameter: returns (W_new, M_new, O)."""
    M_new = momentum_update(M, G, momentum)
    U = nesterov_blend(G, M_new, momentum, nesterov)
    O = newton_schulz(U, coeffs, mode=mode, restart_after=restart_after, eps=eps, restart_every=restart_every)
    r, c = np.shape(W)
    W_new = apply_update(W, O, lr, weight_decay, update_scale(r, c, scale_coef))
    return W_new, M_new, O


# ---------------------------------------------------------------------------
# Algorithmic FLOP counters: every product counts 2 * rows * cols * K
# ---------------------------------------------------------------------------
def flops_standard_iteration(rows: int, cols: int) -> int:
    """XX^T (2mn^2) + A^2 (2n^3) + BX (2mn^2) with n = short side [GramNS cost list]."""
    n, m = min(rows, cols), max(rows, cols)
    return 2 * m * n * n + 2 * n ** 3 + 2 * m * n * n


def flops_standard(rows: int, cols: int, iters: int) -> int:
    return iters * flops_standard_iteration(rows, cols)


def flops_gram(rows: int, cols: int, iters: int, restart_after: int = 0, restart_every: int = 0) -> int:
    """Products the Gram iteration above executes (pinned to an instrumented
    run of that iteration; the pages' own complexity table was lost).

    R0 = X0 X0^T (2mn^2); per k: R^2 (2n^3), Q Q_acc (2n^3, skipped at k = 1 and
    right after a restart, where Q_acc = I); R update Q R Q (4n^3) for k < K
    unless k is a restart step, which instead costs Q_acc X0 (2mn^2) and
    X X^T (2mn^2); finally Q_acc X0 (2mn^2).
    """
    n, m = min(rows, cols), max(rows, cols)
    sq, cube = 2 * m * n * n, 2 * n ** 3
    total = sq  # R0
    fresh = True  # Q_acc == I
    for k in range(1, iters + 1):
        total += cube  # R^2
        if not fresh:
            total += cube  # Q Q_acc
        fresh = False
        if k == iters:
            break
        if is_restart(k, iters, restart_after, restart_every):
            total += 2 * sq
            fresh = True
        else:
            total += 2 * cube
    return total + sq


def flops(rows: int, cols: int, iters: int, mode: str, restart_after: int = 2, restart_every: int = 0) -> int:
    if mode == STANDARD:
        return flops_standard(rows, cols, iters)
    if mode == GRAM:
        return flops_gram(rows, cols, iters, 0)
    return flops_gram(rows, cols, iters, restart_after, restart_every)


def singular_value_map(sigma: Iterable[float], coeffs: Sequence[Sequence[float]]) -> np.ndarray:
    """Scalar form of the iteration: s <- a s + b s^3 + c s^5, once per (a, b, c)."""
    s = _f64(list(sigma))
    for a, b, c in coeffs:
        s = a * s + b * s ** 3 + c * s ** 5
    return s
