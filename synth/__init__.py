"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random matrices with the structure of the workloads
(Gaussian, low rank plus noise, Haar bases with a prescribed spectrum).  It holds
none of the optimiser's arithmetic; both the CUDA path and the fp64 oracle take
the arrays it returns as plain inputs.

Every draw goes through ``torch.Generator(device).manual_seed(seed)``, so a
matrix is a pure function of (recipe, shape, seed, device).  The CPU and CUDA
generators give different streams; parity tests therefore draw once (on the
device under test) and hand the same values to both sides.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable

import torch

QUINTIC = (3.4445, -4.7750, 2.0315)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def gaussian(rows: int, cols: int, seed: int, device="cpu", std: float = 1.0,
             dtype=torch.float32) -> torch.Tensor:
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def low_rank_plus_noise(rows: int, cols: int, rank: int, noise: float, seed: int,
                        device="cpu", dtype=torch.float32) -> torch.Tensor:
    """A (rows x rank) @ B (rank x cols) with i.i.d. N(0,1) factors, plus noise * N(0,1)."""
    g = _gen(seed, device)
    a = torch.randn(rows, rank, generator=g, device=device)
    b = torch.randn(rank, cols, generator=g, device=device)
    e = torch.randn(rows, cols, generator=g, device=device)
    return (a @ b + noise * e).to(dtype)


def haar(rows: int, cols: int, seed: int, device="cpu") -> torch.Tensor:
    """rows x cols matrix with orthonormal columns (rows >= cols), Haar distributed.

    QR of a Gaussian matrix with the signs of R's diagonal folded into Q.
    """
    assert rows >= cols
    g = _gen(seed, device)
    z = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    q, r = torch.linalg.qr(z)
    d = torch.sign(torch.diagonal(r))
    d[d == 0] = 1.0
    return q * d


def with_spectrum(rows: int, cols: int, sigma: torch.Tensor, seed: int, device="cpu",
                  dtype=torch.float32) -> torch.Tensor:
    """U_H diag(sigma) V_H^T with Haar U_H (rows x k), V_H (cols x k), k = len(sigma)."""
    k = sigma.numel()
    u = haar(rows, k, seed * 2 + 1, device)
    v = haar(cols, k, seed * 2 + 2, device)
    return ((u * sigma.to(device=device, dtype=torch.float32)) @ v.T).to(dtype)


def power_law_sigma(k: int, exponent: float = -1.0) -> torch.Tensor:
    """sigma_i = i ** exponent, i = 1..k (sigma_1 = 1)."""
    i = torch.arange(1, k + 1, dtype=torch.float64)
    return (i ** exponent).to(torch.float32)


def log_uniform_sigma(k: int, lo: float, hi: float, seed: int) -> torch.Tensor:
    g = _gen(seed, "cpu")
    u = torch.rand(k, generator=g, dtype=torch.float64)
    return torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))).to(torch.float32)


# ---------------------------------------------------------------------------
# Workload recipes (shapes and value structure of the five configurations)
# ---------------------------------------------------------------------------
@dataclass
class Group:
    """``count`` parameters of storage shape rows x cols with their tensors."""
    rows: int
    cols: int
    W: list = field(default_factory=list)
    G: list = field(default_factory=list)
    M: list = field(default_factory=list)

    @property
    def count(self) -> int:
        return len(self.W)


@dataclass
class Workload:
    name: str
    groups: list
    hp: dict


def default_hparams(**over) -> dict:
    hp = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, scale_coef=0.2,
              eps=1e-7, coeffs=[QUINTIC] * 5, mode="standard", restart_after=2)
    hp.update(over)
    return hp


def _seed(cfg: int, idx: int, salt: int = 0) -> int:
    return cfg * 1000 + idx + 7919 * salt


def single_fp32(device="cpu") -> Workload:
    """One 64 x 128 fp32 parameter: W, G ~ N(0,1), M = 0."""
    g = Group(64, 128)
    g.W.append(gaussian(64, 128, _seed(1, 0, 1), device))
    g.G.append(gaussian(64, 128, _seed(1, 0, 2), device))
    g.M.append(torch.zeros(64, 128, device=device))
    return Workload("single-64x128-fp32", [g], default_hparams(compute_dtype="fp32"))


def dense_projection(count=64, rows=1024, cols=4096, device="cpu", dtype=torch.bfloat16) -> Workload:
    """count x (rows x cols): G = rank-64 Gaussian product + 0.1 N(0,1); W ~ N(0,1); M = 0."""
    g = Group(rows, cols)
    for i in range(count):
        g.W.append(gaussian(rows, cols, _seed(2, i, 1), device, dtype=dtype))
        g.G.append(low_rank_plus_noise(rows, cols, 64, 0.1, _seed(2, i, 2), device, dtype=dtype))
        g.M.append(torch.zeros(rows, cols, device=device))
    return Workload(f"dense-{count}x{rows}x{cols}", [g], default_hparams())


def moe_layer(experts=64, device="cpu", dtype=torch.bfloat16, shared=4, inter=1408, hidden=2048) -> Workload:
    """experts x {up, gate} (inter x hidden) + experts x down (hidden x inter) + shared hidden^2.

    Gradients have sigma_i = 1/i on Haar bases; M = 0; W ~ N(0, 0.02^2).
    """
    groups = []
    specs = [(inter, hidden, 2 * experts), (hidden, inter, experts), (hidden, hidden, shared)]
    idx = 0
    for rows, cols, count in specs:
        g = Group(rows, cols)
        for _ in range(count):
            k = min(rows, cols)
            g.G.append(with_spectrum(rows, cols, power_law_sigma(k), _seed(3, idx, 2), device, dtype))
            g.W.append(gaussian(rows, cols, _seed(3, idx, 1), device, std=0.02, dtype=dtype))
            g.M.append(torch.zeros(rows, cols, device=device))
            idx += 1
        groups.append(g)
    return Workload(f"moe-{experts}e", groups, default_hparams())


def kimi_k2(experts=216, dense=1, device="cpu", dtype=torch.bfloat16, counts=None) -> Workload:
    """Kimi-K2-shaped set: experts x {up, gate} stored 2048 x 7168, experts x down
    stored 7168 x 2048, dense x {up, gate} stored 18432 x 7168 and dense x down
    stored 7168 x 18432 (all orient to 2048 x 7168 or 7168 x 18432).

    M_prev = rank-64 Gaussian product + 0.1 noise rescaled to entry std 1e-3;
    G ~ N(0, 1e-3^2); W ~ N(0, 0.02^2).  ``counts`` optionally overrides the
    number of matrices per storage group (used for sampled checks).
    """
    specs = [(2048, 7168, 2 * experts), (7168, 2048, experts),
             (18432, 7168, 2 * dense), (7168, 18432, dense)]
    if counts is not None:
        specs = [(r, c, n) for (r, c, _), n in zip(specs, counts)]
    groups = []
    idx = 0
    for rows, cols, count in specs:
        if count == 0:
            continue
        g = Group(rows, cols)
        for _ in range(count):
            m = low_rank_plus_noise(rows, cols, 64, 0.1, _seed(4, idx, 3), device)
            m.mul_(1e-3 / m.std())
            g.M.append(m)
            g.G.append(gaussian(rows, cols, _seed(4, idx, 2), device, std=1e-3, dtype=dtype))
            g.W.append(gaussian(rows, cols, _seed(4, idx, 1), device, std=0.02, dtype=dtype))
            idx += 1
        groups.append(g)
    return Workload(f"kimi-k2-{experts}e", groups, default_hparams())


def stress_point(n: int, alpha: int, count=32, device="cpu", dtype=torch.bfloat16) -> list:
    """count matrices n x (alpha n) with log-uniform sigma in [1e-6, 1] on Haar bases."""
    out = []
    for i in range(count):
        s = log_uniform_sigma(n, 1e-6, 1.0, _seed(5, i, n + alpha))
        out.append(with_spectrum(n, alpha * n, s, _seed(5, i, 31 * n + alpha), device, dtype))
    return out
