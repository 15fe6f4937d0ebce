"""Parity at the workloads' full sizes: every matrix of a workload runs on the
GPU in one call (the launch configuration the bench uses), and sampled matrices
are checked against the fp64 oracle one by one; matrices too large for the
oracle (7168 x 18432, n >= 2048 stress points) are checked through properties
that hold at any size (the sigma band, finiteness, status words).
"""
import math

import numpy as np
import pytest
import torch

import newton_schulz_matrix_b200 as nsm
import oracle
import synth
from parity_util import Q5, chain_of, emulated_band_holds, emulated_floor, rel, sigma_band_error, to_np, tolerance

pytestmark = pytest.mark.gpu
DEV = "cuda"
BENCH_WS = 24 << 30  # the workspace cap bench.py uses


@pytest.fixture(autouse=True)
def _free():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def sigma_band_gpu(U: torch.Tensor, O: torch.Tensor, coeffs=Q5, eps=1e-7) -> float:
    """sigma band through fp64 Gram eigenvalues on the device (any size)."""
    def svals(X):
        X = X.double()
        if X.shape[0] > X.shape[1]:
            X = X.T
        ev = torch.linalg.eigvalsh(X @ X.T).clamp_min(0)
        return torch.sqrt(ev).cpu().numpy()
    su = svals(U)
    so = svals(O)
    t = su / (math.sqrt(float(np.sum(su * su))) + eps)
    pred = np.sort(oracle.singular_value_map(t, coeffs))
    return float(np.max(np.abs(np.sort(so) - pred)))


def step_hp(**kw):
    hp = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, scale_coef=0.2, eps=1e-7, coeffs=Q5)
    hp.update(kw)
    return hp


def run_step(params, grads, moms, ws_bytes=None, **hp):
    st = nsm.MuonStep(params, grads, moms, workspace_bytes=ws_bytes, **hp)
    st()
    torch.cuda.synchronize()
    status = st.status_in_param_order().cpu()
    del st
    return status


def check_sample_fp32_w(W0, W1, G, M0, M1, hp, mode, compute="fp16"):
    """O recovered exactly from an fp32 W update; checked against the oracle.

    The standard form on the default fp16 chain is held to the stated 2e-2.
    The Gram forms (and any bf16 chain) are held to max(2e-2, 1.25 x the
    floor of their 16-bit storage on this input): on the dense recipe the fp16
    Gram chain's own rounding already costs 2.1e-2 (stabilised) and 4.3e-2
    (naive), on the 1/i spectrum the naive form reaches 0.13."""
    r, c = W0.shape
    Wr, Mr, Or = oracle.muon_step(W0, G, M0, mode=mode, restart_after=2, **hp)
    assert rel(M1, Mr) < 1e-6
    step = hp["lr"] * hp["scale_coef"] * math.sqrt(max(r, c))
    O = ((1 - hp["lr"] * hp["weight_decay"]) * W0 - W1) / step
    U = oracle.nesterov_blend(G, Mr, hp["momentum"], hp["nesterov"])
    err = rel(O, Or)
    strict = mode == "standard" and compute != "bf16"
    floor = None if strict else emulated_floor(U, hp["coeffs"], mode, chain=chain_of(mode, compute))
    assert err < tolerance(compute, floor), (err, floor)
    if emulated_band_holds(U, hp["coeffs"], mode, chain=chain_of(mode, compute)):
        assert sigma_band_error(U, O, hp["coeffs"]) < 0.05
    return err, floor


# ---------------------------------------------------------------------------
# 64 x 1024 x 4096 dense projections (rank-64 + noise gradients)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("mode,compute", [("standard", "fp16"), ("gram", "fp16"), ("gram_stabilized", "fp16"),
                                          ("standard", "bf16")])
def test_dense_projection_batch(mode, compute):
    w = synth.dense_projection(device=DEV)
    g = w.groups[0]
    params = [x.float() for x in g.W]   # fp32 W so that O is observable exactly
    W0 = [to_np(p) for p in params[:2]]
    M0 = [to_np(m) for m in g.M[:2]]
    hp = step_hp()
    status = run_step(params, g.G, g.M, mode=mode, compute_dtype=compute, **hp)
    assert int((status != 0).sum()) == 0
    for i in range(2):
        check_sample_fp32_w(W0[i], to_np(params[i]), to_np(g.G[i]), M0[i], to_np(g.M[i]), hp, mode, compute)


# ---------------------------------------------------------------------------
# MoE layer: 64 experts x {up, gate, down} + 4 shared 2048^2, grouped step
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("mode", ["standard", "gram", "gram_stabilized"])
def test_moe_layer_grouped_step(mode):
    w = synth.moe_layer(device=DEV)
    params, grads, moms, samples = [], [], [], []
    for g in w.groups:
        samples.append(len(params))
        params += [x.float() for x in g.W]
        grads += g.G
        moms += g.M
    W0 = {i: to_np(params[i]) for i in samples}
    M0 = {i: to_np(moms[i]) for i in samples}
    hp = step_hp()
    status = run_step(params, grads, moms, mode=mode, **hp)
    assert int((status != 0).sum()) == 0
    for i in samples:
        check_sample_fp32_w(W0[i], to_np(params[i]), to_np(grads[i]), M0[i], to_np(moms[i]), hp, mode)


# ---------------------------------------------------------------------------
# Kimi-K2 set, exactly as the bench runs it (bf16 W, 24 GiB workspace)
# ---------------------------------------------------------------------------
def test_kimi_k2_full_step_as_benchmarked():
    w = synth.kimi_k2(device=DEV)
    params, grads, moms = [], [], []
    firsts = []
    for g in w.groups:
        firsts.append(len(params))
        params += g.W
        grads += g.G
        moms += g.M
    experts = [firsts[0], firsts[1]]          # one wide and one tall expert matrix
    dense = firsts[2]                         # one 18432 x 7168 dense matrix
    keep = experts + [dense]
    W0 = {i: params[i].clone() for i in keep}
    M0 = {i: moms[i].clone() for i in keep}
    hp = step_hp()
    status = run_step(params, grads, moms, ws_bytes=BENCH_WS, mode="standard", **hp)
    assert int((status != 0).sum()) == 0
    decay = 1 - hp["lr"] * hp["weight_decay"]
    for i in experts:
        r, c = params[i].shape
        step = hp["lr"] * hp["scale_coef"] * math.sqrt(max(r, c))
        Wr, Mr, Or = oracle.muon_step(to_np(W0[i]), to_np(grads[i]), to_np(M0[i]), mode="standard", **hp)
        assert rel(to_np(moms[i]), Mr) < 1e-6
        # the bf16 W store quantises the update: measure that part on the oracle's own result
        dW_ref = Wr - to_np(W0[i])
        q = rel(oracle.round_to(Wr, "bf16") - to_np(W0[i]), dW_ref)
        dW = to_np(params[i]) - to_np(W0[i])
        U = oracle.nesterov_blend(to_np(grads[i]), Mr, hp["momentum"], True)
        # the orthogonalisation is held to the stated 2e-2; the bf16 store of W
        # adds its own, independent quantisation q of the update on top
        assert rel(dW, dW_ref) < math.hypot(2e-2, q), (rel(dW, dW_ref), q)
        assert sigma_band_error(U, -(dW - (decay - 1) * to_np(W0[i])) / step, Q5) < 0.05
    # dense matrix: sigma band at full size on the device
    i = dense
    r, c = params[i].shape
    step = hp["lr"] * hp["scale_coef"] * math.sqrt(max(r, c))
    Mn = hp["momentum"] * M0[i] + (1 - hp["momentum"]) * grads[i].float()
    assert float((moms[i] - Mn).norm() / Mn.norm()) < 1e-6
    U = (1 - hp["momentum"]) * grads[i].float() + hp["momentum"] * Mn
    O = (decay * W0[i].float() - params[i].float()) / step
    assert sigma_band_gpu(U, O) < 0.05


def test_kimi_k2_subset_stabilized_gram():
    w = synth.kimi_k2(device=DEV, counts=[8, 4, 1, 0])
    params, grads, moms, firsts = [], [], [], []
    for g in w.groups:
        firsts.append(len(params))
        params += [x.float() for x in g.W]
        grads += g.G
        moms += g.M
    i = firsts[0]
    W0, M0 = to_np(params[i]), to_np(moms[i])
    d = firsts[2]
    Wd0, Md0 = params[d].clone(), moms[d].clone()
    hp = step_hp()
    status = run_step(params, grads, moms, ws_bytes=BENCH_WS, mode="gram_stabilized", **hp)
    assert int((status != 0).sum()) == 0
    check_sample_fp32_w(W0, to_np(params[i]), to_np(grads[i]), M0, to_np(moms[i]), hp, "gram_stabilized")
    r, c = params[d].shape
    step = hp["lr"] * hp["scale_coef"] * math.sqrt(max(r, c))
    Mn = hp["momentum"] * Md0 + (1 - hp["momentum"]) * grads[d].float()
    U = (1 - hp["momentum"]) * grads[d].float() + hp["momentum"] * Mn
    O = ((1 - hp["lr"] * hp["weight_decay"]) * Wd0 - params[d]) / step
    assert sigma_band_gpu(U, O) < 0.05


# ---------------------------------------------------------------------------
# stress sweep: log-uniform spectra in [1e-6, 1], all twelve (n, alpha) points
# ---------------------------------------------------------------------------
STRESS_POINTS = [(n, a) for n in (1024, 2048, 4096) for a in (1, 2, 4, 8)]


@pytest.mark.parametrize("n,alpha", STRESS_POINTS)
def test_stress_sweep(n, alpha):
    """Every form on 32 ill-conditioned matrices (default fp16 chains): no
    Inf/NaN in the standard or stabilised form, the sigma band on the device
    (fp64 Gram eigenvalues) for matrix 0 at every size, and matrix 0 against
    the fp64 oracle up to n = 2048 (at n = 4096 the oracle takes minutes per
    matrix; the same recipe is checked against it at n = 1024 and 2048).  The
    standard and stabilised forms meet the stated 2e-2; the naive Gram form is
    held to 1.25 x its own fp16 floor (the write-up's instability)."""
    mats = synth.stress_point(n, alpha, count=32, device=DEV)
    U0 = to_np(mats[0]) if n <= 2048 else None
    for mode in ("standard", "gram", "gram_stabilized"):
        ys = [m.clone() for m in mats]
        st = torch.full((32,), -1, dtype=torch.int32, device=DEV)
        nsm.muon_ns_batched(ys, mode=mode, status=st)
        torch.cuda.synchronize()
        flags = st.cpu().numpy()
        if mode != "gram":
            assert int((flags != 0).sum()) == 0  # no Inf/NaN in the standard or stabilised form
        if not torch.isfinite(ys[0]).all():
            # the fp16 naive Gram form may overflow on this spectrum (the write-up's Inf): then
            # the status word must say so
            assert mode == "gram" and flags[0] == 1
            continue
        assert flags[0] == 0
        assert sigma_band_gpu(mats[0], ys[0]) < 0.05, mode
        if U0 is None:
            continue
        want = oracle.newton_schulz(U0, Q5, mode=mode)
        floor = emulated_floor(U0, Q5, mode) if mode == "gram" else None
        assert rel(to_np(ys[0]), want) < tolerance("fp16", floor), (mode, rel(to_np(ys[0]), want), floor)
        del ys


# ---------------------------------------------------------------------------
# fp16 storage for the standard form meets the stated 2e-2 outright
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("workload", ["dense", "kimi-k2-subset"])
def test_fp16_standard_meets_the_stated_tolerance(workload):
    if workload == "dense":
        w = synth.dense_projection(device=DEV, count=16)
    else:
        w = synth.kimi_k2(device=DEV, counts=[6, 3, 0, 0])
    params, grads, moms, samples = [], [], [], []
    for g in w.groups:
        samples.append(len(params))
        params += [x.float() for x in g.W]
        grads += g.G
        moms += g.M
    W0 = {i: to_np(params[i]) for i in samples}
    M0 = {i: to_np(moms[i]) for i in samples}
    hp = step_hp()
    status = run_step(params, grads, moms, mode="standard", compute_dtype="fp16", **hp)
    assert int((status != 0).sum()) == 0
    for i in samples:
        r, c = params[i].shape
        Wr, Mr, Or = oracle.muon_step(W0[i], to_np(grads[i]), M0[i], mode="standard", **hp)
        step = hp["lr"] * hp["scale_coef"] * math.sqrt(max(r, c))
        O = ((1 - hp["lr"] * hp["weight_decay"]) * W0[i] - to_np(params[i])) / step
        assert rel(O, Or) < 2e-2
        U = oracle.nesterov_blend(to_np(grads[i]), Mr, hp["momentum"], True)
        assert sigma_band_error(U, O, Q5) < 0.05
