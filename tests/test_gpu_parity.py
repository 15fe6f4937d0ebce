"""CUDA path vs the fp64 oracle, element by element, at sizes the oracle runs in
seconds (several 128 x 256 tiles, ragged tails, tall and wide matrices) plus the
edge cases of the method.  Everything goes through the C ABI (ctypes binding).
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
SHAPES = [(64, 128), (128, 256), (200, 328), (328, 200), (130, 520), (256, 1024), (384, 384), (1, 40), (40, 1)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nsm.load_library()


def gpu_ns(mats, **kw):
    ys = [m.clone() for m in mats]
    st = torch.full((len(ys),), -1, dtype=torch.int32, device=DEV)
    nsm.muon_ns_batched(ys, status=st, **kw)
    torch.cuda.synchronize()
    return ys, st.cpu().tolist()


# ---------------------------------------------------------------------------
# single products: one iteration with (a, b, c) = unit vectors isolates
#   a X  (pack + norm + epilogue C term),  b (X X^T) X  (SYRK + MN-major product),
#   c (X X^T)^2 X  (SYRK of a symmetric operand)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(128, 256), (200, 328), (328, 200), (130, 520), (257, 1031)])
@pytest.mark.parametrize("abc", [(1.0, 0.0, 0.0), (0.0, 1.0, 0.0), (0.0, 0.0, 1.0), (0.5, -0.25, 2.0)])
@pytest.mark.parametrize("compute", ["bf16", "fp16", "fp32"])
def test_single_iteration_products(shape, abc, compute):
    """One product at a time.  The fp16 chain skips the isolated (X X^T)^2 X:
    on a normalised X it is of order sigma^5 (~1e-5 here), below fp16's normal
    range, so its relative error measures fp16's subnormal spacing rather than
    the kernels (in the full iteration the c term is added to a X + b A X and
    the singular values grow towards 1); the sigma^3 term is partly subnormal
    too, hence 5e-3 rather than the ~1e-3 of two fp16 roundings."""
    if compute == "fp16" and abc == (0.0, 0.0, 1.0):
        pytest.skip("isolated sigma^5 term lies in fp16's subnormal range")
    dtype = torch.float32 if compute == "fp32" else torch.bfloat16
    X = synth.gaussian(*shape, seed=shape[0] * 7 + 1, device=DEV, dtype=dtype)
    (Y,), st = gpu_ns([X], coeffs=[abc], compute_dtype=compute)
    want = oracle.newton_schulz(to_np(X), [abc])
    err = rel(to_np(Y), want)
    assert st == [0]
    # one product: inputs and result each rounded once to the storage type
    assert err < {"fp32": 1e-5, "fp16": 5e-3, "bf16": 8e-3}[compute], err


# ---------------------------------------------------------------------------
# full five-iteration quintic NS, all three forms, batched
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mode", ["standard", "gram", "gram_stabilized"])
@pytest.mark.parametrize("compute", ["fp16", "bf16", "fp32"])
def test_ns_batched_vs_oracle(shape, mode, compute):
    """fp32 and the default fp16 chain meet the stated bars outright; the bf16
    chain is held to its storage type's own floor (at most 1.25 x it)."""
    dtype = torch.float32 if compute == "fp32" else torch.bfloat16
    mats = [synth.gaussian(*shape, seed=100 + i + shape[0], device=DEV, dtype=dtype) for i in range(3)]
    ys, st = gpu_ns(mats, mode=mode, compute_dtype=compute)
    assert st == [0, 0, 0]
    for x, y in zip(mats, ys):
        U = to_np(x)
        want = oracle.newton_schulz(U, Q5, mode=mode)
        floor = emulated_floor(U, Q5, mode, chain=chain_of(mode, compute)) if compute == "bf16" else None
        err = rel(to_np(y), want)
        assert err < tolerance(compute, floor), (err, floor)
        if min(shape) > 1:
            assert sigma_band_error(U, to_np(y), Q5) < 0.05


@pytest.mark.parametrize("mode", ["standard", "gram", "gram_stabilized"])
def test_spectrum_inputs_and_sigma_band(mode):
    """Power-law spectrum on Haar bases (the MoE recipe), 256 x 1024, default
    fp16 chain: the stated 2e-2 except for the naive Gram form, which the
    write-up calls unstable in float16 (held to its own floor)."""
    U = synth.with_spectrum(256, 1024, synth.power_law_sigma(256), 5, device=DEV).bfloat16()
    (y,), st = gpu_ns([U], mode=mode)
    Un = to_np(U)
    want = oracle.newton_schulz(Un, Q5, mode=mode)
    floor = emulated_floor(Un, Q5, mode) if mode == "gram" else None
    assert st == [0]
    assert rel(to_np(y), want) < tolerance("fp16", floor)
    if emulated_band_holds(Un, Q5, mode):
        assert sigma_band_error(Un, to_np(y), Q5) < 0.05
    else:
        # naive fp16 Gram on a 1/i spectrum: the method itself leaves the band
        # (negative Gram eigenvalues amplified each step); the GPU must show it too
        assert mode == "gram"
        assert sigma_band_error(Un, to_np(y), Q5) > 0.05


def test_other_coefficient_schedules_and_restart_points():
    X = synth.gaussian(200, 600, seed=3, device=DEV, dtype=torch.bfloat16)
    U = to_np(X)
    sched = [(3.0, -3.2, 1.2), (2.5, -2.0, 0.6), oracle.QUINTIC, (1.5, -0.5, 0.0), (1.9, -1.3, 0.4), oracle.QUINTIC]
    for mode, ra in [("standard", 2), ("gram", 2), ("gram_stabilized", 1), ("gram_stabilized", 3), ("gram_stabilized", 5)]:
        (y,), st = gpu_ns([X], coeffs=sched, mode=mode, restart_after=ra)
        want = oracle.newton_schulz(U, sched, mode=mode, restart_after=ra)
        assert st == [0]
        assert rel(to_np(y), want) < 2e-2, (mode, ra)


@pytest.mark.parametrize("compute,shape", [("fp16", (200, 600)), ("bf16", (300, 900)), ("fp32", (64, 160)),
                                           ("fp32", (300, 700))])
@pytest.mark.parametrize("ra,every", [(2, 2), (1, 1), (1, 3)])
def test_periodic_restarts(compute, shape, ra, every):
    """The stabilised form restarted after iteration ra and every `every`
    iterations after it (six quintic iterations): the result matches the
    oracle's, and the products the library launches add up to the oracle's
    FLOP count for exactly those restarts (each restart is a pair of
    rectangular products that a single restart would not run)."""
    dtype = torch.float32 if compute == "fp32" else torch.bfloat16
    X = synth.gaussian(*shape, seed=17 + ra + 5 * every, device=DEV, dtype=dtype)
    coeffs = [oracle.QUINTIC] * 6
    nsm.muon_profile_begin()
    (y,), st = gpu_ns([X], coeffs=coeffs, mode="gram_stabilized", restart_after=ra, restart_every=every,
                      compute_dtype=compute)
    prof = nsm.muon_profile_end()
    assert st == [0]
    want = oracle.newton_schulz(to_np(X), coeffs, mode="gram_stabilized", restart_after=ra, restart_every=every)
    assert rel(to_np(y), want) < tolerance(compute), (compute, rel(to_np(y), want))
    launched = sum(r["flops"] for r in prof if r["kernel"] not in ("pack_kernel", "norm_kernel", "unpack_kernel"))
    assert launched == pytest.approx(oracle.flops(*shape, 6, "gram_stabilized", ra, every), rel=1e-12)
    assert launched != pytest.approx(oracle.flops(*shape, 6, "gram_stabilized", ra, 0), rel=1e-6)


def test_gram_dtype_bf16_option():
    X = synth.gaussian(256, 768, seed=4, device=DEV, dtype=torch.bfloat16)
    for mode in ("gram", "gram_stabilized"):
        (y,), st = gpu_ns([X], mode=mode, gram_dtype="bf16")
        want = oracle.newton_schulz(to_np(X), Q5, mode=mode)
        assert st == [0]
        assert rel(to_np(y), want) < tolerance("bf16", emulated_floor(to_np(X), Q5, mode, chain="bf16"))


# ---------------------------------------------------------------------------
# configuration 1: one 64 x 128 fp32 Muon step; 40 cubic steps = polar factor
# ---------------------------------------------------------------------------
def test_fp32_single_matrix_step():
    w = synth.single_fp32(device=DEV)
    g = w.groups[0]
    hp = w.hp
    W0 = g.W[0].clone()
    W, G, M = g.W[0], g.G[0], g.M[0]
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    nsm.muon_step([W], [G], [M], status=st, compute_dtype="fp32", lr=hp["lr"], momentum=hp["momentum"],
                  nesterov=hp["nesterov"], weight_decay=hp["weight_decay"], scale_coef=hp["scale_coef"])
    torch.cuda.synchronize()
    Wr, Mr, Or = oracle.muon_step(to_np(W0), to_np(G), np.zeros((64, 128)), lr=0.02, momentum=0.95, nesterov=True,
                                  weight_decay=0.1, scale_coef=0.2, eps=1e-7, coeffs=Q5)
    assert st.item() == 0
    assert rel(to_np(M), Mr) < 1e-6
    assert rel(to_np(W), Wr) < 1e-4
    step = 0.02 * 0.2 * math.sqrt(128)
    O_gpu = ((1 - 0.02 * 0.1) * to_np(W0) - to_np(W)) / step
    assert rel(O_gpu, Or) < 1e-4


def test_fp32_cubic_40_steps_is_polar_factor():
    g = synth.single_fp32(device=DEV).groups[0]
    (y,), st = gpu_ns([g.G[0]], coeffs=[oracle.CUBIC] * 40, compute_dtype="fp32")
    P, s, Vt = np.linalg.svd(to_np(g.G[0]), full_matrices=False)
    assert st == [0]
    assert rel(to_np(y), P @ Vt) < 1e-4


# ---------------------------------------------------------------------------
# fp32 chains of small matrices run as one fused launch (one CTA per matrix,
# the whole chain in shared memory): ragged sizes below and across the 16 x 16
# thread grid and the 64 x 64 output tile, batches wider than the SM count, and
# a schedule longer than the fused kernel's coefficient table (chained products)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(37, 53), (17, 200), (100, 64), (64, 65), (90, 91)])
@pytest.mark.parametrize("mode", ["standard", "gram", "gram_stabilized"])
def test_fp32_small_matrix_chain(shape, mode):
    mats = [synth.gaussian(*shape, seed=500 + i + shape[0], device=DEV) for i in range(3)]
    ys, st = gpu_ns(mats, mode=mode, compute_dtype="fp32")
    assert st == [0, 0, 0]
    for x, y in zip(mats, ys):
        U = to_np(x)
        assert rel(to_np(y), oracle.newton_schulz(U, Q5, mode=mode)) < 1e-4


def test_fp32_small_matrix_chain_wide_batch_and_long_schedule():
    mats = [synth.gaussian(48, 96, seed=900 + i, device=DEV) for i in range(300)]
    ys, st = gpu_ns(mats, compute_dtype="fp32")
    assert st == [0] * 300
    for i in (0, 147, 148, 299):
        assert rel(to_np(ys[i]), oracle.newton_schulz(to_np(mats[i]), Q5)) < 1e-4
    coeffs = [oracle.CUBIC] * 70
    (y,), st = gpu_ns(mats[:1], coeffs=coeffs, compute_dtype="fp32")
    assert st == [0]
    assert rel(to_np(y), oracle.newton_schulz(to_np(mats[0]), coeffs)) < 1e-4


# ---------------------------------------------------------------------------
# fp32 chains with n >= 256 run on the tensor cores as 3xTF32 (hi/lo split of
# every operand): ragged 256-tiles, tall and wide, all three forms at the fp32
# bar; symmetric products come out exactly symmetric (mirrored upper triangle)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(300, 700), (520, 260), (640, 640), (256, 2056)])
@pytest.mark.parametrize("mode", ["standard", "gram", "gram_stabilized"])
def test_fp32_tensor_core_chain(shape, mode):
    mats = [synth.gaussian(*shape, seed=700 + i + shape[0], device=DEV) for i in range(2)]
    ys, st = gpu_ns(mats, mode=mode, compute_dtype="fp32")
    assert st == [0, 0]
    for x, y in zip(mats, ys):
        U = to_np(x)
        assert rel(to_np(y), oracle.newton_schulz(U, Q5, mode=mode)) < 1e-4


@pytest.mark.parametrize("abc", [(0.0, 1.0, 0.0), (0.0, 0.0, 1.0)])
def test_fp32_tensor_core_single_products(abc):
    """One iteration isolates X X^T X (b) and (X X^T)^2 X (c) on the 3xTF32 path."""
    X = synth.gaussian(300, 777, seed=31, device=DEV)
    (Y,), st = gpu_ns([X], coeffs=[abc], compute_dtype="fp32")
    assert st == [0]
    assert rel(to_np(Y), oracle.newton_schulz(to_np(X), [abc])) < 1e-5  # one TF32 pass: ~5e-4


@pytest.mark.parametrize("mode", ["standard", "gram", "gram_stabilized"])
def test_fp32_dense_projection_shape(mode):
    """1024 x 4096 (the dense-projection shape): K = 4096 in X X^T, where an
    unfolded tensor-core accumulation would leave the fp32 bar."""
    mats = [synth.low_rank_plus_noise(1024, 4096, 64, 0.1, seed=810 + i, device=DEV) for i in range(2)]
    ys, st = gpu_ns(mats, mode=mode, compute_dtype="fp32")
    assert st == [0, 0]
    U = to_np(mats[0])
    y = to_np(ys[0])
    assert rel(y, oracle.newton_schulz(U, Q5, mode=mode)) < 1e-4
    assert sigma_band_error(U, y, Q5) < 0.05


# ---------------------------------------------------------------------------
# Muon step: momentum, Nesterov, orientation merge, decay and scale
# ---------------------------------------------------------------------------
def _groups_for_step(spec, w_dtype, seed):
    Ws, Gs, Ms = [], [], []
    for i, (r, c) in enumerate(spec):
        Ws.append(synth.gaussian(r, c, seed + 3 * i, DEV, std=0.5).to(w_dtype))
        Gs.append(synth.gaussian(r, c, seed + 3 * i + 1, DEV).bfloat16())
        Ms.append(synth.gaussian(r, c, seed + 3 * i + 2, DEV, std=0.3))
    return Ws, Gs, Ms


@pytest.mark.parametrize("mode", ["standard", "gram_stabilized"])
@pytest.mark.parametrize("nesterov", [True, False])
@pytest.mark.parametrize("compute", ["fp16", "bf16"])
def test_muon_step_vs_oracle(mode, nesterov, compute):
    # 2 wide + 1 tall of the same oriented shape (merged batch), a square one, a ragged one
    spec = [(192, 640), (192, 640), (640, 192), (256, 256), (72, 200)]
    hp = dict(lr=0.05, momentum=0.9, nesterov=nesterov, weight_decay=0.2, scale_coef=0.3, mode=mode,
              compute_dtype=compute)
    Ws, Gs, Ms = _groups_for_step(spec, torch.float32, 11)
    W0 = [to_np(w) for w in Ws]
    M0 = [to_np(m) for m in Ms]
    st = torch.full((len(spec),), -1, dtype=torch.int32, device=DEV)
    nsm.muon_step(Ws, Gs, Ms, status=st, **hp)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0] * len(spec)
    for i, (r, c) in enumerate(spec):
        Wr, Mr, Or = oracle.muon_step(W0[i], to_np(Gs[i]), M0[i], lr=0.05, momentum=0.9, nesterov=nesterov,
                                      weight_decay=0.2, scale_coef=0.3, eps=1e-7, coeffs=Q5, mode=mode)
        assert rel(to_np(Ms[i]), Mr) < 1e-6
        step = 0.05 * 0.3 * math.sqrt(max(r, c))
        O_gpu = ((1 - 0.05 * 0.2) * W0[i] - to_np(Ws[i])) / step
        U = oracle.nesterov_blend(to_np(Gs[i]), Mr, 0.9, nesterov)
        floor = emulated_floor(U, Q5, mode, chain=chain_of(mode, compute)) if compute == "bf16" else None
        assert rel(O_gpu, Or) < tolerance(compute, floor), i
        assert sigma_band_error(U, O_gpu, Q5) < 0.05


def test_bf16_weight_store_rounds_the_exact_update():
    """Same step with fp32 and bf16 W: the bf16 result is RNE(decay W - step O) of
    the O the fp32 run exposes (the orthogonalisation does not depend on W)."""
    spec = [(256, 512), (512, 256)]
    Wf, Gs, Ms = _groups_for_step(spec, torch.float32, 21)
    Wb = [w.bfloat16() for w in Wf]
    Wf = [w.float() for w in Wb]          # identical starting values
    Wf0 = [w.clone() for w in Wf]
    Ms2 = [m.clone() for m in Ms]
    nsm.muon_step(Wf, Gs, Ms)
    nsm.muon_step(Wb, Gs, Ms2)
    torch.cuda.synchronize()
    for i, (r, c) in enumerate(spec):
        step = 0.02 * 0.2 * math.sqrt(max(r, c))
        O = ((1 - 0.002) * Wf0[i].double() - Wf[i].double()) / step
        want = ((1 - 0.002) * Wf0[i] - step * O.float()).bfloat16()
        diff = (Wb[i].float() - want.float()).abs()
        ulp = want.float().abs().clamp_min(1e-30) * 2.0 ** -7
        assert bool((diff <= ulp * 1.01).all())
        assert torch.equal(Ms[i], Ms2[i])


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------
def test_zero_gradient_and_momentum_is_pure_decay():
    W = synth.gaussian(96, 320, 1, DEV)
    W0 = W.clone()
    G = torch.zeros(96, 320, device=DEV, dtype=torch.bfloat16)
    M = torch.zeros(96, 320, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    nsm.muon_step([W], [G], [M], status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(M, torch.zeros_like(M))
    assert torch.allclose(W, W0 * (1 - 0.002), rtol=0, atol=0)


def test_nonfinite_input_is_flagged_per_matrix():
    mats = [synth.gaussian(128, 256, s, DEV, dtype=torch.bfloat16) for s in range(3)]
    mats[1][5, 7] = float("nan")
    ys, st = gpu_ns(mats)
    assert st == [0, 1, 0]
    assert torch.isfinite(ys[0]).all() and torch.isfinite(ys[2]).all()
    # the Muon step reports it in the caller's order too
    Ws, Gs, Ms = _groups_for_step([(64, 192), (192, 64), (64, 192)], torch.float32, 5)
    Gs[2][0, 0] = float("inf")
    st = torch.full((3,), -1, dtype=torch.int32, device=DEV)
    nsm.muon_step(Ws, Gs, Ms, status=st)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0, 0, 1]


def test_empty_and_degenerate_inputs():
    nsm.muon_ns_batched([])  # no-op
    # rank-1 matrix: one singular value, f^K(1 / (1 + eps))
    u = torch.randn(48, 1, device=DEV, dtype=torch.float64)
    v = torch.randn(1, 160, device=DEV, dtype=torch.float64)
    X = (u @ v).float()
    (y,), st = gpu_ns([X], compute_dtype="fp32")
    want = oracle.newton_schulz(to_np(X), Q5)
    assert st == [0] and rel(to_np(y), want) < 1e-4
    # identical matrices in a batch give identical results (no cross-talk)
    base = synth.gaussian(150, 450, 9, DEV, dtype=torch.bfloat16)
    ys, st = gpu_ns([base, base.clone(), base.clone()])
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


def test_chunked_workspace_matches_single_chunk():
    mats = [synth.gaussian(256, 768, 40 + i, DEV, dtype=torch.bfloat16) for i in range(5)]
    full, _ = gpu_ns(mats)
    small = torch.empty(nsm.muon_ns_workspace_size(2, 256, 768), dtype=torch.uint8, device=DEV)
    chunked, st = gpu_ns(mats, workspace=small)
    assert st == [0] * 5
    for a, b in zip(full, chunked):
        assert torch.equal(a, b)


def test_deterministic_bitwise():
    mats = [synth.gaussian(384, 1152, 60 + i, DEV, dtype=torch.bfloat16) for i in range(4)]
    for mode in ("standard", "gram_stabilized"):
        a, _ = gpu_ns(mats, mode=mode)
        b, _ = gpu_ns(mats, mode=mode)
        for x, y in zip(a, b):
            assert torch.equal(x, y)


def test_workspace_too_small_is_rejected():
    X = synth.gaussian(256, 512, 1, DEV, dtype=torch.bfloat16)
    tiny = torch.empty(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(nsm.MuonError):
        nsm.muon_ns_batched([X], workspace=tiny)


def test_captured_step_replays_the_eager_step():
    """A step recorded in a CUDA graph and replayed gives the eager step's bits."""
    spec = [(128, 384), (384, 128), (96, 200)]
    for compute, wdt in (("fp16", torch.bfloat16), ("bf16", torch.bfloat16), ("fp32", torch.float32)):
        Wa, Ga, Ma = _groups_for_step(spec, wdt, 31)
        Wb = [w.clone() for w in Wa]
        Mb = [m.clone() for m in Ma]
        eager = nsm.MuonStep(Wa, Ga, Ma, compute_dtype=compute)
        graphed = nsm.MuonStep(Wb, Ga, Mb, compute_dtype=compute)
        eager()                       # matches the capture's own eager warm-up step
        g = graphed.capture()
        for _ in range(3):
            eager()
            g.replay()
        torch.cuda.synchronize()
        for x, y in zip(Wa + Ma, Wb + Mb):
            assert torch.equal(x, y)
        assert int(graphed.status.abs().sum()) == 0


def test_checkpoint_resume_is_bit_identical():
    """The only optimizer state is M (owned by the caller): saving W and M,
    stepping, restoring and stepping again reproduces the same bits."""
    spec = [(256, 768), (768, 256), (130, 520)]
    for mode in ("standard", "gram_stabilized"):
        Ws, Gs, Ms = _groups_for_step(spec, torch.bfloat16, 41)
        nsm.muon_step(Ws, Gs, Ms, mode=mode)
        saved_W = [w.clone() for w in Ws]
        saved_M = [m.clone() for m in Ms]
        nsm.muon_step(Ws, Gs, Ms, mode=mode)
        after_W = [w.clone() for w in Ws]
        after_M = [m.clone() for m in Ms]
        for w, s in zip(Ws, saved_W):
            w.copy_(s)
        for m, s in zip(Ms, saved_M):
            m.copy_(s)
        nsm.muon_step(Ws, Gs, Ms, mode=mode)
        torch.cuda.synchronize()
        for x, y in zip(Ws + Ms, after_W + after_M):
            assert torch.equal(x, y)


def test_streamed_step_matches_the_device_step():
    """Host-fed, slice-pipelined step (copies overlapped on side streams) gives
    the same bits as the plain step on device-resident gradients."""
    spec = [(256, 768), (768, 256), (128, 384), (384, 128), (200, 200), (256, 512)]
    Wa, Ga, Ma = _groups_for_step(spec, torch.bfloat16, 51)
    Wb = [w.clone() for w in Wa]
    Mb = [m.clone() for m in Ma]
    Gb = [torch.zeros_like(g) for g in Ga]
    hG = [g.cpu().pin_memory() for g in Ga]
    hW = [torch.empty(w.shape, dtype=w.dtype).pin_memory() for w in Wb]
    plain = nsm.MuonStep(Wa, Ga, Ma)
    streamed = nsm.StreamedMuonStep(Wb, Gb, Mb, hG, hW, slice_bytes=300_000)
    assert len(streamed.slices) > 2
    for _ in range(3):
        plain()
        streamed()
    torch.cuda.synchronize()
    for a, b, h in zip(Wa, Wb, hW):
        assert torch.equal(a, b)
        assert torch.equal(a.cpu(), h)
    for a, b in zip(Ma, Mb):
        assert torch.equal(a, b)
