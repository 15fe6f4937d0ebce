"""Pins for the fp64 oracle: it is checked against things other than itself.

Each test ties one oracle function to something the pages or the mathematics
fix: the pages' FLOP formula and shape set (tests/golden/pages_facts.json), an
SVD routine (LAPACK via numpy), closed forms on constructed inputs, and exact
algebraic identities between the standard and Gram forms.  A plausible slip in
the oracle (a dropped term, a wrong sign or index, a transposed operand, eps in
the wrong place, the listing's sqrt(m) kept) fails at least one of them; the
last test plants such slips in a copy of the oracle and checks exactly that.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")
FACTS = json.load(open(GOLDEN))
Q5 = [oracle.QUINTIC] * 5


def rng_matrix(rows, cols, seed):
    return synth.gaussian(rows, cols, seed).double().numpy()


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def svd_prediction(U, coeffs, eps=1e-7):
    """What the iteration must give by the singular-value argument: same singular
    vectors as U, each sigma mapped by s -> a s + b s^3 + c s^5 (K times) after
    dividing by ||U||_F + eps.  Uses only LAPACK's SVD and scalar arithmetic."""
    P, s, Vt = np.linalg.svd(U, full_matrices=False)
    fro = math.sqrt(float(np.sum(s * s)))
    t = s / (fro + eps)
    for a, b, c in coeffs:
        t = a * t + b * t ** 3 + c * t ** 5
    return (P * t) @ Vt


# ---------------------------------------------------------------------------
# FLOP counts the pages print (P-4)
# ---------------------------------------------------------------------------
def test_standard_flops_match_pages_formula():
    f = FACTS["standard_iteration_products"]
    for rows, cols in [(64, 128), (128, 64), (2048, 7168), (7168, 18432), (1408, 2048), (333, 77)]:
        n, m = min(rows, cols), max(rows, cols)
        env = {"m": m, "n": n}
        want = sum(eval(f[k], {}, env) for k in ("XXt", "A2", "BX"))
        assert oracle.flops_standard_iteration(rows, cols) == want
    assert oracle.flops_standard_iteration(64, 128) == 2_621_440
    assert oracle.flops_standard(64, 128, 5) == 5 * 2_621_440


def test_kimi_k2_total_flops():
    k2 = FACTS["kimi_k2_shape_set"]
    experts = k2["expert_count"] * k2["matrices_per_block"]
    dense = k2["dense_count"] * k2["matrices_per_block"]
    total = experts * oracle.flops_standard(*k2["expert_shape"], 5) + dense * oracle.flops_standard(*k2["dense_shape"], 5)
    assert abs(total / 1e12 - 513.2) < 0.05
    # the synthetic K2 set has the page's matrix count and oriented shapes
    w = synth.kimi_k2(counts=[0, 0, 0, 0])
    assert w.groups == []


def test_gram_flops_plausibility_band():
    """The pages' complexity table was lost (our counts are pinned to the
    executed products below).  They must give savings that include the
    surviving 42-58 % band somewhere in alpha > 1."""
    band = FACTS["gram_flop_saving_band"]
    n = 1024
    savings = []
    for alpha in (2, 3, 4, 5, 6, 8):
        std = oracle.flops_standard(n, alpha * n, 5)
        savings.append(1 - oracle.flops_gram(n, alpha * n, 5, 0) / std)
    assert any(band["lo"] <= s <= band["hi"] for s in savings)
    assert all(b > a for a, b in zip(savings, savings[1:]))  # cheaper as alpha grows
    # closed forms of our own count, K = 5
    for alpha in (1, 2, 4, 8):
        assert oracle.flops_gram(n, alpha * n, 5, 0) == (4 * alpha + 34) * n ** 3
        assert oracle.flops_gram(n, alpha * n, 5, 2) == (8 * alpha + 28) * n ** 3
        assert oracle.flops_standard(n, alpha * n, 5) == (20 * alpha + 10) * n ** 3


# ---------------------------------------------------------------------------
# Singular-value map (P-3): the iteration acts on each singular value alone
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(8, 24), (24, 8), (16, 16), (64, 128), (37, 5)])
@pytest.mark.parametrize("mode", oracle.MODES)
def test_singular_value_map(shape, mode):
    U = rng_matrix(*shape, seed=11 + shape[0])
    got = oracle.newton_schulz(U, Q5, mode=mode)
    want = svd_prediction(U, Q5)
    assert rel(got, want) < 1e-10


def test_band_of_quintic():
    """Normalised sigma >= 1e-2 lands in [0.6818, 1.1344] after 5 quintic steps."""
    s = np.logspace(-2, 0, 4001)
    out = oracle.singular_value_map(s, Q5)
    assert out.min() > 0.68 and out.max() < 1.135
    assert abs(oracle.singular_value_map([1.0], Q5[:1])[0] - 0.701) < 1e-12  # a + b + c


def test_cubic_constants_from_page():
    c = FACTS["cubic_iteration"]
    a, b, cc = oracle.CUBIC
    # 1/2 X (3I - X X^T) = (3/2) X - (1/2) X X^T X
    assert a == c["half"] * c["three"] and b == -c["half"] and cc == 0.0


# ---------------------------------------------------------------------------
# Polar limit (P-2): 40 cubic steps on the 64 x 128 fp32 workload
# ---------------------------------------------------------------------------
def test_cubic_converges_to_polar_factor():
    w = synth.single_fp32()
    g = w.groups[0]
    U = g.G[0].double().numpy()  # momentum 0: U is a multiple of G
    got = oracle.newton_schulz(U, [oracle.CUBIC] * 40)
    P, s, Vt = np.linalg.svd(U, full_matrices=False)
    assert rel(got, P @ Vt) < 1e-12
    # tall input: the polar factor of the transpose, transposed
    got_t = oracle.newton_schulz(U.T, [oracle.CUBIC] * 40)
    assert rel(got_t, (P @ Vt).T) < 1e-12


# ---------------------------------------------------------------------------
# Exact equivalence of the three forms (P-1) and Gram invariants (P-5)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(4, 12), (16, 48), (64, 128)])
def test_gram_equals_standard_in_exact_arithmetic(shape):
    X0 = oracle.frobenius_normalize(rng_matrix(*shape, seed=5))
    std = oracle.ns_standard(X0, Q5)
    assert rel(oracle.ns_gram(X0, Q5, 0), std) < 1e-12
    for r in (1, 2, 3, 4):
        assert rel(oracle.ns_gram(X0, Q5, r), std) < 1e-12
        for e in (1, 2, 3):  # periodic restarts
            assert rel(oracle.ns_gram(X0, Q5, r, restart_every=e), std) < 1e-12
    for K in range(1, 6):
        assert rel(oracle.ns_gram(X0, Q5[:K], 0), oracle.ns_standard(X0, Q5[:K])) < 1e-12


def test_gram_trace_invariants():
    X0 = oracle.frobenius_normalize(rng_matrix(16, 48, seed=9))
    R0 = X0 @ X0.T
    tr = []
    oracle.ns_gram(X0, Q5, 0, trace=tr)
    for k, R, Qacc, _ in tr[:-1]:
        Xk = oracle.ns_standard(X0, Q5[:k])
        assert rel(R, Xk @ Xk.T) < 1e-12           # R_k = X_k X_k^T
        assert rel(Qacc @ X0, Xk) < 1e-12          # X_k = Q_acc X_0
        assert rel(Qacc @ R0, R0 @ Qacc) < 1e-12   # Q_acc commutes with R_0
    # stabilised: after the restart the carried X is X_2 and Q_acc restarts at I
    tr = []
    oracle.ns_gram(X0, Q5, 2, trace=tr)
    k, R, Qacc, X2 = tr[1]
    assert k == 2 and np.array_equal(Qacc, np.eye(16))
    assert rel(X2, oracle.ns_standard(X0, Q5[:2])) < 1e-12


def test_converged_qacc_is_inverse_sqrt_of_gram():
    X0 = oracle.frobenius_normalize(rng_matrix(8, 40, seed=3))
    tr = []
    oracle.ns_gram(X0, [oracle.CUBIC] * 40, 0, trace=tr)
    _, _, Qacc, _ = tr[-1]
    lam, V = np.linalg.eigh(X0 @ X0.T)
    assert rel(Qacc, (V / np.sqrt(lam)) @ V.T) < 1e-10


# ---------------------------------------------------------------------------
# Update rule closed forms (P-6) and momentum / Nesterov / eps placement
# ---------------------------------------------------------------------------
HP = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, scale_coef=0.2, eps=1e-7, coeffs=Q5)


def test_zero_gradient_gives_pure_decay():
    W = rng_matrix(16, 32, 1)
    Z = np.zeros_like(W)
    W1, M1, O = oracle.muon_step(W, Z, Z, **HP)
    assert np.array_equal(O, Z) and np.array_equal(M1, Z)
    assert np.array_equal(W1, (1 - 0.02 * 0.1) * W)


def test_orthonormal_rows_closed_form():
    n, m, kappa = 8, 32, 3.0
    Qm = np.linalg.qr(rng_matrix(m, n, 4))[0].T  # n x m, orthonormal rows
    W = rng_matrix(n, m, 2)
    hp = dict(HP, momentum=0.0, nesterov=False)
    W1, M1, O = oracle.muon_step(W, kappa * Qm, np.zeros((n, m)), **hp)
    s0 = kappa / (kappa * math.sqrt(n) + 1e-7)
    fK = oracle.singular_value_map([s0], Q5)[0]
    assert rel(O, fK * Qm) < 1e-12
    scale = 0.2 * math.sqrt(m)
    assert rel(W1, (1 - 0.002) * W - 0.02 * scale * fK * Qm) < 1e-12
    # scale invariance up to eps: kappa -> 1000 kappa changes O only at the eps/||U|| level
    _, _, O2 = oracle.muon_step(W, 1000 * kappa * Qm, np.zeros((n, m)), **hp)
    assert 0 < rel(O2, O) < 1e-7


def test_eps_is_added_to_the_norm():
    """A tiny input shows where eps sits: s0 = k / (k sqrt(n) + eps)."""
    n, m, kappa = 4, 16, 1e-9
    Qm = np.linalg.qr(rng_matrix(m, n, 6))[0].T
    O = oracle.newton_schulz(kappa * Qm, Q5)
    s0 = kappa / (kappa * math.sqrt(n) + 1e-7)
    assert abs(s0 - 0.0098) < 1e-3
    assert rel(O, oracle.singular_value_map([s0], Q5)[0] * Qm) < 1e-12


def test_momentum_and_nesterov_closed_form():
    """G = e1 e1^T, M_prev = e2 e2^T on a 4 x 8 matrix: U is diagonal with known entries."""
    mu = 0.95
    G = np.zeros((4, 8)); G[0, 0] = 1.0
    M = np.zeros((4, 8)); M[1, 1] = 1.0
    W = np.zeros((4, 8))
    for nesterov, (u0, u1) in [(True, ((1 - mu) * (1 + mu), mu * mu)), (False, (1 - mu, mu))]:
        hp = dict(HP, nesterov=nesterov, weight_decay=0.0)
        W1, M1, O = oracle.muon_step(W, G, M, **hp)
        assert M1[0, 0] == pytest.approx(1 - mu) and M1[1, 1] == pytest.approx(mu)
        fro = math.hypot(u0, u1) + 1e-7
        f0, f1 = oracle.singular_value_map([u0 / fro, u1 / fro], Q5)
        want = np.zeros((4, 8)); want[0, 0] = f0; want[1, 1] = f1
        assert rel(O, want) < 1e-12
        assert rel(W1, -0.02 * 0.2 * math.sqrt(8) * want) < 1e-12


def test_momentum_zero_uses_gradient():
    G = rng_matrix(8, 16, 21)
    M = rng_matrix(8, 16, 22)
    hp = dict(HP, momentum=0.0)
    _, M1, O = oracle.muon_step(np.zeros_like(G), G, M, **hp)
    assert np.array_equal(M1, G)
    assert rel(O, svd_prediction(G, Q5)) < 1e-10


def test_update_scale_from_page():
    assert oracle.update_scale(64, 128, 1.0) == math.sqrt(128)
    assert oracle.update_scale(7168, 2048, 0.2) == pytest.approx(0.2 * math.sqrt(7168))


# ---------------------------------------------------------------------------
# Rounding emulation (diagnosis helper) against torch's own conversions
# ---------------------------------------------------------------------------
def test_round_to_matches_torch_conversions():
    x = rng_matrix(64, 64, 8) * np.logspace(-8, 8, 64)[None, :]
    t = torch.from_numpy(x)
    assert np.array_equal(oracle.round_to(x, "bf16"), t.float().bfloat16().double().numpy())
    assert np.array_equal(oracle.round_to(x, "fp16"), t.float().half().double().numpy())
    assert np.array_equal(oracle.round_to(x, "fp32"), t.float().double().numpy())


# ---------------------------------------------------------------------------
# Negative-eigenvalue mechanism (P-7): reduced-precision Gram iteration
# ---------------------------------------------------------------------------
def test_negative_eigenvalue_growth_factor():
    """For lambda < 0, h(lambda) = a + b lambda + c lambda^2 > a, so R <- Q R Q
    multiplies a negative eigenvalue by at least a^2 ~ 11.86 per step."""
    a, b, c = oracle.QUINTIC
    lam = -1e-4
    seq = []
    for _ in range(5):
        h = a + b * lam + c * lam * lam
        lam = h * lam * h
        seq.append(lam)
    assert all(abs(y / x) >= a * a for x, y in zip([-1e-4] + seq, seq))
    assert seq[2] == pytest.approx(-0.17, rel=0.1)


# ---------------------------------------------------------------------------
# Planted mistakes: each plausible slip must fail one of the pins above
# ---------------------------------------------------------------------------
def _std_variant(kind):
    def run(X0, coeffs):
        X = X0.copy()
        for a, b, c in coeffs:
            if kind == "xtx":
                A = X.T @ X
                B = b * A + c * A @ A
                X = a * X + X @ B
                continue
            A = X @ X.T
            if kind == "drop_c":
                B = b * A
            elif kind == "sign_b":
                B = -b * A + c * A @ A
            else:
                B = b * A + c * A @ A
            X = a * X + B @ X
        return X
    return run


@pytest.mark.parametrize("kind", ["drop_c", "sign_b", "xtx_equiv"])
def test_planted_mistakes_are_caught(kind):
    U = rng_matrix(8, 24, 17)
    P, s, Vt = np.linalg.svd(U, full_matrices=False)
    X0 = U / (math.sqrt(float(np.sum(s * s))) + 1e-7)
    want = svd_prediction(U, Q5)
    if kind == "xtx_equiv":
        # iterating on the long side is the same map in exact arithmetic: not a mistake
        assert rel(_std_variant("xtx")(X0, Q5), want) < 1e-10
    else:
        assert rel(_std_variant(kind)(X0, Q5), want) > 1e-3
    # keeping the listing's sqrt(m) in the normalisation is caught too
    X0m = U / ((math.sqrt(float(np.sum(s * s))) + 1e-7) * math.sqrt(8))
    assert rel(oracle.ns_standard(X0m, Q5), want) > 1e-3


def test_fp16_gram_negative_eigenvalues_and_restart():
    """The write-up's stabilised-variant paragraph: in float16 the Gram matrix
    picks up negative eigenvalues that the naive iteration amplifies; restarting
    after step 2 (fresh R = X X^T) keeps them small.  Reproduced with the
    oracle's fp16 stored-precision iteration on an ill-conditioned input."""
    Q5_ = [oracle.QUINTIC] * 5
    U = synth.with_spectrum(64, 256, synth.log_uniform_sigma(64, 1e-6, 1, 5), 9).double().numpy()
    X0 = oracle.frobenius_normalize(U)
    mins = {}
    outs = {}
    for ra in (0, 2):
        tr = []
        outs[ra] = oracle.ns_gram_stored(oracle.round_to(X0, "fp16"), Q5_, "fp16", ra, trace=tr)
        mins[ra] = [np.linalg.eigvalsh(R).min() for _, R, _, _ in tr]
    naive, stab = mins[0], mins[2]
    assert all(v < 0 for v in naive)
    assert all(abs(b / a) > 8 for a, b in zip(naive, naive[1:]))   # ~a^2 growth per step
    assert abs(naive[-1]) > 10 * abs(stab[-1])
    ref = oracle.ns_standard(X0, Q5_)
    assert rel(outs[0], ref) > 3 * rel(outs[2], ref)


# ---------------------------------------------------------------------------
# The stored-precision iterations (they set the bar of a few GPU tests on
# ill-conditioned inputs), pinned two ways:
#   - with no rounding ("fp64") they are the exact iteration, which the pins
#     above tie to the SVD: this fixes their algebra, the mirrored triangles,
#     and where f = 1 / (||U|| + eps) enters when they start from the raw U;
#   - on diagonal inputs every product is a single multiplication per entry,
#     so the iteration reduces to scalar recurrences with one rounding per
#     stored product; written out below entry by entry, they must agree bit for
#     bit.  A rounding too many or too few, or at the wrong point, changes the
#     result (checked with planted variants).
# ---------------------------------------------------------------------------
SCHEDULES = {"quintic": Q5, "cubic": [oracle.CUBIC] * 4,
             "mixed": [(3.0, -3.2, 1.2), oracle.CUBIC, oracle.QUINTIC, (2.5, -2.0, 0.6)]}


@pytest.mark.parametrize("sched", sorted(SCHEDULES))
@pytest.mark.parametrize("mode,ra,every", [("standard", 0, 0), ("gram", 0, 0), ("gram_stabilized", 1, 0),
                                           ("gram_stabilized", 2, 0), ("gram_stabilized", 1, 2)])
@pytest.mark.parametrize("raw", [False, True])
def test_stored_iteration_without_rounding_is_the_exact_iteration(sched, mode, ra, every, raw):
    coeffs = SCHEDULES[sched]
    U = rng_matrix(24, 72, 41) * 37.0
    f = 1.0 / (oracle.frobenius_norm(U) + 1e-7)
    exact = oracle.newton_schulz(U, coeffs, mode=mode, restart_after=ra or 2, restart_every=every)
    start, pre = (U, f) if raw else (U * f, None)
    if mode == "standard":
        got = oracle.ns_standard_stored(start, coeffs, "fp64", prescale=pre)
    else:
        got = oracle.ns_gram_stored(start, coeffs, "fp64", ra, prescale=pre, restart_every=every)
    assert rel(got, exact) < 1e-12


def _scalar_standard(d, coeffs, fmt, f, round_a=True):
    rnd = lambda v: oracle.round_to(np.asarray(v, dtype=np.float64), fmt)
    s = d.copy()
    for a, b, c in coeffs:
        A = f * f * (s * s)
        A = rnd(A) if round_a else A
        if c != 0.0:
            B = rnd(c * (A * A) + b * A)
            s = rnd(f * (a * s + B * s))
        else:
            s = rnd(f * (a * s + b * (A * s)))
        f = 1.0
    return s


def _scalar_gram(d, coeffs, fmt, ra, f, round_t=True):
    rnd = lambda v: oracle.round_to(np.asarray(v, dtype=np.float64), fmt)
    s = d.copy()
    r = rnd(f * f * (s * s))
    qacc = None
    for k, (a, b, c) in enumerate(coeffs, start=1):
        q = rnd(c * (r * r) + b * r + a)
        qacc = q if qacc is None else rnd(q * qacc)
        if k == len(coeffs):
            break
        if ra and k == ra:
            s = rnd(f * (qacc * s))
            f = 1.0
            r = rnd(s * s)
            qacc = None
        else:
            t = q * r
            t = rnd(t) if round_t else t
            r = rnd(t * q)
    return rnd(f * (qacc * s))


def _diagonal_case(fmt, raw, n=400, m=560, seed=6):
    """A diagonal n x m input whose scaled entries spread over [1e-4, 1] (entries
    near 1 make every rounding visible); ``raw``: the stored values are 37.37 x
    larger and the prescale brings them back (the store-point structure is what
    is pinned here; the Frobenius normalisation is pinned by the fp64 test)."""
    rng = np.random.default_rng(seed)
    d = np.exp(rng.uniform(math.log(1e-4), 0.0, n)) * rng.choice([-1.0, 1.0], n)
    scale = 37.37 if raw else 1.0
    d = oracle.round_to(d * scale, fmt)
    X = np.zeros((n, m))
    X[np.arange(n), np.arange(n)] = d
    f = 1.0 / float(np.max(np.abs(d))) if raw else None
    return X, d, f


@pytest.mark.parametrize("fmt", ["bf16", "fp16"])
@pytest.mark.parametrize("sched", sorted(SCHEDULES))
@pytest.mark.parametrize("raw", [False, True])
def test_stored_standard_rounds_exactly_at_the_store_points(fmt, sched, raw):
    coeffs = SCHEDULES[sched]
    X, d, f = _diagonal_case(fmt, raw)
    got = oracle.ns_standard_stored(X, coeffs, fmt, prescale=f)
    want = _scalar_standard(d, coeffs, fmt, 1.0 if f is None else f)
    n = len(d)
    assert np.array_equal(np.diag(got[:, :n]), want)
    assert not np.any(got[:, :n] - np.diag(np.diag(got[:, :n]))) and not np.any(got[:, n:])
    # planted variants: A kept unrounded, or f applied before the first store
    assert not np.array_equal(_scalar_standard(d, coeffs, fmt, 1.0 if f is None else f, round_a=False), want)
    if raw:
        pre = oracle.round_to(d * f, fmt)
        assert not np.array_equal(_scalar_standard(pre, coeffs, fmt, 1.0), want)


@pytest.mark.parametrize("fmt", ["bf16", "fp16"])
@pytest.mark.parametrize("sched", ["quintic", "mixed"])
@pytest.mark.parametrize("ra", [0, 1, 2])
@pytest.mark.parametrize("raw", [False, True])
def test_stored_gram_rounds_exactly_at_the_store_points(fmt, sched, ra, raw):
    coeffs = SCHEDULES[sched]
    X, d, f = _diagonal_case(fmt, raw, seed=7 + ra)
    got = oracle.ns_gram_stored(X, coeffs, fmt, ra, prescale=f)
    want = _scalar_gram(d, coeffs, fmt, ra, 1.0 if f is None else f)
    n = len(d)
    assert np.array_equal(np.diag(got[:, :n]), want)
    assert not np.any(got[:, :n] - np.diag(np.diag(got[:, :n]))) and not np.any(got[:, n:])
    assert not np.array_equal(_scalar_gram(d, coeffs, fmt, ra, 1.0 if f is None else f, round_t=False), want)


def test_stored_symmetric_products_are_exactly_symmetric():
    """The GPU stores X X^T, A A^T, R R^T and the R update's second product as
    a mirrored upper triangle; the stored iteration's R must be too."""
    U = synth.with_spectrum(32, 96, synth.log_uniform_sigma(32, 1e-4, 1, 3), 4).double().numpy()
    tr = []
    oracle.ns_gram_stored(oracle.round_to(oracle.frobenius_normalize(U), "fp16"), Q5, "fp16", 0, trace=tr)
    for _, R, _, _ in tr:
        assert np.array_equal(R, R.T)


# ---------------------------------------------------------------------------
# FLOP counters pinned to the products the iteration actually executes: the
# oracle's own iteration runs on an array wrapper that counts every matrix
# product (2 * rows * cols * inner), skipping products with an exact identity
# operand (Q_acc = I at k = 1 and right after a restart, which the kernels skip)
# ---------------------------------------------------------------------------
class _Counted:
    __array_ufunc__ = None  # numpy's operators defer to the reflected methods below
    flops = [0]

    def __init__(self, a):
        self.a = np.asarray(a, dtype=np.float64)

    @staticmethod
    def _raw(x):
        return x.a if isinstance(x, _Counted) else np.asarray(x)

    @classmethod
    def _count(cls, A, B):
        eye = lambda M: M.ndim == 2 and M.shape[0] == M.shape[1] and np.array_equal(M, np.eye(M.shape[0]))
        if not (eye(A) or eye(B)):
            cls.flops[0] += 2 * A.shape[0] * B.shape[1] * A.shape[1]
        return _Counted(A @ B)

    def __matmul__(self, o):
        return self._count(self.a, self._raw(o))

    def __rmatmul__(self, o):
        return self._count(self._raw(o), self.a)

    def __add__(self, o):
        return _Counted(self.a + self._raw(o))

    __radd__ = __add__

    def __sub__(self, o):
        return _Counted(self.a - self._raw(o))

    def __rsub__(self, o):
        return _Counted(self._raw(o) - self.a)

    def __mul__(self, o):
        return _Counted(self.a * self._raw(o))

    __rmul__ = __mul__

    @property
    def T(self):
        return _Counted(self.a.T)

    @property
    def shape(self):
        return self.a.shape

    def copy(self):
        return _Counted(self.a.copy())


@pytest.mark.parametrize("shape", [(8, 24), (24, 8), (16, 16), (12, 40)])
@pytest.mark.parametrize("iters,restart,every", [(5, 0, 0), (5, 2, 0), (3, 1, 0), (6, 4, 0), (1, 0, 0), (2, 0, 0),
                                                 (5, 2, 2), (7, 1, 3), (5, 2, 1)])
def test_gram_flop_count_equals_the_products_executed(monkeypatch, shape, iters, restart, every):
    from oracle import muon_oracle as mo
    monkeypatch.setattr(mo, "_f64", lambda a: _Counted(a))
    X0 = np.random.default_rng(3).standard_normal(shape)
    X0 = X0 if shape[0] <= shape[1] else X0.T  # the iteration runs on the n x m orientation
    X0 = X0 / np.linalg.norm(X0)
    _Counted.flops[0] = 0
    out = mo.ns_gram(X0, [oracle.QUINTIC] * iters, restart_after=restart, restart_every=every)
    assert isinstance(out, _Counted)
    assert _Counted.flops[0] == oracle.flops_gram(*shape, iters, restart, every)
    mode = oracle.GRAM if restart == 0 else oracle.GRAM_STABILIZED
    if restart == 0 or restart < iters:
        assert _Counted.flops[0] == oracle.flops(*shape, iters, mode, restart_after=restart or 2, restart_every=every)


@pytest.mark.parametrize("iters,restart,every,points", [(5, 2, 2, [2, 4]), (7, 1, 3, [1, 4]), (5, 2, 1, [2, 3, 4]),
                                                        (5, 2, 0, [2]), (5, 4, 1, [4]), (3, 2, 5, [2])])
def test_periodic_restart_points(iters, restart, every, points):
    """Restarts come after iteration restart_after and every restart_every
    iterations after it, never after the last iteration; each restart leaves
    Q_acc = I and R = X X^T of the materialised X (seen in the trace)."""
    assert [k for k in range(1, iters + 1) if oracle.is_restart(k, iters, restart, every)] == points
    X0 = oracle.frobenius_normalize(rng_matrix(12, 36, 8))
    tr = []
    out = oracle.ns_gram(X0, Q5[:1] * iters, restart, trace=tr, restart_every=every)
    for k, R, Qacc, X in tr:
        if k in points:
            assert np.array_equal(Qacc, np.eye(12))
            assert np.allclose(R, X @ X.T, rtol=0, atol=1e-14)
    assert rel(out, oracle.ns_standard(X0, Q5[:1] * iters)) < 1e-12


@pytest.mark.parametrize("shape", [(8, 24), (16, 16)])
def test_standard_flop_count_equals_the_products_executed(monkeypatch, shape):
    from oracle import muon_oracle as mo
    monkeypatch.setattr(mo, "_f64", lambda a: _Counted(a))
    _Counted.flops[0] = 0
    X0 = np.random.default_rng(4).standard_normal(shape)
    mo.ns_standard(X0 / np.linalg.norm(X0), [oracle.QUINTIC] * 5)
    assert _Counted.flops[0] == oracle.flops_standard(*shape, 5)
