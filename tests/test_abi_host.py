"""Host-only checks of the C ABI: the library loads, exports every entry point
include/muon.h declares, and its host logic (argument checks, workspace sizes,
FLOP counts, status strings) behaves, all without touching a GPU."""
import ctypes
import os
import re

import pytest

import newton_schulz_matrix_b200 as nsm
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon.h")


@pytest.fixture(scope="module")
def lib():
    from newton_schulz_matrix_b200 import build
    build.build()
    return nsm.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"MUON_API\s+[\w\s\*]+?\b(muon_\w+)\s*\(", text)


def test_header_declares_the_binding_names():
    assert sorted(declared_symbols()) == sorted(nsm.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # and nothing else from the C++ side leaks out as a muon_ symbol
    out = os.popen(f"nm -D --defined-only {nsm.library_path()}").read()
    exported = set(re.findall(r" T (muon_\w+)", out))
    assert exported == set(declared_symbols())


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, 1, 2, 3):
        assert nsm.muon_status_string(code) != "unknown code"
    assert nsm.muon_status_string(99) == "unknown code"


def _ns(coeffs=(nsm.QUINTIC,) * 5, mode="standard", restart_after=2, compute="bf16", gram="fp16", every=0):
    return nsm._ns_params(coeffs, mode, restart_after, 1e-7, compute, gram, every)


@pytest.mark.parametrize("rows,cols", [(64, 128), (2048, 7168), (7168, 18432), (1408, 2048), (333, 77)])
@pytest.mark.parametrize("mode", ["standard", "gram", "gram_stabilized"])
def test_flop_counts_agree_with_oracle(lib, rows, cols, mode):
    ns, _a = _ns(mode=mode)
    got = lib.muon_ns_flops(rows, cols, ctypes.byref(ns))
    assert got == float(oracle.flops(rows, cols, 5, mode, 2))


@pytest.mark.parametrize("iters,restart,every", [(5, 2, 2), (7, 1, 3), (5, 2, 1), (6, 3, 0)])
def test_periodic_restart_flop_counts_agree_with_oracle(lib, iters, restart, every):
    ns, _a = _ns(coeffs=(nsm.QUINTIC,) * iters, mode="gram_stabilized", restart_after=restart, every=every)
    assert lib.muon_ns_flops(2048, 7168, ctypes.byref(ns)) == float(
        oracle.flops(2048, 7168, iters, "gram_stabilized", restart, every))
    bad, _b = _ns(mode="gram_stabilized", every=-1)
    assert lib.muon_ns_flops(2048, 7168, ctypes.byref(bad)) == 0.0


def test_ns_workspace_size(lib):
    ns, _a = _ns()
    one = lib.muon_ns_workspace_size(1, 2048, 7168, ctypes.byref(ns))
    two = lib.muon_ns_workspace_size(2, 7168, 2048, ctypes.byref(ns))
    # 2 X buffers + A + B in bf16, plus partials and alignment slack
    per = 2 * 2048 * 7168 * 2 + 2 * 2048 * 2048 * 2
    assert per < one < per + 64 * 1024
    assert two - one == pytest.approx(one, rel=1e-3)
    nsg, _a = _ns(mode="gram")
    assert lib.muon_ns_workspace_size(1, 2048, 7168, ctypes.byref(nsg)) > one  # five Gram-sized buffers
    # invalid arguments give 0
    assert lib.muon_ns_workspace_size(0, 64, 64, ctypes.byref(ns)) == 0
    bad, _a = _ns(mode="gram_stabilized", restart_after=5)
    assert lib.muon_ns_workspace_size(1, 64, 64, ctypes.byref(bad)) == 0


def test_fp32_workspace_holds_the_tf32_planes(lib):
    """fp32 chains whose products run as 3xTF32 (n >= 256) also hold their
    operands' TF32 hi / lo planes, one X-sized and two n x n pairs:
    2 (n m + 2 n^2) x 4 bytes per matrix on top of the chain's own buffers
    (twice the 16-bit ones); the fused small-matrix path (n < 256) holds none."""
    ns16, _a = _ns()
    ns32, _b = _ns(compute="fp32")

    def per_matrix(ns, n, m):
        return lib.muon_ns_workspace_size(2, n, m, ctypes.byref(ns)) - lib.muon_ns_workspace_size(1, n, m, ctypes.byref(ns))

    n, m = 512, 1024
    planes = 2 * (n * m + 2 * n * n) * 4
    extra = per_matrix(ns32, n, m) - 2 * per_matrix(ns16, n, m)
    assert planes - 4096 < extra <= planes  # less the doubled per-matrix partials and counters
    n, m = 128, 256
    assert abs(per_matrix(ns32, n, m) - 2 * per_matrix(ns16, n, m)) < 4096


def _fake_group(rows, cols, count, wdt=nsm.BF16, gdt=nsm.BF16, ptr=1 << 20):
    arrs = [(ctypes.c_void_p * count)(*[ptr + 4096 * i for i in range(count)]) for _ in range(3)]
    return nsm._Group(rows, cols, count, wdt, gdt, *arrs), arrs


def test_workspace_queries_and_merge_by_orientation(lib):
    g1, k1 = _fake_group(1408, 2048, 4)
    g2, k2 = _fake_group(2048, 1408, 2)
    groups = (nsm._Group * 2)(g1, g2)
    ns, _a = _ns()
    hp = nsm._hparams(0.02, 0.95, 0.1, 0.2, 1, ns)
    full = lib.muon_workspace_size(groups, 2, ctypes.byref(hp))
    mn = lib.muon_workspace_min(groups, 2, ctypes.byref(hp))
    single = lib.muon_ns_workspace_size(6, 1408, 2048, ctypes.byref(ns))
    assert full == single          # both groups share one 1408 x 2048 batch
    assert mn == lib.muon_ns_workspace_size(1, 1408, 2048, ctypes.byref(ns))


def test_argument_errors_are_caught_on_the_host(lib):
    ns, _a = _ns()
    hp = nsm._hparams(0.02, 0.95, 0.1, 0.2, 1, ns)
    g, keep = _fake_group(64, 128, 1)
    groups = (nsm._Group * 1)(g)
    ws = ctypes.c_void_p(1 << 24)
    # zero groups, null workspace, misaligned pointer, bad dtype, bad shape, small workspace
    assert lib.muon_step(groups, 0, ctypes.byref(hp), ws, 1 << 30, None, None) == -1
    assert lib.muon_step(groups, 1, ctypes.byref(hp), None, 1 << 30, None, None) == -1
    assert lib.muon_step(groups, 1, ctypes.byref(hp), ctypes.c_void_p((1 << 24) + 8), 1 << 30, None, None) == -1
    bad, k2 = _fake_group(64, 128, 1, ptr=(1 << 20) + 4)
    assert lib.muon_step((nsm._Group * 1)(bad), 1, ctypes.byref(hp), ws, 1 << 30, None, None) == -1
    bad, k3 = _fake_group(64, 128, 1, wdt=7)
    assert lib.muon_step((nsm._Group * 1)(bad), 1, ctypes.byref(hp), ws, 1 << 30, None, None) == -2
    bad, k4 = _fake_group(0, 128, 1)
    assert lib.muon_step((nsm._Group * 1)(bad), 1, ctypes.byref(hp), ws, 1 << 30, None, None) == -1
    assert lib.muon_step(groups, 1, ctypes.byref(hp), ws, 1024, None, None) == -3
    # NaN hyper-parameter and bad coefficient count
    hp_nan = nsm._hparams(float("nan"), 0.95, 0.1, 0.2, 1, ns)
    assert lib.muon_step(groups, 1, ctypes.byref(hp_nan), ws, 1 << 30, None, None) == -1
    ns0, _b = _ns(coeffs=())
    hp0 = nsm._hparams(0.02, 0.95, 0.1, 0.2, 1, ns0)
    assert lib.muon_step(groups, 1, ctypes.byref(hp0), ws, 1 << 30, None, None) == -1
    # muon_ns_batched: null array, misaligned matrix
    X = (ctypes.c_void_p * 1)((1 << 20) + 2)
    assert lib.muon_ns_batched(X, 1, 64, 64, nsm.BF16, ctypes.byref(ns), ws, 1 << 30, None, None) == -1
    assert lib.muon_ns_batched(None, 1, 64, 64, nsm.BF16, ctypes.byref(ns), ws, 1 << 30, None, None) == -1
    # zero matrices is a no-op
    assert lib.muon_ns_batched(X, 0, 64, 64, nsm.BF16, ctypes.byref(ns), ws, 1 << 30, None, None) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    w = torch.zeros(4, 8)
    with pytest.raises(nsm.MuonError):
        nsm.muon_step([w], [w.clone()], [w.clone()])
    with pytest.raises(nsm.MuonError):
        nsm.muon_ns_batched([w])
