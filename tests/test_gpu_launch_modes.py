"""The library's launch modes give the same bits.

The product launches of a chain can go out one by one (the default: tiles
from a per-launch counter, programmatic dependent launch) or as one
persistent launch per chunk (MUON_CHAIN=1: products ordered by per-matrix
dependency counters, gemm_chain.cu); the Muon update can be written by the
last product's epilogue or by a separate pass (MUON_FUSED_UPDATE); launches
may or may not overlap the previous kernel's drain (MUON_PDL=0); tiles can be
handed out round-robin instead of from the counter (MUON_TILE_ORDER=static).
Each switch is read when the library loads, so the tests run every case in
a child process per variant and compare W, M, X and the status words bit for
bit with the default run in this process.  The arithmetic is the same in
every mode (same tiles, same k order, same epilogue, the update's rounding
pinned), so any difference is a scheduling or memory-ordering fault.

Cases: wide and tall matrices merged in one batch, ragged shapes whose rows
are not 16-byte multiples, every W dtype, all three forms, a non-finite
gradient, small batches (few matrices: the dependency waits decide the
order), and a nine-iteration chain (27 products: two chain launches).
"""
import os
import subprocess
import sys
import tempfile

import pytest
import torch

import newton_schulz_matrix_b200 as nsm
import synth

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
Q = (3.4445, -4.7750, 2.0315)

STEP_CASES = {
    "merged-bf16": dict(spec=[(256, 640), (256, 640), (640, 256)], wdt="bfloat16", mode="standard", compute="fp16"),
    "ragged-fp32-fp16": dict(spec=[(300, 1001), (1001, 300)], wdt=["float32", "float16"], mode="standard",
                             compute="bf16"),
    "gram-fp16": dict(spec=[(512, 1536), (1536, 512)], wdt="float16", mode="gram_stabilized", compute="fp16"),
    "nan-flag": dict(spec=[(384, 768), (384, 768), (768, 384)], wdt="bfloat16", mode="standard", compute="fp16",
                     nan=1),
}
NS_CASES = {
    "standard-2x": dict(shape=(512, 1408), count=2, mode="standard"),
    "gram-1x": dict(shape=(768, 1024), count=1, mode="gram"),
    "stabilized-5x": dict(shape=(256, 2048), count=5, mode="gram_stabilized"),
    "periodic-3x": dict(shape=(384, 1152), count=3, mode="gram_stabilized", restart_every=2),
    "nine-iterations": dict(shape=(1024, 1024), count=3, mode="standard", iters=9),
}


def run_case(name):
    """Seeded inputs on cuda:0; returns the tensors the case writes and its status words."""
    if name in STEP_CASES:
        c = STEP_CASES[name]
        W, G, M = [], [], []
        for i, (r, k) in enumerate(c["spec"]):
            wdt = c["wdt"][i] if isinstance(c["wdt"], list) else c["wdt"]
            W.append(synth.gaussian(r, k, 100 + i, "cuda", std=0.05).to(getattr(torch, wdt)))
            G.append(synth.gaussian(r, k, 200 + i, "cuda").bfloat16())
            M.append(synth.gaussian(r, k, 300 + i, "cuda", std=0.2))
        if "nan" in c:
            G[c["nan"]][3, 5] = float("nan")
        st = torch.full((len(W),), -1, dtype=torch.int32, device="cuda")
        nsm.muon_step(W, G, M, status=st, mode=c["mode"], compute_dtype=c["compute"])
        out = W + M
    else:
        c = NS_CASES[name]
        out = [synth.gaussian(*c["shape"], seed=500 + i, device="cuda", dtype=torch.bfloat16) for i in range(c["count"])]
        st = torch.full((len(out),), -1, dtype=torch.int32, device="cuda")
        nsm.muon_ns_batched(out, coeffs=[Q] * c.get("iters", 5), mode=c["mode"], status=st,
                            restart_every=c.get("restart_every", 0))
    torch.cuda.synchronize()
    return [t.cpu() for t in out], st.cpu()


def _bits(t):
    """The tensor's bit pattern (NaN compares equal to the same NaN)."""
    return t.view({1: torch.int8, 2: torch.int16, 4: torch.int32}[t.element_size()])


def _in_child(name, env, path):
    code = ("import sys, torch; sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r});"
            "import test_gpu_launch_modes as t; torch.save(t.run_case({name!r}), {path!r})").format(
        root=ROOT, tests=os.path.join(ROOT, "tests"), name=name, path=path)
    subprocess.run([sys.executable, "-c", code], check=True, env=dict(os.environ, **env), cwd=ROOT, timeout=600)
    return torch.load(path)


SWITCHES = [{"MUON_CHAIN": "1"}, {"MUON_FUSED_UPDATE": "0"}, {"MUON_FUSED_UPDATE": "1"}, {"MUON_PDL": "0"},
            {"MUON_TILE_ORDER": "static"}, {"MUON_CHAIN": "1", "MUON_FUSED_UPDATE": "1", "MUON_PDL": "0"}]
MODE_VARS = ("MUON_CHAIN", "MUON_FUSED_UPDATE", "MUON_PDL", "MUON_TILE_ORDER")


@pytest.mark.parametrize("name", sorted(STEP_CASES) + sorted(NS_CASES))
def test_every_launch_mode_gives_the_same_bits(name):
    assert not any(k in os.environ for k in MODE_VARS)  # this process runs the defaults
    got, st = run_case(name)
    if name in STEP_CASES and "nan" in STEP_CASES[name]:
        bad = STEP_CASES[name]["nan"]
        assert st.tolist() == [1 if i == bad else 0 for i in range(len(st))]
    else:
        assert st.tolist() == [0] * len(st)
    with tempfile.TemporaryDirectory() as d:
        for i, env in enumerate(SWITCHES):
            ref, st0 = _in_child(name, env, os.path.join(d, f"ref{i}.pt"))
            assert torch.equal(st, st0), env
            for a, b in zip(got, ref):
                assert a.dtype == b.dtype and torch.equal(_bits(a), _bits(b)), env


def test_profile_of_a_default_step():
    """A default 16-bit step launches its products separately (no chain) and
    runs the update as configured by default."""
    W = [synth.gaussian(512, 1024, 5, "cuda").bfloat16()]
    G = [synth.gaussian(512, 1024, 6, "cuda").bfloat16()]
    M = [torch.zeros(512, 1024, device="cuda")]
    nsm.muon_profile_begin()
    nsm.muon_step(W, G, M)
    prof = {r["kernel"]: r for r in nsm.muon_profile_end()}
    assert "tc_chain" not in prof
    assert prof["tc_product"]["launches"] == 5 and prof["tc_product[symmetric]"]["launches"] == 10
    flops = prof["tc_product"]["flops"] + prof["tc_product[symmetric]"]["flops"]
    assert flops == pytest.approx(nsm.muon_ns_flops(512, 1024), rel=1e-12)


def test_fp32_operand_splits_are_reused():
    """An fp32 chain with n >= 256 reads its operands as TF32 hi/lo planes
    written by split_tf32_kernel, once per buffer content: per standard
    iteration X (reused by the update product X <- aX + BX), A and B, at
    12 bytes per element (x read, hi and lo written)."""
    n, m, count, iters = 512, 1024, 2, 5
    X = [synth.gaussian(n, m, 40 + i, "cuda") for i in range(count)]
    nsm.muon_profile_begin()
    nsm.muon_ns_batched(X, compute_dtype="fp32")
    prof = {r["kernel"]: r for r in nsm.muon_profile_end()}
    assert prof["tc_product[3xtf32]"]["launches"] == 3 * iters
    split = prof["split_tf32_kernel"]
    assert split["launches"] == 3 * iters
    elems_per_iter = count * (n * m + 2 * n * n)
    assert split["bytes"] == pytest.approx(12.0 * elems_per_iter * iters, rel=1e-12)
    assert all(torch.isfinite(x).all() for x in X)
