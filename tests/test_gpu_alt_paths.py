"""Alternative product paths, chosen by switches read when the library loads.

MUON_FP32_TC=0 runs every fp32 product on the CUDA-core kernel instead of
3xTF32 on the tensor cores; MUON_FUSED_SMALL=0 runs the chain of a small fp32
matrix as separate products instead of the one-launch fused chain;
MUON_GEMM_PAIR=0 runs every 16-bit product on the 1-CTA tensor-core kernel
(which also moves the Muon update from the last product's epilogue into the
separate update pass).  Each case runs in a child process with its switch set
and is checked against the fp64 oracle with the parity bar of its chain type:
1e-4 relative Frobenius error for fp32, 2e-2 and the sigma band for fp16.
"""
import math
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

import newton_schulz_matrix_b200 as nsm
import oracle
import synth
from parity_util import Q5, rel, sigma_band_error, to_np, tolerance

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

NS_CASES = {
    "fp32-tc-standard": dict(shape=(512, 1024), count=2, mode="standard", compute="fp32", env={"MUON_FP32_TC": "0"}),
    "fp32-tc-stabilized": dict(shape=(512, 256), count=2, mode="gram_stabilized", compute="fp32",
                               env={"MUON_FP32_TC": "0"}),
    "fp32-small-standard": dict(shape=(64, 128), count=3, mode="standard", compute="fp32",
                                env={"MUON_FUSED_SMALL": "0"}),
    "fp32-small-stabilized": dict(shape=(96, 200), count=2, mode="gram_stabilized", compute="fp32",
                                  env={"MUON_FUSED_SMALL": "0"}),
    "fp16-1cta-standard": dict(shape=(512, 1408), count=2, mode="standard", compute="fp16",
                               env={"MUON_GEMM_PAIR": "0"}),
    "fp16-1cta-stabilized": dict(shape=(1024, 768), count=2, mode="gram_stabilized", compute="fp16",
                                 env={"MUON_GEMM_PAIR": "0"}),
}
STEP_SPEC = [(256, 640), (640, 256), (300, 700)]
STEP_HP = dict(lr=0.05, momentum=0.9, nesterov=True, weight_decay=0.2, scale_coef=0.3)


def ns_inputs(name):
    c = NS_CASES[name]
    dt = torch.float32 if c["compute"] == "fp32" else torch.bfloat16
    return [synth.gaussian(*c["shape"], seed=700 + i, device="cuda", dtype=dt) for i in range(c["count"])]


def step_inputs():
    W, G, M = [], [], []
    for i, (r, k) in enumerate(STEP_SPEC):
        W.append(synth.gaussian(r, k, 800 + 3 * i, "cuda", std=0.5))
        G.append(synth.gaussian(r, k, 801 + 3 * i, "cuda").bfloat16())
        M.append(synth.gaussian(r, k, 802 + 3 * i, "cuda", std=0.3))
    return W, G, M


def run_case(name):
    """Runs in the child process: the case's outputs and status words."""
    if name == "fp16-1cta-step":
        W, G, M = step_inputs()
        st = torch.full((len(W),), -1, dtype=torch.int32, device="cuda")
        nsm.muon_step(W, G, M, status=st, mode="standard", compute_dtype="fp16", **STEP_HP)
        out = W + M
    else:
        c = NS_CASES[name]
        out = ns_inputs(name)
        st = torch.full((len(out),), -1, dtype=torch.int32, device="cuda")
        nsm.muon_ns_batched(out, mode=c["mode"], compute_dtype=c["compute"], status=st)
    torch.cuda.synchronize()
    return [t.cpu() for t in out], st.cpu()


def _in_child(name, env):
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "out.pt")
        code = ("import sys, torch; sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r});"
                "import test_gpu_alt_paths as t; torch.save(t.run_case({name!r}), {path!r})").format(
            root=ROOT, tests=os.path.join(ROOT, "tests"), name=name, path=path)
        subprocess.run([sys.executable, "-c", code], check=True, env=dict(os.environ, **env), cwd=ROOT, timeout=600)
        return torch.load(path)


@pytest.mark.parametrize("name", sorted(NS_CASES))
def test_alternative_product_path_matches_the_oracle(name):
    c = NS_CASES[name]
    outs, st = _in_child(name, c["env"])
    assert st.tolist() == [0] * c["count"]
    for U, O in zip(ns_inputs(name), outs):
        U = to_np(U)
        want = oracle.newton_schulz(U, Q5, mode=c["mode"])
        assert np.isfinite(to_np(O)).all()
        assert rel(to_np(O), want) < tolerance(c["compute"]), name
        if c["compute"] != "fp32":
            assert sigma_band_error(U, to_np(O), Q5) < 0.05


def test_muon_step_on_the_1cta_kernel_matches_the_oracle():
    """With MUON_GEMM_PAIR=0 the update runs as the separate pass."""
    outs, st = _in_child("fp16-1cta-step", {"MUON_GEMM_PAIR": "0"})
    assert st.tolist() == [0] * len(STEP_SPEC)
    W0, G0, M0 = step_inputs()
    n = len(STEP_SPEC)
    for i, (r, k) in enumerate(STEP_SPEC):
        Wr, Mr, Or = oracle.muon_step(to_np(W0[i]), to_np(G0[i]), to_np(M0[i]), eps=1e-7, coeffs=Q5,
                                      mode="standard", **STEP_HP)
        assert rel(to_np(outs[n + i]), Mr) < 1e-6
        step = STEP_HP["lr"] * STEP_HP["scale_coef"] * math.sqrt(max(r, k))
        O = ((1 - STEP_HP["lr"] * STEP_HP["weight_decay"]) * to_np(W0[i]) - to_np(outs[i])) / step
        assert rel(O, Or) < tolerance("fp16"), i
