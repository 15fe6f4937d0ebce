"""The seeded input recipes (CPU): each workload has the shapes and value
structure the configurations state, and every draw is reproducible from its
seed.  The oracle and the CUDA path both take their inputs from here, so these
checks pin what both sides are fed."""
import math

import numpy as np
import torch

import synth


def _sv(x: torch.Tensor) -> np.ndarray:
    return np.linalg.svd(x.double().numpy(), compute_uv=False)


def test_draws_are_reproducible_and_seed_dependent():
    a = synth.gaussian(32, 48, 5)
    assert torch.equal(a, synth.gaussian(32, 48, 5))
    assert not torch.equal(a, synth.gaussian(32, 48, 6))
    assert torch.equal(synth.log_uniform_sigma(16, 1e-6, 1.0, 3), synth.log_uniform_sigma(16, 1e-6, 1.0, 3))
    assert torch.equal(synth.stress_point(16, 2, count=2)[1], synth.stress_point(16, 2, count=2)[1])


def test_haar_columns_are_orthonormal():
    q = synth.haar(64, 24, 11).double()
    assert torch.allclose(q.T @ q, torch.eye(24, dtype=torch.float64), atol=1e-5)


def test_with_spectrum_imposes_the_singular_values():
    sigma = synth.power_law_sigma(20)
    assert torch.allclose(sigma, 1.0 / torch.arange(1, 21, dtype=torch.float32))
    x = synth.with_spectrum(20, 50, sigma, 4)
    assert np.allclose(_sv(x), np.sort(sigma.double().numpy())[::-1], rtol=1e-4, atol=1e-6)


def test_log_uniform_sigma_spans_its_range_in_log_space():
    s = synth.log_uniform_sigma(4000, 1e-6, 1.0, 2).double()
    assert float(s.min()) >= 1e-6 * (1 - 1e-6) and float(s.max()) <= 1.0
    logs = torch.log10(s)
    assert abs(float(logs.mean()) + 3.0) < 0.1          # uniform on [-6, 0]: mean -3
    assert abs(float(logs.std()) - 6 / math.sqrt(12)) < 0.1


def test_dense_projection_gradients_are_rank_64_plus_noise():
    w = synth.dense_projection(count=2, rows=128, cols=256)
    g = w.groups[0]
    assert (g.rows, g.cols, g.count) == (128, 256, 2)
    sv = _sv(g.G[0].float())
    assert sv[63] / sv[64] > 3                            # 64 dominant directions over a 0.1 noise floor
    assert float(g.M[0].abs().max()) == 0.0 and g.G[0].dtype == torch.bfloat16


def test_moe_layer_shapes_and_power_law_spectrum():
    w = synth.moe_layer(experts=2, inter=48, hidden=80, shared=1)
    assert [(g.rows, g.cols, g.count) for g in w.groups] == [(48, 80, 4), (80, 48, 2), (80, 80, 1)]
    sv = _sv(w.groups[1].G[0].float())
    assert np.allclose(sv, 1.0 / np.arange(1, 49), rtol=2e-2, atol=2e-3)  # bf16 storage of 1/i on Haar bases
    assert abs(float(w.groups[0].W[0].float().std()) - 0.02) < 0.004


def test_kimi_k2_shape_set_and_entry_scales():
    w = synth.kimi_k2(counts=[1, 1, 0, 0])
    assert [(g.rows, g.cols) for g in w.groups] == [(2048, 7168), (7168, 2048)]
    g = w.groups[0]
    assert abs(float(g.M[0].std()) - 1e-3) < 1e-6          # rescaled to entry std 1e-3
    assert abs(float(g.G[0].float().std()) - 1e-3) < 2e-5
    assert abs(float(g.W[0].float().std()) - 0.02) < 4e-4
    full = synth.kimi_k2(counts=[0, 0, 0, 0], experts=216)
    assert full.groups == []


def test_stress_point_spectrum_lies_in_the_stated_band():
    x = synth.stress_point(24, 2, count=1)[0].float()
    assert tuple(x.shape) == (24, 48)
    sv = _sv(x)
    assert sv.max() <= 1.0 + 1e-2 and sv.min() >= 1e-6 * 0.5
