"""Host logic of bench.py (no GPU): the roofline built from the library's
per-launch profile, for the 16-bit product kernels and for the 3xTF32 ones,
and the weak-scaling aggregate."""
import pytest

import bench

PEAKS = {"bf16_tflops": 1637.0, "bf16_tflops_sustained": 1386.2, "hbm_gbs": 6543.4}


def _prof(kernel, launches, ms, flops):
    return {"kernel": kernel, "launches": launches, "ms": ms, "flops": flops, "bytes": 0.0}


def test_bf16_roofline_counts_only_the_16_bit_product_kernels():
    prof = [_prof("pack_kernel", 4, 10.0, 0.0),
            _prof("tc_product[symmetric]", 30, 120.0, 150e12),
            _prof("tc_product", 15, 180.0, 363e12),
            _prof("tc_product[3xtf32]", 5, 50.0, 1e12)]
    r = bench.roofline_from_profile(prof, PEAKS, "measured", "kimi-k2", "bf16")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(513e12 / 0.300 / 1e12, rel=1e-3)
    assert r["peak"] == PEAKS["bf16_tflops_sustained"]
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-3)
    assert r["per_launch_ms"] == pytest.approx(300.0 / 45, rel=1e-3)
    assert r["traffic"] == bench.PRODUCT_TRAFFIC_PER_LAUNCH[("kimi-k2", "bf16")]


def test_fp32_roofline_counts_three_tf32_mmas_against_the_tf32_peak():
    prof = [_prof("tc_product[symmetric]", 3, 1.0, 1e12),
            _prof("tc_product[3xtf32]", 15, 40.0, 6.2e12),
            _prof("mirror_upper_kernel", 10, 1.0, 0.0)]
    r = bench.roofline_from_profile(prof, PEAKS, "measured", "dense", "fp32")
    assert r["algorithmic_tflops"] == pytest.approx(6.2e12 / 0.040 / 1e12, rel=1e-3)
    assert r["achieved"] == pytest.approx(3 * r["algorithmic_tflops"], rel=1e-3)
    assert r["peak"] == pytest.approx(PEAKS["bf16_tflops"] * 1.1 / 2.25, abs=0.1)
    assert r["traffic"] == bench.PRODUCT_TRAFFIC_PER_LAUNCH[("dense", "fp32")]


def test_roofline_is_absent_without_product_launches():
    assert bench.roofline_from_profile([_prof("pack_kernel", 1, 1.0, 0.0)], PEAKS, "measured", "single", "fp32") is None


def test_traffic_is_only_reported_for_captured_workloads():
    prof = [_prof("tc_product", 1, 1.0, 1e12)]
    assert bench.roofline_from_profile(prof, PEAKS, "measured", "moe", "bf16")["traffic"] is None
    assert bench.roofline_from_profile(prof, PEAKS, "measured", "kimi-k2", "fp16")["traffic"] is None


def test_weak_scaling_value_is_all_ranks_work_over_the_slowest_step():
    assert bench.whole_job_tflops(4, 513.2e12, 400.0) == pytest.approx(4 * 513.2e12 / 0.4 / 1e12)
    assert bench.max_over_ranks(12.5, None, None) == 12.5


def test_streamed_slices_take_the_widest_short_side_first_and_respect_the_budget():
    from newton_schulz_matrix_b200 import plan_slices
    shapes = [(2048, 7168)] * 3 + [(7168, 2048)] + [(7168, 18432)] * 2 + [(64, 128)]
    nbytes = [r * c * 2 for r, c in shapes]
    slices = plan_slices(shapes, nbytes, 64 << 20)
    flat = [i for sl in slices for i in sl]
    assert sorted(flat) == list(range(len(shapes)))              # every tensor exactly once
    assert flat[:2] == [4, 5]                                    # n = 7168 first
    assert flat[-1] == 6                                         # the 64 x 128 matrix last
    for sl in slices:                                            # budget, or a single oversized tensor
        assert len(sl) == 1 or sum(nbytes[i] for i in sl) <= 64 << 20
    assert [len(sl) for sl in slices] == [1, 1, 2, 3]             # 29 MB experts pair up (the small one joins); 264 MB dense alone
    assert plan_slices([], [], 1) == []
