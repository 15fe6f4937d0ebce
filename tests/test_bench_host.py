"""Host logic of bench.py (no GPU): the roofline built from the library's
per-launch profile, for the 16-bit product kernels and for the 3xTF32 ones,
and the weak-scaling aggregate."""
import pytest

import bench

PEAKS = {"bf16_tflops": 1637.0, "bf16_tflops_sustained": 1386.2, "hbm_gbs": 6543.4}


def _prof(kernel, launches, ms, flops, exec_flops=None, nbytes=0.0):
    return {"kernel": kernel, "launches": launches, "ms": ms, "flops": flops,
            "exec_flops": flops if exec_flops is None else exec_flops, "bytes": nbytes}


def test_16_bit_roofline_takes_the_dominant_class_at_its_executed_flops():
    # symmetric products execute only their upper-triangle tiles: 36 of 64 at n = 2048
    prof = [_prof("pack_kernel", 6, 30.0, 0.0, nbytes=118.9e9),
            _prof("tc_product[symmetric]", 30, 140.0, 290e12, exec_flops=290e12 * 36 / 64),
            _prof("tc_product", 15, 200.0, 223e12),
            _prof("tc_product[3xtf32]", 5, 50.0, 1e12)]
    r = bench.roofline_from_profile(prof, PEAKS, "measured", "kimi-k2", "fp16")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["kernel"] == "tc_product"                       # most device time
    assert r["achieved"] == pytest.approx(223e12 / 0.200 / 1e12, rel=1e-3)
    assert r["peak"] == PEAKS["bf16_tflops_sustained"]
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-3) and r["frac"] < 1
    assert r["per_launch_ms"] == pytest.approx(200.0 / 15, rel=1e-3)
    by = {x["kernel"]: x for x in r["by_kernel"]}
    sym = by["tc_product[symmetric]"]
    assert sym["executed_tflops"] == pytest.approx(290e12 * 36 / 64 / 0.140 / 1e12, rel=1e-3)
    assert sym["algorithmic_tflops"] == pytest.approx(290e12 / 0.140 / 1e12, rel=1e-3)
    assert by["pack_kernel"]["bound"] == "hbm"
    assert by["pack_kernel"]["gbs"] == pytest.approx(118.9e9 / 0.030 / 1e9, rel=1e-3)
    assert by["pack_kernel"]["frac"] == pytest.approx(by["pack_kernel"]["gbs"] / PEAKS["hbm_gbs"], rel=1e-3)


def test_fp32_roofline_counts_three_tf32_mmas_against_the_tf32_peak():
    prof = [_prof("tc_product[symmetric]", 3, 1.0, 1e12),
            _prof("tc_product[3xtf32]", 15, 40.0, 6.2e12, exec_flops=3 * 6.4e12),
            _prof("gemm_simt_kernel", 10, 1.0, 1e9)]
    r = bench.roofline_from_profile(prof, PEAKS, "measured", "dense", "fp32")
    assert r["kernel"] == "tc_product[3xtf32]"
    assert r["algorithmic_tflops"] == pytest.approx(6.2e12 / 0.040 / 1e12, rel=1e-3)
    assert r["achieved"] == pytest.approx(3 * 6.4e12 / 0.040 / 1e12, rel=1e-3)
    assert r["peak"] == pytest.approx(PEAKS["bf16_tflops"] * 1.1 / 2.25, abs=0.1)


def test_roofline_is_absent_without_product_launches():
    assert bench.roofline_from_profile([_prof("pack_kernel", 1, 1.0, 0.0)], PEAKS, "measured", "single", "fp32") is None


def test_traffic_is_reported_only_for_a_capture_of_the_current_kernel_source(monkeypatch):
    prof = [_prof("tc_product", 1, 1.0, 1e12)]
    assert bench.roofline_from_profile(prof, PEAKS, "measured", "moe", "fp16")["traffic"] is None
    h = bench.kernel_source_hash("tc_product")
    assert h and h == bench.kernel_source_hash("tc_product[symmetric]")
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("moe", "fp16", "tc_product"), (h, 1.5e9))
    assert bench.roofline_from_profile(prof, PEAKS, "measured", "moe", "fp16")["traffic"] == 1.5e9
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("moe", "fp16", "tc_product"), ("0" * 16, 1.5e9))
    assert bench.roofline_from_profile(prof, PEAKS, "measured", "moe", "fp16")["traffic"] is None


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


def test_a_chain_launch_is_a_tensor_class_of_its_own():
    prof = [_prof("pack_kernel", 6, 30.0, 0.0, nbytes=118.9e9),
            _prof("tc_chain", 3, 380.0, 513e12, exec_flops=420e12),
            _prof("status_or_kernel", 6, 0.1, 0.0, nbytes=1e3)]
    r = bench.roofline_from_profile(prof, PEAKS, "measured", "kimi-k2", "fp16")
    assert r["kernel"] == "tc_chain"
    assert r["achieved"] == pytest.approx(420e12 / 0.380 / 1e12, rel=1e-3)
    assert r["algorithmic_tflops"] == pytest.approx(513e12 / 0.380 / 1e12, rel=1e-3)
