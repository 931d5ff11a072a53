"""Host-side logic of bench.py, on CPU: the kernel names it reports, its launch count per step
(against the launch list ncu recorded for the 15k-history step: 82 launches), its algorithmic
work model (against the FLOP count worked out by hand), the parser of the clock samples taken
during the timed region, and the oracle sampler behind `cpu_baseline` and the reference arm."""
import importlib.util
import os
import statistics

import pytest

from wukong_hstu_cross_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_kernel_name_demangles_the_library_kernels(bench):
    assert bench.kernel_name("_ZN5whale17abs_scores_kernelILi2EEEv14CUtensorMap_stS1_S1_NS_7AbsArgsE") == \
        "abs_scores_kernel<2>"
    assert bench.kernel_name("_ZN5whale14gemm_tc_kernelILi64ELi2ELb0ELb1EEEv14CUtensorMap_stS1_S1_S1_S1_NS_8GemmArgsE") \
        == "gemm_tc_kernel<64,2,0,1>"
    assert bench.kernel_name("_ZN5whale16abs_merge_kernelENS_7AbsArgsE") == "abs_merge_kernel"
    assert bench.kernel_name("not_mangled") == "not_mangled"


def test_launches_per_step_matches_the_recorded_launch_list(bench):
    # one step of the 15k-history stack under ncu: residual set-up, unit starts, then per layer the
    # Q GEMM, qa GEMM, pass A, pass B, merge, W_V GEMM, two Fusion GEMMs, up|gate and down GEMMs
    w = I.WORKLOADS["hist15k_d512"]
    assert bench.launches_per_step(w, fold_per_call=False, absorbed=True) == 82
    assert bench.launches_per_step(w, fold_per_call=True, absorbed=True) == 90


def test_step_work_absorbed_attention_flops_by_hand(bench):
    w = I.WORKLOADS["hist15k_d512"]
    total_L = 403481
    work = bench.step_work(w, total_L, absorbed=True)
    # scores and weighted sums of 256 absorbed queries over every row: 2 x 2 x 256 x 403481 x 512;
    # the per-head query and output GEMMs: 2 x 2 x 2048 x 512 x 512
    assert work["attention_absorbed"]["flops"] == 2 * 2 * 256 * 403481 * 512 + 2 * 2 * 2048 * 512 * 512
    assert abs(work["attention_absorbed"]["flops"] / 1e9 - 213.69) < 0.01
    # the states read once in bf16 dominate the bytes: 2 x 403481 x 512
    assert work["attention_absorbed"]["bytes"] == 2 * (403481 * 512 + 2 * 2048 * 512 + 2 * 512 * 512)


def test_clock_sampler_summary(bench, tmp_path):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    s.proc = object()  # as if nvidia-smi had been started
    rows = ["0, 1680, 1965, 812.5, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1710, 1965, 830.1, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1620, 1965, 790.0, 0x0, Not Active, Not Active, Not Active, Not Active",
            "garbage line"]
    with open(s.path, "w") as fh:
        fh.write("\n".join(rows) + "\n")
    r = s.summary()
    assert r == {"sm_mhz": statistics.median([1680, 1710, 1620]), "sm_max_mhz": 1965.0,
                 "reasons": ["sw_power_cap"], "samples": 3}
    rows[0] = "0, 1200, 1965, 700.0, 0x8, Active, Not Active, Not Active, Not Active"
    with open(s.path, "w") as fh:
        fh.write("\n".join(rows) + "\n")
    assert bench.ClockSampler.summary(s)["reasons"] == ["hw_slowdown", "sw_power_cap"]
    s.proc = None  # nvidia-smi unavailable: no clock record
    assert s.summary() is None


def test_oracle_sampler_counts_whole_examples(bench):
    w = I.WORKLOADS["tiny_fp32"]
    s = bench.OracleSampler(w)
    s.run(0.0, max_examples=2)  # at least one example even with no time budget
    assert s.done >= 1 and s.t > 0.0
    out = s.summary("first examples")
    assert out["unit"] == "examples/s" and out["kind"] == "oracle" and out["cores"] >= 1
    assert out["value"] == pytest.approx(s.done / s.t)
    # the time budget ends a run (after one example at least); max_examples caps it; the sampler
    # walks the whole batch in order and starts again at example 0
    c = bench.OracleSampler(w)
    c.run(60.0, max_examples=3)
    assert c.done == 3 and c.next_b == 3 % w.batch
    assert len(c.step_s) == 1 and c.step_s[0] == pytest.approx(c.t)
    c.run(60.0, max_examples=2, count=False)  # an untimed warm-up run leaves the counts alone
    assert c.done == 3 and len(c.step_s) == 1


def test_roofline_bound_is_the_larger_algorithmic_time(bench):
    # pass A at the 15k-history batch: 105.8 GFLOP and 413 MB in 129.9 us against the burst figures
    fa, ba = 2.0 * 256 * 403481 * 512, 2.0 * 403481 * 512
    r = bench.roofline_of(fa, ba, 0.1299, 1717.8, 6456.5)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["frac"] == pytest.approx(ba / 6456.5e9 / 129.9e-6)
    assert r["achieved"] / r["peak"] == pytest.approx(r["frac"])
    # against the sustained figure the FLOP time is the larger one
    r2 = bench.roofline_of(fa, ba, 0.1299, 1424.0, 6456.5)
    assert r2["bound"] == "tensor" and r2["frac"] == pytest.approx(fa / 1424e12 / 129.9e-6)


def test_tensor_peak_follows_the_sampled_clock(bench):
    peaks = {"bf16_tflops": 1717.8, "bf16_tflops_sustained": 1424.0, "sm_max_mhz": 1965.0, "hbm_gbs": 6456.5}
    assert bench.tensor_peak(peaks, {"sm_mhz": 1965.0})[0] == 1717.8
    assert bench.tensor_peak(peaks, {"sm_mhz": 1372.0})[0] == 1424.0
    assert bench.tensor_peak(peaks, None)[0] == 1717.8
