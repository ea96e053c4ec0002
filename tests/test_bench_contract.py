"""Host tests of the bench line's contents (no GPU): the roofline object, the
secondary figures and the workload config that bench.py prints, built from
synthetic timings by the same functions the GPU run uses."""
import pytest

import bench
from block_sparse_attention_29_b200 import workloads

PEAKS = {"hbm_gbs": 6543.4, "bf16_tflops": 1623.7, "bf16_tflops_sustained": 1380.6}
CLOCKS = {"sm_mhz": 1900.0, "sm_max_mhz": 1965, "reasons": [], "samples": 100, "source": "nvml"}


def _prefill_S(flops):
    return dict(metric="effective TFLOP/s (computed blocks)", unit="TFLOP/s", bound="tensor",
                flops=flops, exact_flops=flops * 0.9, dense_flops=flops * 1.5, algo_bytes=1 << 30,
                kernel="prefill_kernel",
                kernel_files=["prefill_sm100.cu", "softmax_util.cuh", "ptx.cuh", "common.h",
                              "pattern_compiler.cu"],
                extra={"blocks_listed": 10})


def test_prefill_line_has_the_roofline_of_the_kernel():
    w = workloads.WORKLOADS["bsfa_causal"]
    flops = 6.6e12
    out = bench.summarize(_prefill_S(flops), w, 1, 10, 3, [8.0] * 10, 80.0, CLOCKS, PEAKS,
                          "measured")
    assert out["unit"] == "TFLOP/s" and out["steps"] == 10 and out["warmup"] == 3
    assert out["ms_per_step"] == pytest.approx(8.0)
    assert out["value"] == pytest.approx(flops / 8e-3 / 1e12, rel=1e-4)
    r = out["roofline"]
    assert set(r) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == 1623.7
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], abs=1e-4)
    # traffic is the committed capture's, present only while the sources still match it
    assert r["traffic"] is None or r["traffic"] > 0
    assert out["clocks"] is CLOCKS
    assert out["secondary"]["pct_bf16_peak_burst"] == pytest.approx(100 * r["frac"], abs=0.01)


def test_value_is_whole_job_over_ranks():
    """N replicas timed by the slowest: the value scales with N at equal time."""
    w = workloads.WORKLOADS["mistral_swa"]
    one = bench.summarize(_prefill_S(1e12), w, 1, 5, 3, [1.0] * 5, 5.0, CLOCKS, PEAKS, "m")
    four = bench.summarize(_prefill_S(1e12), w, 4, 5, 3, [1.0] * 5, 5.0, CLOCKS, PEAKS, "m")
    assert four["value"] == pytest.approx(4 * one["value"], rel=1e-6)
    assert four["roofline"]["achieved"] == pytest.approx(one["roofline"]["achieved"], rel=1e-6)


def test_hbm_bound_line():
    w = workloads.WORKLOADS["gather_decode"]
    S = dict(metric="gather GB/s", unit="GB/s", bound="hbm", flops=0, algo_bytes=2.17e9,
             kernel="gather_kernel", kernel_files=["gather_sm100.cu"], extra={})
    out = bench.summarize(S, w, 1, 10, 3, [0.36] * 10, 3.6, CLOCKS, PEAKS, "measured")
    r = out["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6543.4
    assert r["achieved"] == pytest.approx(2.17e9 / 0.36e-3 / 1e9, rel=1e-4)
    assert out["secondary"]["pct_hbm_peak"] == pytest.approx(100 * r["frac"], abs=0.01)


@pytest.mark.parametrize("name", ["bsfa_causal", "mistral_swa", "longformer_bigbird",
                                  "gather_decode", "window_decode", "topk_decode", "tiny_static"])
def test_config_names_the_workload(name):
    cfg = bench.config_of(workloads.WORKLOADS[name], 1)
    assert cfg["workload"] == name
    assert "model" not in cfg
    assert cfg["l2"].startswith("256 MiB flush")


def test_headline_and_secondary_workloads_exist():
    assert bench.HEADLINE == "bsfa_causal"
    for name in bench.SECONDARY:
        assert name in workloads.WORKLOADS
