"""bench.py's measurement arithmetic on the host (CPU only, no GPU).

The FLOP counts are the algorithmic ones of the block (2 x contraction per
output element, three GEMM passes per layer for fwd+bwd), checked against
closed forms; the per-kernel breakdown adds up to the step; the workload
table holds the five configurations the block is measured on.
"""

import pytest

import bench


def test_step_flops_closed_forms():
    s7 = bench.WORKLOADS["7B"][1]
    M, K, d, F = s7["M"], s7["K"], s7["d"], s7["F"]
    assert bench._flops("grg", s7, True) == pytest.approx(6.0 * M * d * (K + 2 * F))
    assert bench._flops("grg", s7, True) == pytest.approx(5.257e12, rel=1e-3)
    assert bench._flops("grg", bench.WORKLOADS["70B"][1], True) == pytest.approx(13.19e12, rel=1e-3)
    s1 = bench.WORKLOADS["1B"][1]
    assert bench._flops("grg", s1, False) == pytest.approx(2.0 * 8192 * 2048 * (2048 + 2 * 8192))
    sw = bench.WORKLOADS["swiglu"][1]
    assert bench._flops("swiglu", sw, True) == pytest.approx(18.0 * 16384 * 4096 * 14336)
    sx = bench.WORKLOADS["xent"][1]
    assert bench._flops("xent", sx, True) == pytest.approx(3 * 2.0 * 8192 * 4096 * 128256)


def test_kernel_breakdown_adds_up_to_the_step():
    for name in ("tiny", "7B", "70B"):
        kind, s, bwd = bench.WORKLOADS[name]
        ks = bench._grg_kernels(s, bwd)
        tensor = sum(a for _, _, bound, a in ks if bound == "tensor")
        assert tensor == pytest.approx(bench._flops(kind, s, bwd)), name
        fold = [a for kid, _, _, a in ks if kid == 16][0]
        assert fold == 4.0 * (2 * s["F"]) * s["d"] + 2.0 * s["d"]
        assert len(ks) == (9 if bwd else 3)  # the row reduce runs in the gate/up GEMM's epilogue


def test_workload_table_matches_the_configurations():
    w = bench.WORKLOADS
    assert w["tiny"][1] == dict(M=256, K=512, d=512, F=1024, eps=1e-6) and w["tiny"][2]
    assert (w["1B"][1]["M"], w["1B"][1]["d"], w["1B"][1]["F"], w["1B"][2]) == (8192, 2048, 8192, False)
    assert (w["7B"][1]["M"], w["7B"][1]["d"], w["7B"][1]["F"], w["7B"][2]) == (8192, 4096, 11008, True)
    assert (w["70B"][1]["M"], w["70B"][1]["d"], w["70B"][1]["F"], w["70B"][1]["eps"]) == (4096, 8192, 28672, 1e-5)
    assert (w["swiglu"][1]["M"], w["swiglu"][1]["d"], w["swiglu"][1]["F"]) == (16384, 4096, 14336)


def test_replica_throughput_and_source_hash():
    # 2 ranks, each 5.257 TFLOP per step, 10 steps, slowest rank 50 ms -> 2102.8 TFLOP/s
    assert bench.replica_throughput(5.257e12, 10, 2, 50.0) == pytest.approx(2102.8)
    h = bench._kernel_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0


def test_clock_summary_from_nvml_samples():
    """Median SM clock over the samples under load, the maximum clock, and the
    clock-event reasons named from NVML's bits."""
    c = bench.ClockSampler(0)
    c.rows = [(1965.0, 1965.0, 90.0, 0x1),          # idle sample before the region: not under load
              (1800.0, 1965.0, 980.0, 0x4),         # sw power cap
              (1700.0, 1965.0, 1000.0, 0x4 | 0x8),  # + hw slowdown
              (1750.0, 1965.0, 990.0, 0x0)]
    s = c.summary()
    assert s["sm_mhz"] == 1750.0 and s["sm_max_mhz"] == 1965.0
    assert s["samples"] == 4 and s["samples_under_load"] == 3
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"] and s["source"] == "nvml"
    assert bench.ClockSampler(0).summary()["samples"] == 0
