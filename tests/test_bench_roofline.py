"""bench.py's roofline bookkeeping (CPU): the bound is the resource whose
roofline time is longer, and the fractions are the achieved rates over the
measured peaks.  The expected values are those of bench lines measured on a
B200 (memory-bound and variable-length workloads)."""
import pytest

import bench

HBM, TC_BURST, TC_SUS = 6541.5, 1617.9, 1374.1


def test_memory_bound_workload_is_hbm_bound():
    r = bench.attention_roofline(603_979_776, 18_253_611_008, 0.12698, HBM, TC_BURST, TC_SUS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == HBM
    assert r["achieved"] == pytest.approx(4756.5, abs=0.1)
    assert r["frac"] == pytest.approx(0.7271, abs=1e-4)


def test_varlen_workload_sits_on_the_ridge():
    # 313.6 MB at the copy bandwidth (47.9 us) outlasts 75.8 GFLOP at the
    # burst GEMM rate (46.9 us) by a hair: the slower roofline is the HBM one,
    # and the tensor fraction is reported beside it
    r = bench.attention_roofline(313_598_592, 75_821_170_688, 0.13011, HBM, TC_BURST, TC_SUS)
    assert r["bound"] == "hbm" and r["peak"] == HBM
    assert r["frac"] == pytest.approx(0.3684, abs=1e-4)
    assert r["tensor_frac"] == pytest.approx(0.3602, abs=1e-4)


def test_mtp_workload_is_tensor_bound():
    # the timed loops last milliseconds: the fraction is of the burst peak,
    # the sustained (power-capped) one is reported beside it
    r = bench.attention_roofline(2_491_416_576, 1_204_698_079_232, 1.742, HBM, TC_BURST, TC_SUS)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == TC_BURST
    assert r["frac"] == pytest.approx(0.4274, abs=1e-4)
    assert r["frac_of_sustained_peak"] == pytest.approx(r["achieved"] / TC_SUS, abs=1e-3)


def test_bound_flips_where_the_roofline_times_cross():
    # 1 GB at 6541.5 GB/s takes as long as F FLOPs at 1617.9 TFLOP/s
    f_cross = 1e9 / (HBM * 1e9) * TC_BURST * 1e12
    assert bench.attention_roofline(10 ** 9, int(f_cross * 0.99), 1.0, HBM, TC_BURST, TC_SUS)["bound"] == "hbm"
    assert bench.attention_roofline(10 ** 9, int(f_cross * 1.01), 1.0, HBM, TC_BURST, TC_SUS)["bound"] == "tensor"


def test_traffic_figures_belong_to_the_current_kernels():
    # the captured traffic figures are tied to the sources they were captured
    # with: after a kernel change, capture again (and record the new digest)
    # or set the entries to None
    for kernel, digest in bench.ATTN_TRAFFIC_SOURCE_SHA256.items():
        assert bench.kernel_sources_sha256(kernel) == digest, kernel
    assert bench.attn_traffic("C2", "mla_decode_kernel") == bench.ATTN_TRAFFIC_BYTES["C2"]
    assert bench.attn_traffic("C5", "mla_decode_fp8_kernel") == bench.ATTN_TRAFFIC_BYTES["C5"]


def test_stale_traffic_is_reported_as_null(monkeypatch):
    monkeypatch.setitem(bench.ATTN_TRAFFIC_SOURCE_SHA256, "mla_decode_kernel", "0" * 64)
    assert bench.attn_traffic("C2", "mla_decode_kernel") is None
    assert bench.attn_traffic("C5", "mla_decode_fp8_kernel") == bench.ATTN_TRAFFIC_BYTES["C5"]
