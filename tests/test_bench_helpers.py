"""Host-side helpers of bench.py (CPU): secondary roofline denominators, the
measured-traffic record, the CPU description."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_datasheet_fractions():
    # V3: 302 MB of cache and 73 GFLOP; at 100 us the memory side binds
    f = bench.datasheet_fracs(302.0e6, 73.0e9, 100e-6)
    assert abs(f["hbm_frac"] - 302.0e6 / 7700e9 / 100e-6) < 1e-4
    assert abs(f["tensor_frac"] - 73.0e9 / 2250e12 / 100e-6) < 1e-4
    assert f["binding_frac"] == max(f["hbm_frac"], f["tensor_frac"])
    # a tensor-bound case
    g = bench.datasheet_fracs(1e6, 1e12, 1e-3)
    assert g["binding_frac"] == g["tensor_frac"]


def test_traffic_reported_only_for_the_profiled_source():
    # the record names the sha256 of the kernel source it was measured on; any
    # other source (or workload) gets no traffic figure
    assert bench.decode_traffic("tiny") is None
    value = bench.decode_traffic("v3")
    assert value is None or value == bench.MEASURED_TRAFFIC["v3"][0]


def test_cpu_model_is_text():
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()


def test_nonabsorbed_sample_extrapolates_by_tokens_and_heads():
    r = bench.oracle_nonabsorbed_sample("tiny", budget_s=0.5)
    assert r["us_per_token_head"] > 0
    # tiny: one sequence of 256 cached tokens, 16 heads, one query
    est = r["us_per_token_head"] * 256 * 16 * 1e-6
    assert abs(r["extrapolated_full_s"] - est) <= 1e-3 * est + 1e-4
    assert "extrapolated" in r["sample"]
