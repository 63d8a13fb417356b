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
    for config, (nbytes, src, sha) in bench.MEASURED_TRAFFIC.items():
        value = bench.decode_traffic(config)
        assert value == (nbytes if bench.kernel_source_digest(src) == sha else None)


def test_cpu_model_is_text():
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()


def test_nonabsorbed_sample_extrapolates_by_tokens_and_heads():
    r = bench.oracle_nonabsorbed_sample("tiny", budget_s=0.5)
    assert r["us_per_token_head"] > 0
    # tiny: one sequence of 256 cached tokens, 16 heads, one query
    est = r["us_per_token_head"] * 256 * 16 * 1e-6
    assert abs(r["extrapolated_full_s"] - est) <= 1e-3 * est + 1e-4
    assert "extrapolated" in r["sample"]


def test_tensor_peak_follows_the_mma_kind():
    peaks = {"bf16_tflops": 1640.7, "hbm_gbs": 6550.4}
    assert bench.tensor_peak(peaks, "bf16")[0] == 1640.7
    # e4m3 x e4m3: the measured bf16 figure x the nominal fp8 / bf16 ratio (4.5 / 2.25)
    assert bench.tensor_peak(peaks, "fp8")[0] == 2 * 1640.7
    assert bench.tensor_peak(dict(peaks, fp8_tflops=3100.0), "fp8")[0] == 3100.0
    f = bench.datasheet_fracs(608.2e6, 584.1e9, 1e-3, "fp8")
    assert abs(f["tensor_frac"] - 584.1e9 / 4500e12 / 1e-3) < 1e-6
