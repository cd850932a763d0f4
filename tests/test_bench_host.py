"""Host-side logic of bench.py that needs no GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_linear_bytes_counts_codes_scales_zeros_and_vectors():
    # N x K/2 packed codes, two bf16 parameters per group, bf16 x and y
    assert bench.linear_bytes(1, 256, 1024) == 256 * 512 + 2 * 2 * 256 * 8 + 2 * 1024 + 2 * 256
    assert bench.linear_bytes(128, 8192, 8192) == 8192 * 4096 + 4 * 8192 * 64 + 2 * 128 * 8192 * 2


def test_traffic_is_reported_only_for_the_profiled_sources(tmp_path, monkeypatch):
    src = [tmp_path / "a.cu", tmp_path / "b.cuh"]
    for i, p in enumerate(src):
        p.write_text(f"kernel source {i}\n")
    prof = tmp_path / "prof.txt"
    monkeypatch.setattr(bench, "M1_SOURCES", [str(p) for p in src])
    monkeypatch.setattr(bench, "M1_PROFILE", str(prof))
    h = bench.kernel_source_hash([str(p) for p in src])
    prof.write_text(f"header\ntraffic_per_launch_bytes: 123456\nkernel_source_sha256: {h}\n")
    assert bench.m1_traffic_per_launch() == 123456
    src[1].write_text("kernel source changed\n")
    assert bench.m1_traffic_per_launch() is None
    prof.unlink()
    assert bench.m1_traffic_per_launch() is None


def test_clock_summary_flags_throttle_reasons():
    c = bench.Clocks(0)
    c.out = ("0, 1965, 1965, 700.5, 0x0, Not Active, Not Active, Not Active, Active\n"
             "0, 1950, 1965, 710.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
             "0, 1965, 1965, 120.0, 0x0, Active, Not Active, Not Active, Not Active\n")
    s = c.summary()
    assert s["samples"] == 2  # the idle sample (power <= 200 W) is not under load
    assert s["reasons"] == ["sw_power_cap"]
    assert s["sm_max_mhz"] == 1965.0


def test_workload_config_counts_the_model():
    c = bench.workload_config(80)
    assert c["linears_per_step"] == 320 and c["layers"] == 80
    assert c["weights"] == 80 * (8192 * 10240 + 8192 * 8192 + 8192 * 57344 + 28672 * 8192)
    assert c["bytes_per_step"] == 80 * sum(bench.linear_bytes(1, N, K) for K, N in
                                           ((8192, 10240), (8192, 8192), (8192, 57344), (28672, 8192)))


def test_both_arms_describe_the_same_workload():
    """The reference arm's config is workload_config; the GPU arm spells the same keys out in its line."""
    import inspect
    src = inspect.getsource(bench.main)
    c = bench.workload_config(80)
    for key in c:
        assert f'"{key}"' in src, key
    assert "W4A16 g128 bf16 s/z, M=1" in c["workload"] and "W4A16 g128 bf16 s/z, M=1" in src
