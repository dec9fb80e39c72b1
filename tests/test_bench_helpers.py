"""bench.py's host-side helpers (no GPU): the clock record it attaches to a
measurement, the DRAM traffic it takes from a committed ncu capture, and the
algorithmic bytes of a launch."""
import numpy as np

import bench
import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs


class _FakeSmi:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def _row(sm, mx, hw="Not Active", thermal="Not Active", sw_thermal="Not Active", power="Not Active"):
    return f"0, {sm}, {mx}, 650.0, 0x0, {hw}, {thermal}, {sw_thermal}, {power}"


def test_clock_record_uses_samples_in_the_timed_region():
    s = bench.ClockSampler(0)
    s.proc = _FakeSmi()
    s.t0, s.t1 = 100.0, 101.0
    s.lines = [
        (98.0, _row(1200, 1965, hw="Active")),  # before the timed region: ignored
        (100.1, _row(1965, 1965)),
        (100.5, _row(1950, 1965, power="Active")),
        (100.9, _row(1965, 1965)),
        (103.0, _row(900, 1965, thermal="Active")),  # after: ignored
        (100.6, "garbage line"),
    ]
    rec = s.stop()
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["samples_in_timed_region"] == 3


def test_clock_record_reports_slowdowns_and_missing_smi():
    s = bench.ClockSampler(0)
    s.proc = _FakeSmi()
    s.t0, s.t1 = 10.0, 11.0
    s.lines = [(10.2, _row(1100, 1965, hw="Active", sw_thermal="Active"))]
    rec = s.stop()
    assert rec["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"] and rec["sm_mhz"] == 1100.0
    assert bench.ClockSampler(0).stop()["reasons"] == ["nvidia-smi unavailable"]


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    rec = tmp_path / "traffic_x.txt"
    rec.write_text("# note\nkernel_source_sha256_16: abc\nworkload: 2\nelements: 1000\n"
                   "dram_bytes_read: 3000\ndram_bytes_write: 2000\n")
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.recorded_traffic(2, 1000) == 5000.0
    assert bench.recorded_traffic(2, 2000) == 10000.0  # scaled by outputs
    assert bench.recorded_traffic(4, 1000) is None     # another workload
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "def")
    assert bench.recorded_traffic(2, 1000) is None     # the kernel changed since the capture


def test_kernel_source_hash_covers_the_shared_decode_header(monkeypatch, tmp_path):
    a, b = tmp_path / "a.cu", tmp_path / "b.cuh"
    a.write_text("kernel")
    b.write_text("decode")
    monkeypatch.setattr(bench, "KERNEL_SOURCES", [str(a), str(b)])
    h0 = bench.kernel_source_hash()
    b.write_text("decode changed")
    assert bench.kernel_source_hash() != h0


def test_algorithmic_bytes_of_a_stream():
    # EncodedExponent (valid bits), PackedSignMantissa and Gaps (5 bits per
    # segment) without padding, BlockOffset, LUTs and CodeLengths read; BF16
    # written.  Per element that is 3 bytes plus the code and metadata bits.
    w = inputs.gaussian(100_000, [40])
    s = df11.build_format(w).scalars()
    got = bench.stream_algorithmic_bytes(s)
    n = s["n"]
    bits = s["total_bits"] + 5 * s["num_segments"]
    assert got == 3 * n + -(-s["total_bits"] // 8) + -(-5 * s["num_segments"] // 8) \
        + 4 * (s["num_blocks"] + 1) + 256 * (s["num_luts"] + 1)
    assert 3 * n + bits / 8 < got < 3 * n + bits / 8 + 4 * (s["num_blocks"] + 1) + 256 * 18 + 2
    assert 3.3 < got / n < 3.4  # ~2.6 code bits + 0.08 Gaps bits per element on N(0, 0.02)


def test_all_core_oracle_baseline_rebuilds_the_stream(oracle_mod):
    # the all-core CPU baseline splits one stream at format-block boundaries
    # (each run from its first code start to the next run's) and must give
    # back every element, for several run counts and both block sizes
    for T in (32, 64):
        w = inputs.stress(300_001, key=(41, T))
        fmt = oracle_mod.build_format(w, T)
        for threads in (1, 3, 8):
            got = bench._oracle_decode_all_cores(oracle_mod, fmt, threads)
            assert np.array_equal(got, w)


def test_host_cpu_record():
    rec = bench.host_cpu()
    assert rec["nproc"] >= 1 and isinstance(rec["cpu_model"], str) and rec["cpu_model"]
