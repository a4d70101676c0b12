"""Host-side arithmetic behind bench.py's roofline line (no GPU).

The roofline's `achieved` is the algorithmic bytes of one launch over its measured time, and
its `traffic` comes from the committed ncu summary only while that summary's source hash
matches the kernel sources. These tests fix the byte counts of the 1 GiB workload and check
that the committed traffic summary is self-consistent."""
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
N = 65536 * 8192   # the 1 GiB BF16 workload


def test_algorithmic_bytes_of_the_1gib_workload():
    b = bench.algorithmic_bytes(N, 1)
    # quantize: read x (2 B) and the amax; write codes (1/2 B), one scale byte per 16 elements,
    # one choice bit per block, one tensor scale: 2.5703 B per element
    assert b["quantize"] == 1379926024
    assert abs(b["quantize"] / N - 2.5703) < 1e-4
    assert b["amax"] == 2 * N + 4
    assert b["dequantize"] == N // 2 + N // 16 + 4 + 2 * N


def test_algorithmic_bytes_per_group():
    one, many = bench.algorithmic_bytes(N, 1), bench.algorithmic_bytes(N, 64)
    assert many["quantize"] - one["quantize"] == 8 * 63   # an amax read and a tensor scale per group
    assert many["amax"] - one["amax"] == 4 * 63


def _traffic_file():
    vals = {}
    with open(os.path.join(ROOT, "profiles", "dram_traffic.txt")) as f:
        for ln in f:
            if ":" in ln and not ln.startswith("#"):
                k, v = ln.split(":", 1)
                vals[k.strip()] = v.strip()
    return vals


def test_committed_traffic_summary_is_consistent():
    v = _traffic_file()
    rd, wr, tot = (float(v[f"quantize_bytes_{k}"]) for k in ("read_per_launch", "write_per_launch", "per_launch"))
    assert abs(rd + wr - tot) <= 0.2e6
    # DRAM traffic cannot exceed what the kernel must move by much; the tail of the output may
    # still sit in L2 when the kernel ends, so it may be a little below
    algo = float(v["quantize_algorithmic_bytes_per_launch"])
    assert abs(algo - bench.algorithmic_bytes(N, 1)["quantize"]) <= 0.1e6
    assert 0.95 * algo <= tot <= 1.02 * algo
    assert len(v["source_sha256_16"]) == 16
    # the bench reports it only while the kernel sources are the ones it was captured on
    assert bench.ncu_traffic("quantize") in (None, tot)


def test_peak_comes_from_the_measured_file():
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
        hbm = float(json.load(f)["hbm_gbs"])
    assert bench.measured_peak() == (hbm, "measured")
