"""Host logic of bench.py (CPU): the measured peaks it divides by, the rule
that a recorded ncu traffic figure is reported only for the kernel sources
it was captured on, and the timing defaults of its command line."""
import json
import os
import re

import pytest

from conftest import ROOT


def _bench():
    import bench
    return bench


def test_default_arguments_meet_the_timing_rules():
    a = _bench().parse_args([])
    assert a.gpus == 1 and a.impl == "ours"
    assert a.warmup >= 3                  # at least three untimed warm-up steps
    assert a.steps >= 10


def test_measured_peaks_are_loaded():
    peaks, kind = _bench().load_peaks()
    if not os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        pytest.skip("no measured peaks in this checkout")
    assert kind == "measured"
    for key in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained"):
        assert peaks[key] > 0
    assert peaks["bf16_tflops_sustained"] <= peaks["bf16_tflops"]


def test_source_digest_is_stable():
    b = _bench()
    d = b.source_digest("split_partial")
    assert re.fullmatch(r"[0-9a-f]{16}", d)
    assert b.source_digest("split_partial") == d


def test_code_digest_ignores_comments_only():
    b = _bench()
    a = 'int f(int x) { // doubles\n  return 2 * x; /* no "//" here */ }\nconst char* s = "a // b";'
    c = 'int f(int x) {\n\n  return 2 * x;   }\n// another comment\nconst char* s = "a // b";'
    assert b.code_only(a) == b.code_only(c)
    assert '"a // b"' in b.code_only(a)              # string literals are code
    assert b.code_only(a) != b.code_only(a.replace("2 * x", "3 * x"))
    assert b.code_only(a) != b.code_only(a.replace('"a // b"', '"a / b"'))


def test_traffic_is_reported_only_for_the_recorded_sources():
    b = _bench()
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    with open(path) as f:
        rec = json.load(f)["scale1m_bf16"]["split_partial"]
    got = b.ncu_traffic("split_partial", "scale1m_bf16")
    if rec["source_digest"] == b.source_digest("split_partial"):
        assert got == rec["dram_bytes_per_launch"]
        # the figure is per launch at full size: at least the algorithmic bytes
        # of the lighter split pass (k0 once: B*H*N*D*2 = 1 GiB)
        assert got >= 8 * 1048576 * 64 * 2
    else:
        assert got is None
    assert b.ncu_traffic("split_partial", "no_such_workload") is None


def test_traffic_record_scaling_is_consistent():
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)["scale1m_bf16"]["split_partial"]
    full = rec["full_size_bytes"]
    assert rec["dram_bytes_per_launch"] == (full["synthesis"] + full["encode"]) // 2
    small = rec["small_case_bytes"]
    writes = 37 * 8 * 512 * 66 * 4       # the full-size plan's partial triples per launch
    for p in ("synthesis", "encode"):
        assert full[p] == 8 * small[p]["read"] + writes


def test_simt_peak_arithmetic():
    b = _bench()
    assert b.fp32_simt_peak_tflops({"sm_max_mhz": 1000.0}) == pytest.approx(148 * 128 * 2 * 1e9 / 1e12)
