"""Host logic of bench.py's roofline object (no GPU): which launch is the dominant kernel, its
algorithmic TFLOP/s, and DRAM traffic that is reported only while the kernel source is the one
the ncu capture was taken on.  Also checks that the committed profile summaries name commands
that run committed files with the clocks left alone."""
import glob
import os
import re
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PK = {"bf16_tflops": 1665.3, "hbm_gbs": 6455.6, "source": "measured"}


def test_fused_launch_is_the_dominant_kernel_with_whole_layer_flops():
    res = {"T": 4096, "H_k": 16, "H_v": 48, "kernel_ms": {"prep": 0.0026, "scan": 0.40, "helpers+gaps": 0.02}}
    r = bench.prefill_roofline(res, 1, PK, 0.42)
    assert r["kernel"] == "prefill_fused_kernel"
    flops = 7_602_176 * 4096  # prep 1,310,720 + scan 6,291,456 per token at 16/48 heads
    assert r["algorithmic_flop_per_launch"] == flops
    assert r["achieved"] == pytest.approx(flops / 0.40e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / PK["bf16_tflops"])
    assert r["whole_step"]["achieved"] == pytest.approx(flops / 0.42e-3 / 1e12)


def test_two_launches_pick_the_longer_kernel_with_its_own_flops():
    res = {"T": 4096, "H_k": 16, "H_v": 48, "kernel_ms": {"prep": 0.20, "scan": 0.25, "helpers+gaps": 0.01}}
    r = bench.prefill_roofline(res, 1, PK, 0.46)
    assert r["kernel"] == "scan_kernel"
    assert r["algorithmic_flop_per_launch"] == 6_291_456 * 4096
    res["kernel_ms"] = {"prep": 0.30, "scan": 0.25, "helpers+gaps": 0.01}
    r = bench.prefill_roofline(res, 1, PK, 0.56)
    assert r["kernel"] == "prep_kernel"
    assert r["algorithmic_flop_per_launch"] == 1_310_720 * 4096


def test_traffic_only_for_the_captured_kernel_source(monkeypatch):
    res = {"T": 4096, "H_k": 16, "H_v": 48, "kernel_ms": {"prep": 0.0026, "scan": 0.40, "helpers+gaps": 0.02}}
    entry = bench.TRAFFIC[(1, "prefill_fused")]
    monkeypatch.setattr(bench, "src_sha", lambda name: entry["sha"])
    assert bench.prefill_roofline(res, 1, PK, 0.42)["traffic"] == entry["bytes"]
    monkeypatch.setattr(bench, "src_sha", lambda name: "0" * 16)  # the kernel changed since the capture
    assert bench.prefill_roofline(res, 1, PK, 0.42)["traffic"] is None
    res["prefix"] = True  # a shortened run: the full case's capture does not apply
    monkeypatch.setattr(bench, "src_sha", lambda name: entry["sha"])
    assert bench.prefill_roofline(res, 1, PK, 0.42)["traffic"] is None


def test_profiles_name_committed_commands_and_leave_clocks_alone():
    files = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))
    assert files
    for f in files:
        text = open(f).read()
        assert "_work" not in text, f
        for script in re.findall(r"python\s+(\S+\.py)", text):
            assert os.path.isfile(os.path.join(ROOT, script)), (f, script)
        for line in text.splitlines():
            if re.match(r"\s+ncu\s", line):  # a command line (indented), not prose about a capture
                if "$M" in line:  # the metrics and flags given once, as M = `...`, above the commands
                    assert re.search(r"M = `[^`]*--clock-control none", text), (f, line)
                else:
                    assert "--clock-control none" in line, (f, line)
