"""Host logic of bench.py that needs no GPU: the ncu traffic record is used only
while the GEMM kernel's sources are the ones it was taken with."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_record_matches_current_sources():
    rec = dict(l.split(": ", 1) for l in open(bench.TRAFFIC_RECORD).read().splitlines()
               if l and not l.startswith("#") and ": " in l)
    alg = int(rec["algorithmic_bytes_per_launch"])
    got = bench.recorded_w13_traffic(alg)
    # either the record is current (and then it is what the file says) or stale (None)
    assert got is None or got == int(rec["traffic_bytes_per_launch"])
    assert bench.recorded_w13_traffic(alg + 1) is None


def test_traffic_record_is_dropped_when_a_source_changes(tmp_path, monkeypatch):
    changed = tmp_path / "gemm_fp8.cu"
    with open(os.path.join(ROOT, bench.GEMM_SOURCES[-1]), "rb") as f:
        changed.write_bytes(f.read() + b"\nstatic int edited_code;\n")
    monkeypatch.setattr(bench, "GEMM_SOURCES", bench.GEMM_SOURCES[:-1] + (str(changed),))
    rec = dict(l.split(": ", 1) for l in open(bench.TRAFFIC_RECORD).read().splitlines()
               if l and not l.startswith("#") and ": " in l)
    assert bench.recorded_w13_traffic(int(rec["algorithmic_bytes_per_launch"])) is None


def test_comment_edits_keep_the_record(tmp_path, monkeypatch):
    changed = tmp_path / "gemm_fp8.cu"
    with open(os.path.join(ROOT, bench.GEMM_SOURCES[-1]), "rb") as f:
        changed.write_bytes(f.read() + b"\n// a comment\n/* and a\n block */\n")
    before = bench.gemm_sources_sha256()
    monkeypatch.setattr(bench, "GEMM_SOURCES", bench.GEMM_SOURCES[:-1] + (str(changed),))
    assert bench.gemm_sources_sha256() == before


def test_reference_step_sampler_and_rank_split():
    import argparse
    import math
    import synth
    step = bench.oracle_step_sampler(synth.TINY, tok=32, rows=16)
    v = step(0)
    assert math.isfinite(v) and v > 0
    args = argparse.Namespace(steps=1, warmup=0)
    assert bench.run_reference(args, rank=1, world=2) is None    # only rank 0 works


def _fake_smi(tmp_path, period_s: float, mhz: int):
    """A stand-in nvidia-smi on PATH that prints one CSV sample per period."""
    exe = tmp_path / "nvidia-smi"
    exe.write_text("#!/usr/bin/env python3\nimport sys, time\n"
                   f"while True:\n    print('0, {mhz}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Active',"
                   " flush=True)\n"
                   f"    time.sleep({period_s})\n")
    exe.chmod(0o755)
    return str(tmp_path)


def test_clock_sampler_region_and_short_region(tmp_path, monkeypatch):
    """Samples come from the region only (the sampler waits for its first sample
    before the region starts); a region shorter than the period is described by
    the first sample after it, and says so."""
    import os
    import time
    import bench
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, 0.05, 1800) + os.pathsep + os.environ["PATH"])
    with bench.ClockSampler(0) as clk:
        time.sleep(0.3)
    s = clk.summary()
    assert s["sm_mhz"] == 1800.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] >= 3 and "window" not in s
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, 0.3, 1500) + os.pathsep + os.environ["PATH"])
    with bench.ClockSampler(0) as clk:
        pass
    s = clk.summary()
    assert s["sm_mhz"] == 1500.0 and s["samples"] >= 1 and "window" in s
