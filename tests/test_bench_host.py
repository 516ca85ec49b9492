"""Host-side pieces of bench.py (CPU only): algorithmic bytes against their formula, the
profile-traffic lookup gated by the kernel-source hash, the reference arm (the CPU
oracle) producing its JSON line, and the parsing of sampled GPU clocks."""
import argparse
import os

import numpy as np
import pytest

import bench
from paged_kv_cache_320_b200 import synth


def test_algorithmic_bytes_formula():
    wl = synth.make_workload("llama3_8b_gqa", values_on="none")
    sp = wl.spec
    kv, roof = bench.algorithmic_bytes(wl)
    lens = wl.context_lens.astype(np.int64)
    assert kv == int(lens.sum()) * sp.num_kv_heads * sp.head_dim * 2 * 2
    blocks = int(((lens + sp.block_size - 1) // sp.block_size).sum())
    assert roof == kv + wl.num_seqs * sp.num_heads * sp.head_dim * 4 + blocks * 4 + wl.num_seqs * 4


def test_traffic_is_read_only_for_the_current_kernel_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    good = bench.kernel_source_hash()
    (prof / "paged_decode_partition__demo.md").write_text(
        f"kernel_source_sha256: {good}\ntraffic_bytes_per_launch[block_size=16]: 1234\n")
    (prof / "paged_decode_step__demo.md").write_text(
        f"kernel_source_sha256: {good}\ntraffic_bytes_per_launch[block_size=16]: 99\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the kernel sources are read relative to ROOT: link them in
    for src in bench.STEP_SOURCES:
        dst = tmp_path / src
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(os.path.dirname(bench.__file__), src), "rb").read())
    assert bench.read_traffic("demo", 16) == 1234.0
    assert bench.read_traffic("demo", 8) is None                 # no line for this block size
    assert bench.read_traffic("other", 16) is None               # no summary at all
    # the step kernel's summary is gated by a hash over its own sources as well
    assert bench.read_traffic("demo", 16, "paged_decode_step") is None
    (prof / "paged_decode_step__demo.md").write_text(
        f"kernel_source_sha256: {bench.kernel_source_hash(bench.STEP_SOURCES)}\n"
        "traffic_bytes_per_launch[block_size=16]: 99\n")
    assert bench.read_traffic("demo", 16, "paged_decode_step") == 99.0


def test_reference_arm_line():
    args = argparse.Namespace(workload="long_context", block_size=16, steps=1, warmup=1,
                              gpus=1, cpu_seconds=1.0)
    res = bench.reference_arm(args, 0)
    assert res["impl"] == "reference"
    assert res["unit"] == "GB/s" and res["value"] > 0
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["value"] == res["value"]
    assert res["cpu_baseline"]["kind"] == "oracle"
    assert res["config"]["description"].endswith("(run with block_size 16)")
    assert bench.reference_arm(args, 1) is None                  # other ranks do nothing


def test_clock_summary_parses_nvidia_smi_samples():
    """Median SM clock, max clock and the throttle reasons that were active in any sample
    ("Not Active" must not count); malformed lines are skipped."""
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1740, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1800, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage",
    ]
    r = s.summary()
    assert r == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    s.lines = ["0, 1200, 1965, 500, 0x8, Active, Not Active, Active, Not Active"]
    assert s.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    s.lines = []
    assert s.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"],
                           "samples": 0}
