"""Host-side pieces of bench.py (CPU only): algorithmic bytes against their formula, the
profile-traffic lookup gated by the kernel-source hash, and the reference arm (the CPU
oracle) producing its JSON line."""
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
