"""Pins of the utilisation formula (CPU only): hand-computed values in
tests/golden/utilisation.json; the block manager's state gives the same number;
the per-sequence waste bound holds on the synthetic length distributions."""
import json
import os

import numpy as np
import pytest

from oracle import block_manager as BM
from oracle import utilisation as U
from paged_kv_cache_320_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "utilisation.json")


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"])
def test_hand_computed_values(case):
    assert U.paged_utilisation(case["lens"], case["block_size"]) == pytest.approx(case["paged"], abs=1e-15)
    assert U.contiguous_utilisation(case["lens"], case["max_len"]) == pytest.approx(case["contiguous"], abs=1e-15)
    mgr = BM.BlockManagerModel(64, case["block_size"], 64)
    for s, n in enumerate(case["lens"]):
        assert mgr.append(s, n)[0] == 0
    free, held, tokens, util = mgr.stats()
    assert held == case["blocks"]
    assert util == pytest.approx(case["paged"], abs=1e-15)


@pytest.mark.parametrize("name", ["llama7b_mha", "llama3_8b_gqa", "long_context"])
def test_waste_bound_on_synthetic_lengths(name):
    wl = synth.make_workload(name, values_on="none")
    u = U.paged_utilisation(wl.context_lens, wl.spec.block_size)
    assert U.waste_lower_bound(wl.context_lens, wl.spec.block_size) <= u <= 1.0
    assert u > 0.9          # paged utilisation "90%+" at bs 16 for these lengths
