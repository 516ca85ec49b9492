"""Pins of the utilisation formulas (CPU only): hand-computed values in
tests/golden/utilisation.json for every function of oracle.utilisation (the paged
ratio, the ratio from a manager's state with and without sharing, the contiguous
analogue and the per-sequence waste bound); the block manager model's state gives the
same numbers; the waste bound holds, and is tight where every last block is one token
short of the worst case, on the synthetic length distributions."""
import json
import os

import numpy as np
import pytest

from oracle import block_manager as BM
from oracle import utilisation as U
from paged_kv_cache_320_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "utilisation.json")
DATA = json.load(open(GOLDEN))


@pytest.mark.parametrize("case", DATA["cases"])
def test_hand_computed_values(case):
    bs = case["block_size"]
    assert U.paged_utilisation(case["lens"], bs) == pytest.approx(case["paged"], abs=1e-15)
    assert U.contiguous_utilisation(case["lens"], case["max_len"]) == pytest.approx(
        case["contiguous"], abs=1e-15)
    assert U.waste_lower_bound(case["lens"], bs) == pytest.approx(case["waste_bound"], abs=1e-15)
    assert U.utilisation_from_state(case["tokens"], case["blocks"], bs) == pytest.approx(
        case["paged"], abs=1e-15)
    mgr = BM.BlockManagerModel(64, bs, 64)
    for s, n in enumerate(case["lens"]):
        assert mgr.append(s, n)[0] == 0
    free, held, tokens, util = mgr.stats()
    assert (held, tokens) == (case["blocks"], case["tokens"])
    assert util == pytest.approx(case["paged"], abs=1e-15)


def test_utilisation_from_state_with_sharing():
    """Logical tokens over held blocks may exceed 1 once blocks are shared (hand-worked
    fork and copy-on-write trace)."""
    sc = DATA["shared_cases"]
    bs = sc["block_size"]
    mgr = BM.BlockManagerModel(16, bs, 16)
    for step in sc["steps"]:
        if step["op"] == "append":
            assert mgr.append(step["seq"], step["n"])[0] == 0
        else:
            assert mgr.fork(step["parent"], step["child"]) == 0
        _, held, tokens, util = mgr.stats()
        assert (held, tokens) == (step["blocks"], step["tokens"])
        assert U.utilisation_from_state(tokens, held, bs) == pytest.approx(step["util"], abs=1e-15)
        assert util == pytest.approx(step["util"], abs=1e-15)
    assert U.utilisation_from_state(0, 0, bs) == 0.0


@pytest.mark.parametrize("name", ["llama7b_mha", "llama3_8b_gqa", "long_context"])
def test_waste_bound_on_synthetic_lengths(name):
    wl = synth.make_workload(name, values_on="none")
    bs = wl.spec.block_size
    u = U.paged_utilisation(wl.context_lens, bs)
    assert U.waste_lower_bound(wl.context_lens, bs) <= u <= 1.0
    assert u > 0.9          # paged utilisation "90%+" at bs 16 for these lengths
    # every length one past a block boundary leaves bs - 1 empty slots: the bound is met
    worst = (np.asarray(wl.context_lens[:64]) // bs) * bs + 1
    assert U.waste_lower_bound(worst, bs) == pytest.approx(U.paged_utilisation(worst, bs),
                                                           rel=1e-12)
