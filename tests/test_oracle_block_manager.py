"""Pins of the block-manager model (CPU only): hand-worked traces in
tests/golden/alloc_traces.json, and invariants on seeded random op sequences
(free + held = pool; refcounts = references from the tables; without sharing
sum of refcounts = sum ceil(len/bs); every slot lies in its sequence's block)."""
import json
import os

import numpy as np
import pytest

from oracle import block_manager as BM

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "alloc_traces.json")


def run_trace(mgr, tr):
    for op in tr["ops"]:
        if op["op"] == "append":
            st, slots, cows = mgr.append(op["seq"], op["n"])
            assert st == op["status"], op
            if st == 0:
                assert slots == op["slots"], op
                assert [list(c) for c in cows] == op["cow"], op
        elif op["op"] == "fork":
            assert mgr.fork(op["parent"], op["child"]) == op["status"], op
        elif op["op"] == "free":
            assert mgr.free(op["seq"]) == op["status"], op


@pytest.mark.parametrize("trace", json.load(open(GOLDEN))["traces"], ids=lambda t: t["name"])
def test_hand_worked_traces(trace):
    mgr = BM.BlockManagerModel(trace["num_blocks"], trace["block_size"],
                               trace["max_blocks_per_seq"], trace["initial_order"])
    run_trace(mgr, trace)
    for seq, (row, n) in trace["final_tables"].items():
        assert mgr.block_table(int(seq)) == (row, n)
    free, held, tokens, util = mgr.stats()
    fs = trace["final_stats"]
    assert (free, held, tokens) == (fs["free"], fs["held"], fs["tokens"])
    assert util == pytest.approx(fs["util"], abs=1e-15)


def check_invariants(mgr):
    free, held, tokens, _ = mgr.stats()
    assert free + held == mgr.nb
    refs = [0] * mgr.nb
    for seq, table in mgr.tables.items():
        assert len(table) == -(-mgr.lens[seq] // mgr.bs)
        for b in table:
            refs[b] += 1
    assert refs == mgr.refcount
    assert len(set(mgr.free_stack)) == len(mgr.free_stack)
    assert all(mgr.refcount[b] == 0 for b in mgr.free_stack)


@pytest.mark.parametrize("seed", range(20))
def test_random_op_sequences_keep_invariants(seed):
    rng = np.random.default_rng(seed)
    nb, bs = 32, 4
    mgr = BM.BlockManagerModel(nb, bs, 8, rng.permutation(nb))
    live = []
    next_id = 0
    for _ in range(300):
        r = rng.random()
        if r < 0.5 or not live:
            seq = live[rng.integers(len(live))] if live and rng.random() < 0.7 else next_id
            if seq == next_id:
                next_id += 1
            n = int(rng.integers(0, 7))
            before = (list(mgr.free_stack), list(mgr.refcount), {k: list(v) for k, v in mgr.tables.items()})
            old_len = mgr.lens.get(seq, 0)
            st, slots, cows = mgr.append(seq, n)
            if st == 0:
                if seq not in live:
                    live.append(seq)
                table = mgr.tables[seq]
                for i, slot in enumerate(slots):
                    pos = old_len + i
                    assert slot // bs == table[pos // bs] and slot % bs == pos % bs
                for old, new in cows:
                    assert mgr.refcount[new] >= 1
            else:
                assert mgr.free_stack == before[0] and mgr.refcount == before[1]
                assert mgr.tables == before[2]
        elif r < 0.7:
            parent = live[rng.integers(len(live))]
            assert mgr.fork(parent, next_id) == 0
            live.append(next_id)
            next_id += 1
        else:
            seq = live.pop(rng.integers(len(live)))
            assert mgr.free(seq) == 0
        check_invariants(mgr)


def test_unshared_refcount_sum_equals_blocks_needed():
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 60, size=10)
    mgr = BM.BlockManagerModel(200, 16, 8, rng.permutation(200))
    for s, n in enumerate(lens):
        assert mgr.append(s, int(n))[0] == 0
    assert sum(mgr.refcount) == sum(-(-int(n) // 16) for n in lens)


def test_placement_recipe_matches_in_order_appends():
    """A pool seeded with a permutation and filled by appending each sequence's
    tokens in order hands out exactly consecutive slices of the permutation."""
    from paged_kv_cache_320_b200 import synth
    wl = synth.make_workload("llama3_8b_gqa", values_on="none")
    mgr = BM.BlockManagerModel(wl.num_blocks, 16, wl.max_blocks_per_seq, wl.perm)
    last_slots = []
    for s, n in enumerate(wl.context_lens):
        st, slots, cows = mgr.append(s, int(n))
        assert st == 0 and not cows
        last_slots.append(slots[-1])
        row, ln = mgr.block_table(s)
        assert ln == n
        np.testing.assert_array_equal(row, wl.block_tables[s])
    np.testing.assert_array_equal(last_slots, wl.slot_mapping)
