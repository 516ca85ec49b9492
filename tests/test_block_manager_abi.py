"""The C++ block manager (through the C-ABI) against the hand-worked traces in
tests/golden/alloc_traces.json and, op by op, against the oracle's independent
Python model on seeded random op sequences: identical statuses, slots,
copy-on-write pairs, block tables and statistics (CPU only)."""
import json
import os

import numpy as np
import pytest

from oracle import block_manager as BM
from paged_kv_cache_320_b200 import BlockManager, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "alloc_traces.json")


@pytest.mark.parametrize("trace", json.load(open(GOLDEN))["traces"], ids=lambda t: t["name"])
def test_hand_worked_traces(trace):
    mgr = BlockManager(trace["num_blocks"], trace["block_size"], trace["max_blocks_per_seq"],
                       trace["initial_order"])
    for op in trace["ops"]:
        if op["op"] == "append":
            st, slots, cows = mgr.pkv_seq_append(op["seq"], op["n"])
            assert st == op["status"], op
            if st == 0:
                assert slots.tolist() == op["slots"], op
                assert cows.tolist() == op["cow"], op
        elif op["op"] == "fork":
            assert mgr.pkv_seq_fork(op["parent"], op["child"]) == op["status"], op
        else:
            assert mgr.pkv_seq_free(op["seq"]) == op["status"], op
    for seq, (row, n) in trace["final_tables"].items():
        st, tables, lens = mgr.pkv_block_tables([int(seq)])
        assert st == 0 and tables[0].tolist() == row and lens[0] == n
    free, held, tokens, util = mgr.pkv_stats()
    fs = trace["final_stats"]
    assert (free, held, tokens) == (fs["free"], fs["held"], fs["tokens"])
    assert util == pytest.approx(fs["util"], abs=1e-15)


def compare_states(c, m, seqs):
    fc, hc, tc, uc = c.pkv_stats()
    fm, hm, tm, um = m.stats()
    assert (fc, hc, tc) == (fm, hm, tm)
    assert uc == pytest.approx(um, abs=1e-12)
    assert c.pkv_alloc_refcounts().tolist() == m.refcount
    if seqs:
        st, tables, lens = c.pkv_block_tables(seqs)
        assert st == 0
        for i, s in enumerate(seqs):
            row, n = m.block_table(s)
            assert tables[i].tolist() == row and lens[i] == n


@pytest.mark.parametrize("chunk", range(8))
def test_random_op_sequences_match_the_model(chunk):
    """2000 seeded op sequences (250 per chunk) of 40 ops each, with errors."""
    for seed in range(chunk * 250, (chunk + 1) * 250):
        rng = np.random.default_rng(seed)
        nb = int(rng.integers(4, 24))
        bs = int(rng.choice([1, 2, 4, 8]))
        mb = int(rng.integers(1, 6))
        order = rng.permutation(nb)
        c = BlockManager(nb, bs, mb, order)
        m = BM.BlockManagerModel(nb, bs, mb, order)
        ids = list(range(6))
        for _ in range(40):
            r = rng.random()
            a = int(rng.choice(ids))
            if r < 0.6:
                n = int(rng.integers(0, 2 * bs + 2))
                sc, slc, cwc = c.pkv_seq_append(a, n)
                sm, slm, cwm = m.append(a, n)
                assert sc == sm, (seed, a, n)
                assert slc.tolist() == slm
                assert cwc.tolist() == [list(x) for x in cwm]
            elif r < 0.8:
                b = int(rng.choice(ids))
                assert c.pkv_seq_fork(a, b) == m.fork(a, b)
            else:
                assert c.pkv_seq_free(a) == m.free(a)
        compare_states(c, m, sorted(m.tables))
        c.close()


def test_workload_placement_reproduced_by_in_order_appends():
    wl = synth.make_workload("long_context", values_on="none", block_size=8)
    mgr = BlockManager(wl.num_blocks, 8, wl.max_blocks_per_seq, wl.perm)
    last = []
    for s, n in enumerate(wl.context_lens):
        st, slots, cows = mgr.pkv_seq_append(s, int(n))
        assert st == 0 and len(cows) == 0
        last.append(slots[-1])
    st, tables, lens = mgr.pkv_block_tables(np.arange(wl.num_seqs))
    np.testing.assert_array_equal(tables, wl.block_tables)
    np.testing.assert_array_equal(lens, wl.context_lens)
    np.testing.assert_array_equal(last, wl.slot_mapping)


@pytest.mark.parametrize("seed", range(40))
def test_batched_append_equals_appends_in_order(seed):
    """pkv_seq_append_batch == pkv_seq_append per sequence, in order, against the model;
    on failure the sequences before the failing one keep their appends."""
    rng = np.random.default_rng(500 + seed)
    nb, bs, mb = int(rng.integers(6, 30)), int(rng.choice([2, 4, 8])), int(rng.integers(2, 6))
    order = rng.permutation(nb)
    c = BlockManager(nb, bs, mb, order)
    m = BM.BlockManagerModel(nb, bs, mb, order)
    for s in range(4):
        n0 = int(rng.integers(1, bs * 2))
        assert c.pkv_seq_append(s, n0)[0] == m.append(s, n0)[0]
    if rng.random() < 0.5:
        assert c.pkv_seq_fork(0, 7) == m.fork(0, 7)
    for _ in range(6):
        ids = [int(x) for x in rng.choice([0, 1, 2, 3, 7, 9], size=int(rng.integers(1, 6)))]
        k = int(rng.integers(0, 3))
        st, done, slots, cows = c.pkv_seq_append_batch(ids, k)
        exp_slots, exp_cows, exp_done, exp_st = [], [], 0, 0
        for sid in ids:
            s2, sl, cw = m.append(sid, k)
            if s2 != 0:
                exp_st = s2
                break
            exp_slots.append(sl)
            exp_cows += [list(x) for x in cw]
            exp_done += 1
        assert st == exp_st and done == exp_done
        for i in range(done):
            assert slots[i].tolist() == exp_slots[i]
        assert cows.tolist() == exp_cows
        compare_states(c, m, sorted(m.tables))
    c.close()


@pytest.mark.parametrize("seed", range(30))
def test_append_with_tables_equals_the_model(seed):
    """pkv_seq_append_tables == the model's appends in order, then its block tables and
    lengths of the same sequences; on a failed append the caller's tables are untouched
    and the sequences before the failing one keep their appends. Outputs written into
    caller arrays (as into a pinned buffer) equal the returned ones."""
    rng = np.random.default_rng(900 + seed)
    nb, bs, mb = int(rng.integers(6, 30)), int(rng.choice([2, 4, 8])), int(rng.integers(2, 6))
    order = rng.permutation(nb)
    c = BlockManager(nb, bs, mb, order)
    m = BM.BlockManagerModel(nb, bs, mb, order)
    for s in range(4):
        n0 = int(rng.integers(1, bs * 2))
        assert c.pkv_seq_append(s, n0)[0] == m.append(s, n0)[0]
    if rng.random() < 0.5:
        assert c.pkv_seq_fork(0, 7) == m.fork(0, 7)
    for _ in range(6):
        ids = [int(x) for x in rng.choice([0, 1, 2, 3, 7, 9], size=int(rng.integers(1, 6)))]
        k = int(rng.integers(0, 3))
        given = rng.random() < 0.5
        outs = {}
        if given:
            outs = dict(slots_out=np.full((len(ids), k), -7, np.int64),
                        cows_out=np.full((len(ids) * k, 2), -7, np.int32),
                        tables_out=np.full((len(ids), mb), -7, np.int32),
                        lens_out=np.full(len(ids), -7, np.int32))
        st, done, slots, cows, tables, lens = c.pkv_seq_append_tables(ids, k, **outs)
        exp_slots, exp_cows, exp_done, exp_st = [], [], 0, 0
        for sid in ids:
            s2, sl, cw = m.append(sid, k)
            if s2 != 0:
                exp_st = s2
                break
            exp_slots.append(sl)
            exp_cows += [list(x) for x in cw]
            exp_done += 1
        assert st == exp_st and done == exp_done
        for i in range(done):
            assert slots[i].tolist() == exp_slots[i]
        assert cows.tolist() == exp_cows
        if st == 0:
            for i, sid in enumerate(ids):
                row, n = m.block_table(sid)
                assert tables[i].tolist() == row and lens[i] == n
        elif given:
            assert (outs["tables_out"] == -7).all() and (outs["lens_out"] == -7).all()
        if given:
            assert outs["tables_out"] is tables and outs["slots_out"] is slots
        compare_states(c, m, sorted(m.tables))
    c.close()


def test_append_with_tables_rejects_missing_or_wrong_outputs():
    c = BlockManager(16, 4, 4)
    assert c.pkv_seq_append(1, 3)[0] == 0
    with pytest.raises(ValueError):
        c.pkv_seq_append_tables([1], 1, tables_out=np.zeros((1, 3), np.int32))   # shape
    with pytest.raises(ValueError):
        c.pkv_seq_append_tables([1], 1, slots_out=np.zeros((1, 1), np.int32))    # dtype
    from paged_kv_cache_320_b200 import _binding as B
    import ctypes
    # the C call refuses a missing tables_out before changing anything
    ids = np.array([1], np.int64)
    slots = np.zeros(1, np.int64)
    cows = np.zeros((1, 2), np.int32)
    n_cow, done = ctypes.c_int(0), ctypes.c_int(0)
    rc = B.lib().pkv_seq_append_tables(c._h, ids.ctypes.data, 1, 1, slots.ctypes.data,
                                       cows.ctypes.data, ctypes.byref(n_cow), ctypes.byref(done),
                                       None, None)
    assert rc == B.PKV_ERR_INVALID_ARG
    st, tables, lens = c.pkv_block_tables([1])
    assert lens.tolist() == [3]
    c.close()


@pytest.mark.parametrize("seed", range(30))
def test_batched_fork_and_free_equal_calls_in_order(seed):
    """pkv_seq_fork_batch / pkv_seq_free_batch == the single calls in order, against the
    model; on the first failure the calls before it keep their effects."""
    rng = np.random.default_rng(700 + seed)
    nb, bs, mb = int(rng.integers(10, 40)), int(rng.choice([2, 4, 8])), int(rng.integers(2, 6))
    order = rng.permutation(nb)
    c = BlockManager(nb, bs, mb, order)
    m = BM.BlockManagerModel(nb, bs, mb, order)
    for s in range(4):
        n0 = int(rng.integers(0, bs * 2))
        assert c.pkv_seq_append(s, n0)[0] == m.append(s, n0)[0]
    for _ in range(8):
        k = int(rng.integers(0, 6))
        if rng.random() < 0.5:
            parents = [int(x) for x in rng.choice([0, 1, 2, 3, 11, 12], size=k)]
            children = [int(x) for x in rng.choice([10, 11, 12, 13, 14, 0], size=k)]
            st, done = c.pkv_seq_fork_batch(parents, children)
            exp_st, exp_done = 0, 0
            for pa, ch in zip(parents, children):
                r = m.fork(pa, ch)
                if r != 0:
                    exp_st = r
                    break
                exp_done += 1
        else:
            ids = [int(x) for x in rng.choice([0, 1, 2, 3, 10, 11, 12, 13, 14], size=k)]
            st, done = c.pkv_seq_free_batch(ids)
            exp_st, exp_done = 0, 0
            for sid in ids:
                r = m.free(sid)
                if r != 0:
                    exp_st = r
                    break
                exp_done += 1
        assert (st, done) == (exp_st, exp_done)
        compare_states(c, m, sorted(m.tables))
    c.close()


@pytest.mark.parametrize("seed", range(6))
def test_many_sequences_forks_and_frees_match_the_model(seed):
    """Hundreds of live sequences, fork chains and frees in a large pool: sequence records
    are created, released and reused many times over (and their storage grows while
    forks copy from it); every status, slot, copy-on-write pair and final table matches
    the model."""
    rng = np.random.default_rng(1000 + seed)
    nb, bs, mb = 3000, int(rng.choice([4, 16])), 24
    order = rng.permutation(nb)
    c = BlockManager(nb, bs, mb, order)
    m = BM.BlockManagerModel(nb, bs, mb, order)
    live, next_id = [], 0
    for step in range(1500):
        r = rng.random()
        if r < 0.35 or not live:
            sid = next_id
            next_id += 1
            n = int(rng.integers(1, 3 * bs))
            sc, slc, cwc = c.pkv_seq_append(sid, n)
            sm, slm, cwm = m.append(sid, n)
            assert sc == sm and slc.tolist() == slm, (seed, step)
            if sc == 0:
                live.append(sid)
        elif r < 0.6:
            parent = int(rng.choice(live))
            child = next_id
            next_id += 1
            st = c.pkv_seq_fork(parent, child)
            assert st == m.fork(parent, child), (seed, step)
            if st == 0:
                live.append(child)
        elif r < 0.85:
            sid = int(rng.choice(live))
            n = int(rng.integers(0, bs + 2))
            sc, slc, cwc = c.pkv_seq_append(sid, n)
            sm, slm, cwm = m.append(sid, n)
            assert sc == sm and slc.tolist() == slm, (seed, step)
            assert cwc.tolist() == [list(x) for x in cwm]
        else:
            sid = live.pop(int(rng.integers(0, len(live))))
            assert c.pkv_seq_free(sid) == m.free(sid)
    assert len(live) > 100
    compare_states(c, m, sorted(m.tables))
    c.close()


GUARD_PROBE = r"""
import ctypes, resource, sys
sys.path.insert(0, sys.argv[1])
from paged_kv_cache_320_b200 import _binding as B
L = B.lib()
size = next(int(l.split()[1]) * 1024 for l in open("/proc/self/status") if l.startswith("VmSize:"))
cap = size + (256 << 20)
resource.setrlimit(resource.RLIMIT_AS, (cap, cap))
h = ctypes.c_void_p()
print(L.pkv_alloc_create(ctypes.byref(h), 100_000_000, 16, 8, None), h.value is None)
print(L.pkv_alloc_create(ctypes.byref(h), 1000, 16, 8, None), h.value is not None)
"""


@pytest.mark.skipif(not os.path.exists("/proc/self/status"), reason="needs Linux /proc")
def test_host_allocation_failure_is_a_status_not_an_exception():
    """A manager too large for the process's address-space limit: std::bad_alloc inside
    the library comes back as PKV_ERR_HOST_MEMORY (no exception crosses the C ABI, no
    handle is returned), and the next, small manager is created normally."""
    import subprocess
    import sys
    from paged_kv_cache_320_b200 import _binding as B
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", GUARD_PROBE, root], capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.split("\n")
    assert lines[0] == f"{B.PKV_ERR_HOST_MEMORY} True"
    assert lines[1] == f"{B.PKV_OK} True"


def test_prefix_groups_hand_worked():
    """bs 4. Sequence 1: 9 tokens (blocks a, b, c; c holds one token). 2 and 3 are forked
    from 1; 2 then appends 3 tokens, so its shared partial block c is copied (c') and it
    has 12 tokens = 3 full blocks a, b, c'. 4: 2 tokens (no full block). 5: 6 tokens of its
    own. Listed as [4, 2, 5, 1, 3]: group {4} (no full block), group {2, 1, 3} (first block
    a; full blocks 3, 2, 2 -> at most 2 in common, and a, b are common: prefix 8), group {5}."""
    c = BlockManager(64, 4, 8)
    m = BM.BlockManagerModel(64, 4, 8)
    for mgr in (c, m):
        ap = mgr.pkv_seq_append if mgr is c else mgr.append
        fk = mgr.pkv_seq_fork if mgr is c else mgr.fork
        ap(1, 9)
        fk(1, 2)
        fk(1, 3)
        ap(2, 3)
        ap(4, 2)
        ap(5, 6)
    st, order, starts, pre = c.pkv_prefix_groups([4, 2, 5, 1, 3])
    assert st == 0
    assert order.tolist() == [4, 2, 1, 3, 5]
    assert starts.tolist() == [0, 1, 4, 5]
    assert pre.tolist() == [0, 8, 0]
    assert m.prefix_groups([4, 2, 5, 1, 3]) == ([4, 2, 1, 3, 5], [0, 1, 4, 5], [0, 8, 0])
    # 1 and 3 alone still share the partly filled block c: only full blocks count, so the
    # prefix is 8 tokens (a, b), not 12
    st, order, starts, pre = c.pkv_prefix_groups([3, 1])
    assert (st, order.tolist(), starts.tolist(), pre.tolist()) == (0, [3, 1], [0, 2], [8])
    assert m.prefix_groups([3, 1]) == ([3, 1], [0, 2], [8])
    # unknown and repeated ids are refused
    from paged_kv_cache_320_b200 import _binding as B
    assert c.pkv_prefix_groups([1, 77])[0] == B.PKV_ERR_UNKNOWN_SEQ
    assert c.pkv_prefix_groups([1, 2, 1])[0] == B.PKV_ERR_INVALID_ARG
    st, order, starts, pre = c.pkv_prefix_groups([])
    assert st == 0 and len(order) == 0 and starts.tolist() == [0] and len(pre) == 0
    c.close()


@pytest.mark.parametrize("seed", range(20))
def test_prefix_groups_match_the_model(seed):
    """Seeded streams of appends, forks, frees and prefix-cached admissions: the library's
    groups equal the oracle model's for a random subset of the live sequences."""
    rng = np.random.default_rng(1300 + seed)
    nb, bs, mb = 64, int(rng.choice([2, 4, 8])), 12
    c = BlockManager(nb, bs, mb)
    m = BM.BlockManagerModel(nb, bs, mb)
    assert c.pkv_alloc_set_prefix_cache(1) == 0
    m.set_prefix_cache(True)
    prompts = [rng.integers(0, 50, int(rng.integers(1, 4 * bs)), dtype=np.int32).tolist()
               for _ in range(3)]
    live, nxt = [], 0
    for _ in range(40):
        op = rng.random()
        if op < 0.35 or not live:
            toks = prompts[int(rng.integers(0, 3))] + \
                rng.integers(0, 50, int(rng.integers(1, bs + 2)), dtype=np.int32).tolist()
            st, got = c.pkv_seq_share_prefix(nxt, toks[:-1])
            assert (st, got) == m.share_prefix(nxt, toks[:-1])
            st2 = c.pkv_seq_append_tokens(nxt, toks[got:])[0]
            assert st2 == m.append_tokens(nxt, toks[got:])[0]
            if st == 0 and st2 == 0:
                live.append(nxt)
            elif st == 0:
                assert c.pkv_seq_free(nxt) == m.free(nxt) == 0
            nxt += 1
        elif op < 0.55:
            parent = int(rng.choice(live))
            if c.pkv_seq_fork(parent, nxt) == m.fork(parent, nxt) == 0:
                live.append(nxt)
            nxt += 1
        elif op < 0.8:
            s_ = int(rng.choice(live))
            k = int(rng.integers(1, bs + 1))
            assert c.pkv_seq_append(s_, k)[0] == m.append(s_, k)[0]
        else:
            s_ = live.pop(int(rng.integers(0, len(live))))
            assert c.pkv_seq_free(s_) == m.free(s_) == 0
        if live:
            pick = [int(x) for x in rng.permutation(live)[:int(rng.integers(1, len(live) + 1))]]
            st, order, starts, pre = c.pkv_prefix_groups(pick)
            assert st == 0
            assert (order.tolist(), starts.tolist(), pre.tolist()) == m.prefix_groups(pick)
    c.close()
