"""Prefix caching in the block manager ("vLLM / PagedAttention — 分页 KV Cache 分析"
§2.3 and §3.2: common prefixes are found and their pages reused across requests;
§五: only identical token sequences share).

Pins of the oracle's model: the published splitmix64 outputs, the hand-worked trace
in tests/golden/prefix_cache_trace.json, and a content check that records, for every
slot, the token prefix its K/V was computed from (a sequence built on shared blocks
must read back exactly its own prefixes). The C++ allocator is then compared with the
model op by op on seeded random request streams. CPU only."""
import json
import os

import numpy as np
import pytest

from oracle import block_manager as BM
from paged_kv_cache_320_b200 import BlockManager

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "prefix_cache_trace.json")


def test_splitmix64_matches_published_outputs():
    """The splitmix64 generator seeded with 0 (state advanced by the golden-ratio
    increment before each output) starts 0xe220a8397b1dcdaf, 0x6e789e6aa1b965f4,
    0x06c45d188009454f."""
    gamma = 0x9E3779B97F4A7C15
    outs = [BM.splitmix64((i * gamma) & ((1 << 64) - 1)) for i in range(3)]
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_prefix_hash_depends_on_every_token_and_order():
    base = [5, 6, 7, 8]
    h = BM.prefix_hash(base)
    assert BM.prefix_hash([]) == 0
    for i in range(4):
        changed = list(base)
        changed[i] += 1
        assert BM.prefix_hash(changed) != h
    assert BM.prefix_hash([6, 5, 7, 8]) != h
    assert BM.prefix_hash(base + [0]) != h          # a trailing 0 still counts
    assert BM.prefix_hash([-1]) == BM.prefix_hash([0xFFFFFFFF])   # ids as unsigned 32-bit


class ModelAdapter:
    """The oracle's model behind the calls the trace uses."""

    def __init__(self, t):
        self.m = BM.BlockManagerModel(t["num_blocks"], t["block_size"], t["max_blocks_per_seq"],
                                      t["initial_order"])

    def cache(self, e):
        return self.m.set_prefix_cache(e)

    def append_tokens(self, s, toks):
        return self.m.append_tokens(s, toks)

    def append(self, s, n):
        return self.m.append(s, n)

    def share(self, s, toks):
        return self.m.share_prefix(s, toks)

    def free(self, s):
        return self.m.free(s)

    def stats(self):
        return self.m.stats()

    def prefix_stats(self):
        return self.m.prefix_cache_stats()

    def free_list(self):
        return self.m.free_list()

    def table(self, s):
        return self.m.block_table(s)


class LibAdapter:
    def __init__(self, t):
        self.c = BlockManager(t["num_blocks"], t["block_size"], t["max_blocks_per_seq"],
                              t["initial_order"])

    def cache(self, e):
        return self.c.pkv_alloc_set_prefix_cache(e)

    def append_tokens(self, s, toks):
        st, sl, cw = self.c.pkv_seq_append_tokens(s, toks)
        return st, sl.tolist(), [tuple(x) for x in cw.tolist()]

    def append(self, s, n):
        st, sl, cw = self.c.pkv_seq_append(s, n)
        return st, sl.tolist(), [tuple(x) for x in cw.tolist()]

    def share(self, s, toks):
        return self.c.pkv_seq_share_prefix(s, toks)

    def free(self, s):
        return self.c.pkv_seq_free(s)

    def stats(self):
        return self.c.pkv_stats()

    def prefix_stats(self):
        return self.c.pkv_prefix_cache_stats()

    def free_list(self):
        return self.c.pkv_alloc_free_list().tolist()

    def table(self, s):
        st, tables, lens = self.c.pkv_block_tables([s])
        assert st == 0
        return tables[0].tolist(), int(lens[0])


@pytest.mark.parametrize("impl", [ModelAdapter, LibAdapter], ids=["model", "library"])
def test_hand_worked_trace(impl):
    t = json.load(open(GOLDEN))
    x = impl(t)
    for op in t["ops"]:
        kind = op["op"]
        if kind == "cache":
            assert x.cache(op["enable"]) == 0
        elif kind in ("append_tokens", "append"):
            st, slots, cows = (x.append_tokens(op["seq"], op["tokens"]) if kind == "append_tokens"
                               else x.append(op["seq"], op["n"]))
            assert st == op["status"], op
            if st == 0:
                assert list(slots) == op["slots"], op
                assert [list(c) for c in cows] == op["cow"], op
        elif kind == "share":
            assert x.share(op["seq"], op["tokens"]) == (op["status"], op["covered"]), op
        elif kind == "free":
            assert x.free(op["seq"]) == op["status"], op
        elif kind == "stats":
            free, held, tokens, _ = x.stats()
            assert (free, held, tokens) == (op["free"], op["held"], op["tokens"]), op
        elif kind == "prefix_stats":
            assert tuple(x.prefix_stats()) == (op["cached"], op["evictable"], op["query"],
                                               op["hit"]), op
    for seq, (row, n) in t["final_tables"].items():
        assert x.table(int(seq)) == (row, n)
    free, held, tokens, util = x.stats()
    fs = t["final_stats"]
    assert (free, held, tokens) == (fs["free"], fs["held"], fs["tokens"])
    assert util == pytest.approx(fs["util"], abs=1e-15)
    ps = t["final_prefix_stats"]
    assert tuple(x.prefix_stats()) == (ps["cached"], ps["evictable"], ps["query"], ps["hit"])
    # the free stack hands its blocks out last pushed first
    bs = t["block_size"]
    st, slots, _ = x.append(99, bs * len(t["final_free_order"]))
    assert st == 0
    assert [s // bs for s in slots[::bs]] == t["final_free_order"][::-1]


class SlotContents:
    """What every slot holds, as the cache write would leave it. A token's K/V depends on
    the whole prefix up to it, so a slot stands for that prefix (the tuple of ids up to
    and including its token); copy-on-write copies a whole block first."""

    def __init__(self, nb, bs):
        self.bs = bs
        self.v = [None] * (nb * bs)

    def write(self, slots, cows, before, toks):
        for src, dst in cows:
            self.v[dst * self.bs:(dst + 1) * self.bs] = self.v[src * self.bs:(src + 1) * self.bs]
        for i, s in enumerate(slots):
            self.v[s] = tuple(before) + tuple(toks[:i + 1])

    def read(self, row, n):
        return [self.v[row[p // self.bs] * self.bs + p % self.bs] for p in range(n)]

    @staticmethod
    def expected(ids):
        return [tuple(ids[:p + 1]) for p in range(len(ids))]


def random_stream(seed, impl_factory, check_contents=True):
    """Requests built from a few shared prompts plus private tails; decode appends, forks,
    frees and rare cache switches. Returns the op log (for the differential test)."""
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(6, 40))
    bs = int(rng.choice([1, 2, 4]))
    mb = int(rng.integers(2, 8))
    order = rng.permutation(nb).tolist()
    t = {"num_blocks": nb, "block_size": bs, "max_blocks_per_seq": mb, "initial_order": order}
    x = impl_factory(t)
    x.cache(1)
    prompts = [rng.integers(0, 5, size=int(rng.integers(1, 3 * bs + 2))).tolist()
               for _ in range(3)]
    ids = {}                       # live seq -> its token ids (-1 where appended without)
    contents = SlotContents(nb, bs)
    log = []
    next_id = 0
    for _ in range(60):
        r = rng.random()
        live = sorted(ids)
        if r < 0.35 or not live:
            toks = list(prompts[int(rng.integers(0, 3))])
            toks += rng.integers(0, 5, size=int(rng.integers(0, 2 * bs))).tolist()
            s = next_id
            next_id += 1
            st, covered = x.share(s, toks)
            log.append(("share", s, tuple(toks), st, covered))
            assert st == 0
            ids[s] = toks[:covered]
            st, slots, cows = x.append_tokens(s, toks[covered:])
            log.append(("append_tokens", s, st, tuple(slots), tuple(cows)))
            if st == 0:
                contents.write(slots, cows, toks[:covered], toks[covered:])
                ids[s] = toks
        elif r < 0.7:
            s = live[int(rng.integers(0, len(live)))]
            toks = rng.integers(0, 5, size=int(rng.integers(1, bs + 2))).tolist()
            if rng.random() < 0.1:
                st, slots, cows = x.append(s, len(toks))
                toks = [-1] * len(toks)
            else:
                st, slots, cows = x.append_tokens(s, toks)
            log.append(("append", s, st, tuple(slots), tuple(cows)))
            if st == 0:
                contents.write(slots, cows, ids[s], toks)
                ids[s] = ids[s] + toks
        elif r < 0.8:
            s = live[int(rng.integers(0, len(live)))]
            c = next_id
            next_id += 1
            x.m.fork(s, c) if isinstance(x, ModelAdapter) else x.c.pkv_seq_fork(s, c)
            ids[c] = list(ids[s])
            log.append(("fork", s, c))
        elif r < 0.97:
            s = live[int(rng.integers(0, len(live)))]
            assert x.free(s) == 0
            del ids[s]
            log.append(("free", s))
        else:
            on = int(rng.random() < 0.5)
            x.cache(on)
            log.append(("cache", on))
        log.append(("stats", tuple(x.stats()[:3]), tuple(x.prefix_stats())))
        if check_contents:
            for s, want in ids.items():
                row, n = x.table(s)
                assert n == len(want)
                # positions appended without ids stand as -1 on both sides
                assert contents.read(row, n) == SlotContents.expected(want), (seed, s)
    for s in sorted(ids):
        log.append(("table", s, x.table(s)))
    # the free list is the order the next allocations take
    fl = list(x.free_list())
    log.append(("free_list", tuple(fl)))
    k = min(len(fl), mb)
    if k:
        st, slots, _ = x.append(10_000, k * bs)
        assert st == 0
        assert [sl // bs for sl in slots[::bs]] == fl[:k]
    return log


@pytest.mark.parametrize("seed", range(60))
def test_model_reads_back_own_tokens(seed):
    """No sequence built on cached blocks ever sees another request's tokens."""
    random_stream(seed, ModelAdapter)


@pytest.mark.parametrize("chunk", range(4))
def test_library_matches_model_on_random_streams(chunk):
    for seed in range(chunk * 100, (chunk + 1) * 100):
        a = random_stream(1000 + seed, ModelAdapter, check_contents=False)
        b = random_stream(1000 + seed, LibAdapter, check_contents=seed % 10 == 0)
        assert a == b, seed


def test_stream_reuses_blocks():
    """The random streams do exercise sharing: hits happen and blocks are reused."""
    hits = 0
    for seed in range(20):
        log = random_stream(seed, ModelAdapter, check_contents=False)
        hits += sum(1 for e in log if e[0] == "share" and e[4] > 0)
    assert hits > 20


def test_cache_off_behaves_like_plain_allocator():
    """With the cache off, append_tokens/share_prefix equal append/new sequence."""
    rng = np.random.default_rng(5)
    for _ in range(30):
        nb, bs, mb = 16, 4, 5
        order = rng.permutation(nb)
        plain = BlockManager(nb, bs, mb, order)
        ids = BlockManager(nb, bs, mb, order)
        for s in range(8):
            toks = rng.integers(0, 3, size=int(rng.integers(0, 12))).tolist()
            assert ids.pkv_seq_share_prefix(s, toks) == (0, 0)
            a = plain.pkv_seq_append(s, len(toks))
            b = ids.pkv_seq_append_tokens(s, toks)
            assert a[0] == b[0] and a[1].tolist() == b[1].tolist()
            if rng.random() < 0.4:
                assert plain.pkv_seq_free(s) == ids.pkv_seq_free(s) == 0
        assert plain.pkv_stats() == ids.pkv_stats()
        assert ids.pkv_prefix_cache_stats() == (0, 0, 0, 0)


def test_invalid_arguments():
    mgr = BlockManager(8, 4, 4)
    assert mgr.pkv_alloc_set_prefix_cache(1) == 0
    from paged_kv_cache_320_b200 import _binding as B
    L = B.lib()
    assert L.pkv_alloc_set_prefix_cache(mgr._h, 2) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_seq_append_tokens(mgr._h, 0, None, 3, None, None, None) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_seq_share_prefix(mgr._h, 0, None, 3, None) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_seq_share_prefix(mgr._h, 0, None, 0, None) == 0
    assert L.pkv_seq_share_prefix(mgr._h, 0, None, 0, None) == B.PKV_ERR_SEQ_EXISTS
    assert L.pkv_prefix_cache_stats(None, None, None, None, None) == B.PKV_ERR_INVALID_ARG


def test_bench_request_stream_hits_every_repeated_prompt():
    """The benchmark's request stream (small): with the cache on, every request after the
    first of its prompt finds the whole prompt cached (whole blocks of it); off, none."""
    import bench
    from paged_kv_cache_320_b200 import synth
    sp = synth.SPECS["shared_prefix"]
    r = bench.prefix_cache_measurement(sp, requests=64, concurrency=8, decode_len=4)
    assert r["cache_off"]["prefill_tokens_cached"] == 0
    full = (sp.prefix // sp.block_size) * sp.block_size
    first_uses = r["prompts"]
    on = r["cache_on"]["prefill_tokens_cached"]
    assert on >= (64 - first_uses) * full
    assert r["cache_on"]["peak_blocks_held"] < r["cache_off"]["peak_blocks_held"]


def test_bench_memory_utilisation_matches_the_oracle():
    """The benchmark's pool utilisation equals the oracle's closed forms: paged
    Σ len / (Σ⌈len/bs⌉·bs) and contiguous Σ len / (B·max_len) on an unshared workload;
    with shared prefixes each shared slot counts once in the physical form."""
    import bench
    from oracle import utilisation as U
    from paged_kv_cache_320_b200 import synth
    wl = synth.make_workload("llama7b_mha", values_on="none")
    mgr = bench.replay_block_manager(wl)
    m = bench.memory_utilisation(wl, mgr)
    mgr.close()
    lens = wl.context_lens
    assert m["logical"] == pytest.approx(U.paged_utilisation(lens, 16), abs=1e-4)
    assert m["physical"] == m["logical"]
    assert m["contiguous_prealloc"] == pytest.approx(
        U.contiguous_utilisation(lens, wl.spec.max_len), abs=1e-4)
    wl = synth.make_workload("shared_prefix", values_on="none")
    mgr = bench.replay_block_manager(wl)
    m = bench.memory_utilisation(wl, mgr)
    mgr.close()
    sp = wl.spec
    unique = sp.prompts * sp.prefix + int((wl.context_lens - sp.prefix).sum())
    assert m["physical"] == pytest.approx(unique / (m["held_blocks"] * 16), abs=1e-4)
    assert m["logical"] > 1.0
