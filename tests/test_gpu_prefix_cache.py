"""Decode through blocks found by prefix caching ("vLLM / PagedAttention — 分页 KV Cache
分析" §2.3 and §3.2: common prefixes such as a system prompt are found automatically and
their pages reused across requests; §五: only identical token sequences share).

A request stream with three system prompts is admitted through the library's block
manager with the cache on (pkv_seq_share_prefix, then pkv_seq_append_tokens for what was
not cached); each token the request appends has its K/V written through
pkv_reshape_and_cache; some requests finish (their cached blocks stay, evictable) and
later requests find them again. A token's K/V is drawn from a generator seeded by the
hash of the token's whole prefix, as a model's would be a function of it: a block is
reused only if it holds exactly what the new request would have written.

Checked against the oracle: the oracle's block-manager model, given the same calls,
returns the same statuses, cached-token counts, slots and tables (bit-exact); the device
pool equals the oracle's cache writes; every live sequence's pages hold exactly the K/V of
its own prefixes; the decode over the shared pages equals the oracle's attention on the
model's tables (4e-3 + 1e-2|ref|). And the sharing is physical: requests on the same
prompt hold the same prompt blocks; pkv_prefix_groups finds them (as the oracle's model
groups them) and the shared-prefix-aware decode over those groups equals the oracle too."""
import numpy as np
import pytest
import torch

import paged_kv_cache_320_b200 as pkv
from oracle import attention as A
from oracle import block_manager as BM
from oracle import cache_ops as C
from paged_kv_cache_320_b200 import synth
from tests.gpu_util import assert_close, to_bits, to_dev

pytestmark = pytest.mark.gpu

BS, HQ, HKV, D, NB, MB = 16, 8, 2, 64, 96, 16
DT = synth.F16


def token_kv(tokens, t):
    """K and V rows [Hkv, D] of position t of a sequence: a function of tokens[:t + 1]."""
    rng = np.random.default_rng(BM.prefix_hash(tokens[:t + 1]) & ((1 << 63) - 1))
    k = synth.round_to_bits(rng.standard_normal((HKV, D), dtype=np.float32), DT)
    v = synth.round_to_bits(rng.standard_normal((HKV, D), dtype=np.float32), DT)
    return k, v


def test_decode_over_prefix_cached_blocks(cuda_device):
    rng = np.random.default_rng(2024)
    prompts = [rng.integers(0, 32000, n, dtype=np.int32).tolist() for n in (96, 64, 40)]
    lib_mgr = pkv.BlockManager(NB, BS, MB)
    model = BM.BlockManagerModel(NB, BS, MB)
    assert lib_mgr.pkv_alloc_set_prefix_cache(1) == 0
    model.set_prefix_cache(True)
    kc_d = torch.zeros((NB, HKV, BS, D), dtype=torch.float16, device="cuda")
    vc_d = torch.zeros_like(kc_d)
    kc_o = np.zeros((NB, HKV, BS, D), np.uint16)
    vc_o = np.zeros_like(kc_o)
    seqs = {}                                   # live request id -> its token ids
    cached_tokens = 0

    def admit(sid, toks):
        nonlocal kc_o, vc_o, cached_tokens
        st, got = lib_mgr.pkv_seq_share_prefix(sid, toks[:-1])
        mst, mgot = model.share_prefix(sid, toks[:-1])
        assert (st, got) == (mst, mgot) and st == 0
        st, slots, cows = lib_mgr.pkv_seq_append_tokens(sid, toks[got:])
        mst, mslots, mcows = model.append_tokens(sid, toks[got:])
        assert st == mst == 0 and slots.tolist() == mslots and len(cows) == len(mcows) == 0
        kv = [token_kv(toks, t) for t in range(got, len(toks))]
        kn = np.stack([k for k, _ in kv])
        vn = np.stack([v for _, v in kv])
        pkv.pkv_reshape_and_cache(to_dev(kn, DT), to_dev(vn, DT), kc_d, vc_d,
                                  torch.from_numpy(slots).cuda())
        kc_o, vc_o = C.reshape_and_cache(kn, vn, kc_o, vc_o, slots)
        seqs[sid] = toks
        cached_tokens += got

    def request(p, qlen):
        return prompts[p] + rng.integers(0, 32000, qlen, dtype=np.int32).tolist()

    # first wave: every prompt's first request fills the cache; later ones hit it
    sid = 0
    for p in (0, 1, 0, 2, 1, 0):
        admit(sid, request(p, int(rng.integers(3, 40))))
        sid += 1
    assert cached_tokens >= 96 + 64 + 96           # prompts 0 (twice more) and 1 (once more)
    # some requests finish: their cached blocks stay, evictable, and are found again
    for done in (0, 3, 4):
        assert lib_mgr.pkv_seq_free(done) == model.free(done) == 0
        del seqs[done]
    before = cached_tokens
    for p in (2, 1, 0, 2):
        admit(sid, request(p, int(rng.integers(3, 40))))
        sid += 1
    assert cached_tokens - before >= 32 + 64 + 96 + 32
    assert lib_mgr.pkv_prefix_cache_stats()[:2] == model.prefix_cache_stats()[:2]

    ids = np.array(sorted(seqs), np.int64)
    st, tables, lens = lib_mgr.pkv_block_tables(ids)
    assert st == 0
    mt = np.array([model.block_table(int(s))[0] for s in ids], np.int32)
    ml = np.array([model.block_table(int(s))[1] for s in ids], np.int32)
    assert np.array_equal(tables, mt) and np.array_equal(lens, ml)
    # physical sharing: requests on one prompt hold the same full prompt blocks
    by_prompt = {}
    for i, s in enumerate(ids):
        for p, pr in enumerate(prompts):
            if seqs[int(s)][:len(pr)] == pr:
                by_prompt.setdefault(p, []).append(i)
    for p, rows in by_prompt.items():
        full = len(prompts[p]) // BS
        assert len(rows) >= 2
        for i in rows[1:]:
            assert np.array_equal(tables[i, :full], tables[rows[0], :full])

    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status() == 0
    assert np.array_equal(to_bits(kc_d), kc_o) and np.array_equal(to_bits(vc_d), vc_o)
    # every live sequence's pages hold the K/V of its own prefixes
    for i, s in enumerate(ids):
        toks = seqs[int(s)]
        for t in range(len(toks)):
            b, r = tables[i, t // BS], t % BS
            k, v = token_kv(toks, t)
            assert np.array_equal(kc_o[b, :, r, :], k) and np.array_equal(vc_o[b, :, r, :], v)

    q = synth.round_to_bits(rng.standard_normal((len(ids), HQ, D), dtype=np.float32), DT)
    out = torch.empty((len(ids), HQ, D), dtype=torch.float16, device="cuda")
    for P in (64, 0):                               # several partitions, then one
        pkv.pkv_paged_attention_decode(out, to_dev(q, DT), kc_d, vc_d,
                                       torch.from_numpy(tables).cuda(),
                                       torch.from_numpy(lens).cuda(), MB * BS, partition_size=P)
        torch.cuda.synchronize()
        assert pkv.pkv_get_device_status() == 0
        ref = A.paged_decode_attention(q, kc_o, vc_o, mt, ml, 1 / np.sqrt(D), DT)
        assert_close(to_bits(out), ref, DT, f"prefix-cached decode, partition {P}")

    # the groups the block manager finds for the shared-prefix-aware decode: the oracle
    # model's grouping of the same tables, one group per prompt holding at least the
    # prompt's full blocks, and the grouped decode equal to the oracle's attention
    st, order, gstart, gpre = lib_mgr.pkv_prefix_groups(ids)
    morder, mstart, mpre = model.prefix_groups(ids)
    assert st == 0
    assert order.tolist() == morder and gstart.tolist() == mstart and gpre.tolist() == mpre
    pos = {int(s): i for i, s in enumerate(ids)}
    perm = np.array([pos[int(s)] for s in order])
    for p, rows in by_prompt.items():
        members = {int(ids[i]) for i in rows}
        g = [k for k in range(len(gstart) - 1)
             if members <= set(order[gstart[k]:gstart[k + 1]].tolist())]
        assert len(g) == 1 and gpre[g[0]] >= len(prompts[p]) // BS * BS
    qg, tg, lg = q[perm], tables[perm], lens[perm]
    for P in (64, 0):
        pkv.pkv_paged_attention_decode_shared_prefix(
            out, to_dev(qg, DT), kc_d, vc_d, torch.from_numpy(np.ascontiguousarray(tg)).cuda(),
            torch.from_numpy(np.ascontiguousarray(lg)).cuda(), torch.from_numpy(gstart).cuda(),
            torch.from_numpy(gpre).cuda(), MB * BS, partition_size=P)
        torch.cuda.synchronize()
        assert pkv.pkv_get_device_status() == 0
        ref = A.paged_decode_attention(qg, kc_o, vc_o, mt[perm], ml[perm], 1 / np.sqrt(D), DT)
        assert_close(to_bits(out), ref, DT, f"prefix-cached shared-prefix decode, partition {P}")
    lib_mgr.close()
