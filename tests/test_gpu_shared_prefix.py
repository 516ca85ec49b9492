"""GPU parity of the shared-prefix-aware decode against the fp64 oracle (its result
is the plain definition of attention, so the same oracle applies), within
4e-3 + 1e-2*|ref|: the full shared-prefix workload (sampled sequences, and every
sequence against the plain decode kernel), random groups over head layouts, head
dims and block sizes, a declared prefix that the tables contradict, and a malformed
group list."""
import numpy as np
import pytest
import torch

import paged_kv_cache_320_b200 as pkv
from oracle import attention as A
from paged_kv_cache_320_b200 import synth
from tests.gpu_util import assert_close, sampled_oracle, to_bits, to_dev

pytestmark = pytest.mark.gpu


def grouped_case(rng, group_sizes, prefix_blocks, suffix_max, Hq, Hkv, D, BS, dtype):
    """Groups whose members share their first prefix_blocks[g] physical pages, then
    private pages; unwritten rows hold the NaN canary."""
    tables, lens = [], []
    next_page = 0
    perm_pages = []
    for gs, pb in zip(group_sizes, prefix_blocks):
        shared = list(range(next_page, next_page + pb))
        next_page += pb
        for _ in range(gs):
            extra = int(rng.integers(1, suffix_max + 1))
            n = pb * BS + extra
            own = -(-extra // BS)
            tables.append(shared + list(range(next_page, next_page + own)))
            next_page += own
            lens.append(n)
    nb = next_page + 3
    relabel = rng.permutation(nb)
    mb = max(len(t) for t in tables) + 1
    bt = np.full((len(tables), mb), -1, np.int32)
    for s, t in enumerate(tables):
        bt[s, :len(t)] = relabel[t]
    lens = np.array(lens, np.int32)
    kc = synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
    vc = synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
    used = np.zeros((nb, BS), bool)
    for s, n in enumerate(lens):
        for t in range(int(n)):
            used[bt[s, t // BS], t % BS] = True
    kc.transpose(0, 2, 1, 3)[~used] = synth.CANARY[dtype]
    vc.transpose(0, 2, 1, 3)[~used] = synth.CANARY[dtype]
    q = synth.round_to_bits(rng.standard_normal((len(lens), Hq, D), dtype=np.float32), dtype)
    starts = np.concatenate([[0], np.cumsum(group_sizes)]).astype(np.int32)
    pre = (np.array(prefix_blocks) * BS).astype(np.int32)
    return q, kc, vc, bt, lens, starts, pre, mb * BS


def run_shared(q, kc, vc, bt, lens, starts, pre, max_len, dtype, scale, partition=0):
    out = torch.empty(q.shape, dtype=torch.float16 if dtype == synth.F16 else torch.bfloat16,
                      device="cuda")
    pkv.pkv_paged_attention_decode_shared_prefix(
        out, to_dev(q, dtype), to_dev(kc, dtype), to_dev(vc, dtype),
        torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(),
        torch.from_numpy(np.asarray(starts, np.int32)).cuda(),
        torch.from_numpy(np.asarray(pre, np.int32)).cuda(), max_len, scale=scale,
        partition_size=partition)
    torch.cuda.synchronize()
    return to_bits(out)


@pytest.mark.parametrize("dtype", [synth.F16, synth.BF16])
@pytest.mark.parametrize("Hq,Hkv,D,BS", [(32, 8, 128, 16), (64, 8, 128, 32), (8, 8, 64, 8),
                                         (16, 1, 128, 16), (6, 2, 64, 16), (12, 4, 128, 8)])
def test_random_groups_match_oracle(cuda_device, dtype, Hq, Hkv, D, BS):
    rng = np.random.default_rng(Hq * 7 + Hkv * 3 + D + BS + dtype)
    sizes = [1, 8, 3, 5, 1, 17, 2]
    pblocks = [0, 9, 1, 20, 4, 6, 0]
    q, kc, vc, bt, lens, starts, pre, max_len = grouped_case(rng, sizes, pblocks, 150, Hq, Hkv,
                                                             D, BS, dtype)
    ref = A.paged_decode_attention(q, kc, vc, bt, lens, 0.1, dtype)
    pkv.pkv_get_device_status(clear=True)
    for partition in (0, 64, 128):
        got = run_shared(q, kc, vc, bt, lens, starts, pre, max_len, dtype, 0.1, partition)
        assert_close(got, ref, dtype, f"P={partition}")
    assert pkv.pkv_get_device_status() == 0


@pytest.mark.parametrize("Hq,Hkv,BS,P", [(32, 8, 16, 1024), (64, 8, 8, 2048), (32, 8, 32, 2048)])
def test_long_prefix_items(cuda_device, Hq, Hkv, BS, P):
    """Prefix items of 1024 and 2048 tokens (the shared path's automatic sizes at full
    batch; 256 blocks of 8 at most), over prefixes that span several such items."""
    rng = np.random.default_rng(Hq + BS + P)
    dtype = synth.BF16
    q, kc, vc, bt, lens, starts, pre, max_len = grouped_case(
        rng, [5, 4], [2304 // BS, 1536 // BS], 300, Hq, Hkv, 128, BS, dtype)
    ref = A.paged_decode_attention(q, kc, vc, bt, lens, 0.08, dtype)
    pkv.pkv_get_device_status(clear=True)
    got = run_shared(q, kc, vc, bt, lens, starts, pre, max_len, dtype, 0.08, P)
    assert_close(got, ref, dtype, f"P={P}")
    assert pkv.pkv_get_device_status() == 0


def test_prefix_declared_longer_than_shared_is_cut(cuda_device):
    """Members share 6 pages but the caller declares 12 (and longer than one member):
    the plan cuts the prefix at the first differing page; results stay exact."""
    rng = np.random.default_rng(60)
    dtype = synth.BF16
    q, kc, vc, bt, lens, starts, pre, max_len = grouped_case(rng, [6, 4], [6, 3], 200, 32, 8,
                                                             128, 16, dtype)
    ref = A.paged_decode_attention(q, kc, vc, bt, lens, 0.09, dtype)
    wrong = np.array([12 * 16, 10_000], np.int32)
    got = run_shared(q, kc, vc, bt, lens, starts, wrong, max_len, dtype, 0.09, 64)
    assert_close(got, ref, dtype, "over-declared prefix")
    assert pkv.pkv_get_device_status() == 0


def test_malformed_groups_fall_back_to_no_sharing(cuda_device):
    rng = np.random.default_rng(61)
    dtype = synth.F16
    q, kc, vc, bt, lens, starts, pre, max_len = grouped_case(rng, [3, 3], [4, 2], 90, 8, 2, 64,
                                                             16, dtype)
    ref = A.paged_decode_attention(q, kc, vc, bt, lens, 0.2, dtype)
    pkv.pkv_get_device_status(clear=True)
    got = run_shared(q, kc, vc, bt, lens, np.array([0, 4, 5], np.int32), pre, max_len, dtype,
                     0.2)   # does not end at num_seqs
    assert pkv.pkv_get_device_status(clear=True) & pkv._binding.STATUS_BAD_LEN
    assert_close(got, ref, dtype, "malformed groups")


@pytest.mark.slow
def test_shared_prefix_workload_full_size(cuda_device):
    """16 prompts x 8 samples sharing a 1024-token prefix (the shared-prefix workload):
    sampled sequences against the oracle, every sequence against plain decode."""
    wl = synth.make_workload("shared_prefix", values_on="cuda")
    sp = wl.spec
    dt = sp.dtype
    kc, vc = wl.k_cache[0], wl.v_cache[0]
    seqs = synth.sample_sequences(wl, 10, seed=3)
    q_bits = to_bits(wl.q[0])
    # this step's token is written first (its slot still holds the NaN canary)
    ref = sampled_oracle(q_bits, kc, vc, wl.block_tables, wl.context_lens, seqs, wl.scale, dt,
                         to_bits(wl.k_new[0]), to_bits(wl.v_new[0]), wl.slot_mapping)
    pkv.pkv_reshape_and_cache(wl.k_new[0], wl.v_new[0], kc, vc,
                              torch.from_numpy(wl.slot_mapping).cuda())
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    starts = torch.arange(0, wl.num_seqs + 1, sp.samples, dtype=torch.int32, device="cuda")
    pre = torch.full((sp.prompts,), sp.prefix, dtype=torch.int32, device="cuda")
    out_s = torch.empty_like(wl.q[0])
    out_p = torch.empty_like(wl.q[0])
    pkv.pkv_paged_attention_decode_shared_prefix(out_s, wl.q[0], kc, vc, bt, lens, starts, pre,
                                                 sp.max_len, scale=wl.scale)
    pkv.pkv_paged_attention_decode(out_p, wl.q[0], kc, vc, bt, lens, sp.max_len, scale=wl.scale)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status() == 0
    got_s, got_p = to_bits(out_s), to_bits(out_p)
    assert_close(got_s[seqs], ref, dt, "shared path, sampled")
    # both GPU paths approximate the same fp64 result: compare them on every sequence
    a, b = A.bits_to_f64(got_s, dt), A.bits_to_f64(got_p, dt)
    assert np.all(np.abs(a - b) <= 2 * (4e-3 + 1e-2 * np.abs(b)))


def test_large_batch_plans_in_workspace_scratch(cuda_device):
    """6400 short sequences in groups of 4: the plan's per-sequence scratch no longer
    fits in shared memory and lives in the workspace."""
    rng = np.random.default_rng(62)
    dtype = synth.BF16
    ngroups = 1600
    q, kc, vc, bt, lens, starts, pre, max_len = grouped_case(
        rng, [4] * ngroups, list(rng.integers(0, 3, ngroups)), 20, 8, 2, 64, 16, dtype)
    assert len(lens) > 6144
    ref = A.paged_decode_attention(q, kc, vc, bt, lens, 0.125, dtype)
    pkv.pkv_get_device_status(clear=True)
    got = run_shared(q, kc, vc, bt, lens, starts, pre, max_len, dtype, 0.125)
    assert pkv.pkv_get_device_status() == 0
    assert_close(got, ref, dtype, "6400 sequences")


def test_one_plan_serves_several_layers(cuda_device):
    """pkv_shared_prefix_plan once, then the planned decode for three layers (own caches
    and queries, shared tables): each equals the one-call path bit for bit and the oracle."""
    rng = np.random.default_rng(63)
    dtype = synth.BF16
    Hq, Hkv, D, BS = 32, 8, 128, 16
    q0, kc0, vc0, bt, lens, starts, pre, max_len = grouped_case(rng, [8, 3, 5], [10, 2, 6], 120,
                                                                Hq, Hkv, D, BS, dtype)
    canary = kc0 == synth.CANARY[dtype]
    layers = []
    for _ in range(3):
        kc = synth.round_to_bits(rng.standard_normal(kc0.shape, dtype=np.float32), dtype)
        vc = synth.round_to_bits(rng.standard_normal(vc0.shape, dtype=np.float32), dtype)
        kc[canary] = synth.CANARY[dtype]
        vc[canary] = synth.CANARY[dtype]
        q = synth.round_to_bits(rng.standard_normal(q0.shape, dtype=np.float32), dtype)
        layers.append((q, kc, vc))
    btd, lensd = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    startsd = torch.from_numpy(np.asarray(starts, np.int32)).cuda()
    pred = torch.from_numpy(np.asarray(pre, np.int32)).cuda()
    ws = torch.empty(pkv.pkv_decode_shared_prefix_workspace_size(len(lens), Hq, Hkv, D, BS,
                                                                 max_len, 64),
                     dtype=torch.uint8, device="cuda")
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_shared_prefix_plan(btd, lensd, startsd, pred, Hq, Hkv, D, BS, max_len, ws,
                               partition_size=64)
    for i, (q, kc, vc) in enumerate(layers):
        qd, kcd, vcd = to_dev(q, dtype), to_dev(kc, dtype), to_dev(vc, dtype)
        out = torch.empty_like(qd)
        pkv.pkv_paged_attention_decode_shared_prefix_planned(out, qd, kcd, vcd, btd, lensd,
                                                             max_len, ws, scale=0.1,
                                                             partition_size=64)
        torch.cuda.synchronize()
        got = to_bits(out)
        one_call = run_shared(q, kc, vc, bt, lens, starts, pre, max_len, dtype, 0.1, 64)
        assert np.array_equal(got, one_call), f"layer {i}"
        ref = A.paged_decode_attention(q, kc, vc, bt, lens, 0.1, dtype)
        assert_close(got, ref, dtype, f"layer {i}")
    assert pkv.pkv_get_device_status() == 0


def test_planned_call_with_other_sizes_writes_nothing(cuda_device):
    rng = np.random.default_rng(64)
    dtype = synth.F16
    q, kc, vc, bt, lens, starts, pre, max_len = grouped_case(rng, [4, 4], [3, 5], 60, 16, 4, 64,
                                                             16, dtype)
    btd, lensd = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    ws = torch.empty(max(pkv.pkv_decode_shared_prefix_workspace_size(len(lens), 16, 4, 64, 16,
                                                                     max_len, p)
                         for p in (64, 128)), dtype=torch.uint8, device="cuda")
    pkv.pkv_shared_prefix_plan(btd, lensd, torch.from_numpy(np.asarray(starts, np.int32)).cuda(),
                               torch.from_numpy(np.asarray(pre, np.int32)).cuda(), 16, 4, 64, 16,
                               max_len, ws, partition_size=128)
    qd = to_dev(q, dtype)
    out = torch.full_like(qd, 3.0)
    pkv.pkv_get_device_status(clear=True)
    # planned for 128-token partitions, called with 64
    pkv.pkv_paged_attention_decode_shared_prefix_planned(out, qd, to_dev(kc, dtype),
                                                         to_dev(vc, dtype), btd, lensd, max_len,
                                                         ws, partition_size=64)
    assert pkv.pkv_get_device_status() & pkv._binding.STATUS_WORKSPACE
    assert (out == 3.0).all()


def explicit_case(rng, groups, Hq, Hkv, D, BS, dtype):
    """groups: (prefix tokens, [suffix tokens of each member]); members share the
    prefix's pages. Unwritten rows hold the NaN canary."""
    tables, lens, starts, pre = [], [], [0], []
    page = 0
    for ptok, sufs in groups:
        assert ptok % BS == 0
        shared = list(range(page, page + ptok // BS))
        page += ptok // BS
        for suf in sufs:
            own = -(-suf // BS)
            tables.append(shared + list(range(page, page + own)))
            page += own
            lens.append(ptok + suf)
        starts.append(starts[-1] + len(sufs))
        pre.append(ptok)
    nb = page + 2
    relabel = rng.permutation(nb)
    mb = max(1, max(len(t) for t in tables)) + 1
    bt = np.full((len(tables), mb), -1, np.int32)
    for s, t in enumerate(tables):
        bt[s, :len(t)] = relabel[t]
    lens = np.array(lens, np.int32)
    kc = synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
    vc = synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
    used = np.zeros((nb, BS), bool)
    for s, n in enumerate(lens):
        for t in range(int(n)):
            used[bt[s, t // BS], t % BS] = True
    kc.transpose(0, 2, 1, 3)[~used] = synth.CANARY[dtype]
    vc.transpose(0, 2, 1, 3)[~used] = synth.CANARY[dtype]
    q = synth.round_to_bits(rng.standard_normal((len(lens), Hq, D), dtype=np.float32), dtype)
    return (q, kc, vc, bt, lens, np.array(starts, np.int32), np.array(pre, np.int32),
            mb * BS)


@pytest.mark.parametrize("Hq,Hkv,BS", [(32, 8, 16), (16, 2, 32), (8, 8, 8), (12, 2, 16),
                                        (10, 2, 8)])
def test_chunks_fused_split_and_empty(cuda_device, Hq, Hkv, BS):
    """Chunks whose prefix and suffixes form one item (written directly) next to chunks
    split into several items (merged in the launch by the chunk's last item): members with
    no suffix, suffixes longer than a partition, a group whose members hold nothing at all,
    groups of one and a group of 19 members; G = 6 and 5 leave chunks of fewer than 16
    rows; each at the automatic partition and at small ones."""
    rng = np.random.default_rng(Hq + Hkv + BS)
    dtype = synth.F16
    groups = [(64 * BS, [0, 3, 0, 700, 1, 0, 65, 64, 2]),   # mixed suffixes, some none
              (0, [0, 0, 0]),                                  # empty contexts
              (2 * BS, [1]),                                   # a group of one
              (0, [900]),
              (10 * BS, [0, 0]),                               # the prefix is everything
              (5 * BS, [130, 2, 2500, 17]),
              (3 * BS, [int(x) for x in rng.integers(0, 90, 19)])]        # 19 members
    q, kc, vc, bt, lens, starts, pre, max_len = explicit_case(rng, groups, Hq, Hkv, 128, BS,
                                                              dtype)
    ref = A.paged_decode_attention(q, kc, vc, bt, lens, 0.09, dtype)
    pkv.pkv_get_device_status(clear=True)
    for partition in (0, 256, 64):
        got = run_shared(q, kc, vc, bt, lens, starts, pre, max_len, dtype, 0.09, partition)
        assert_close(got, ref, dtype, f"P={partition}")
    assert pkv.pkv_get_device_status() == 0
