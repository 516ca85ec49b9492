"""GPU parity of the decode step on the device: pkv_device_append against the oracle's
block-manager model (bit-exact tables, lengths, slots and free-list use, the same
rules as an in-order host append), and pkv_paged_decode_step against the cache write
followed by the decode (identical bits) and against the fp64 oracle (4e-3 + 1e-2|ref|),
with refusals (short free list, full table, length bound, a foreign workspace) leaving
everything unchanged."""
import numpy as np
import pytest
import torch

import paged_kv_cache_320_b200 as pkv
from oracle import attention as A
from oracle import block_manager as BM
from oracle import cache_ops as C
from paged_kv_cache_320_b200 import synth
from tests.gpu_util import assert_close, sampled_oracle, to_bits, to_dev
from tests.test_gpu_decode import random_case

pytestmark = pytest.mark.gpu

NO_BLOCKS = pkv._binding.STATUS_NO_BLOCKS
WORKSPACE = pkv._binding.STATUS_WORKSPACE
SHARED = pkv._binding.STATUS_SHARED_BLOCK
TIMEOUT = pkv._binding.STATUS_WAIT_TIMEOUT


def model_state(rng, nb, bs, mb, nseq, max_len0):
    """A model allocator with nseq sequences (ids 0..nseq-1), some of them forks of a
    block-aligned parent, and a free stack shuffled by frees."""
    order = rng.permutation(nb)
    m = BM.BlockManagerModel(nb, bs, mb, order)
    junk = 10_000
    for j in range(6):                      # sequences that are freed again: shuffle the stack
        m.append(junk + j, int(rng.integers(1, 3 * bs)))
    s = 0
    while s < nseq:
        if s and rng.random() < 0.2:
            parent = int(rng.integers(0, s))
            if m.lens[parent] % bs == 0:
                assert m.fork(parent, s) == 0
                s += 1
                continue
        n = int(rng.integers(0, max_len0))
        if rng.random() < 0.25:
            n = (n // bs) * bs                 # block-aligned: the append takes a new block
        assert m.append(s, n)[0] == 0
        s += 1
    for j in range(6):
        m.free(junk + j)
    return m


def upload_model(m, nseq):
    rows = [m.block_table(s) for s in range(nseq)]
    bt = np.array([r for r, _ in rows], np.int32)
    lens = np.array([n for _, n in rows], np.int32)
    return bt, lens


@pytest.mark.parametrize("seed", range(8))
def test_device_append_matches_model(cuda_device, seed):
    rng = np.random.default_rng(900 + seed)
    bs = int(rng.choice([8, 16, 32]))
    nseq = int(rng.choice([1, 7, 300, 1500]))
    mb = 12
    nb = nseq * mb + 64
    m = model_state(rng, nb, bs, mb, nseq, (mb - 1) * bs)
    bt, lens = upload_model(m, nseq)
    fl = np.array(m.free_list(), np.int32)
    skip = int(rng.integers(0, 5))            # entries already used by earlier steps
    fl_dev = np.concatenate([np.full(skip, -1, np.int32), fl])
    bt_d, lens_d = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    used = torch.tensor([skip], dtype=torch.int32, device="cuda")
    slots = torch.full((nseq,), -7, dtype=torch.int64, device="cuda")
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_device_append(bt_d, lens_d, torch.from_numpy(fl_dev).cuda(), used, nb, mb * bs, bs,
                          slots_out=slots)
    assert pkv.pkv_get_device_status() == 0
    exp_slots = []
    before = len(m.free_stack)
    for s in range(nseq):
        st, sl, cw = m.append(s, 1)
        assert st == 0 and not cw
        exp_slots.append(sl[0])
    taken = before - len(m.free_stack)
    ebt, elens = upload_model(m, nseq)
    np.testing.assert_array_equal(bt_d.cpu().numpy(), ebt)
    np.testing.assert_array_equal(lens_d.cpu().numpy(), elens)
    np.testing.assert_array_equal(slots.cpu().numpy(), np.array(exp_slots, np.int64))
    assert int(used.item()) == skip + taken


@pytest.mark.parametrize("why", ["short list", "table full", "length bound", "bad entry"])
def test_device_append_refuses_and_changes_nothing(cuda_device, why):
    rng = np.random.default_rng(77)
    bs, mb, nseq = 16, 6, 40
    lens = rng.integers(1, (mb - 1) * bs, nseq).astype(np.int32)
    lens[::5] = (lens[::5] // bs) * bs + bs     # these take a block
    bt = rng.integers(0, 500, (nseq, mb)).astype(np.int32)
    fl = np.arange(600, 700, dtype=np.int32)
    max_len = mb * bs
    need = int((lens % bs == 0).sum())
    if why == "short list":
        fl = fl[:need - 1]
    elif why == "table full":
        lens[3] = mb * bs
        max_len = mb * bs + 1
    elif why == "length bound":
        max_len = int(lens.max())
    else:
        fl[need // 2] = 10_000                  # outside the pool of 1000 blocks
    bt_d, lens_d = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    used = torch.zeros(1, dtype=torch.int32, device="cuda")
    slots = torch.full((nseq,), -7, dtype=torch.int64, device="cuda")
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_device_append(bt_d, lens_d, torch.from_numpy(fl).cuda(), used, 1000, max_len, bs,
                          slots_out=slots)
    assert pkv.pkv_get_device_status() & NO_BLOCKS
    np.testing.assert_array_equal(bt_d.cpu().numpy(), bt)
    np.testing.assert_array_equal(lens_d.cpu().numpy(), lens)
    assert int(used.item()) == 0
    assert (slots.cpu().numpy() == -7).all()


def step_case(rng, lens, Hq, Hkv, D, BS, dtype):
    """random_case with post-step lengths; the newest token's row holds the NaN canary
    (only the step's own write may fill it)."""
    q, kc, vc, bt, lens, max_len = random_case(rng, lens, Hq, Hkv, D, BS, dtype)
    slots = np.full(len(lens), -1, np.int64)
    for s, n in enumerate(lens):
        if n > 0:
            slots[s] = int(bt[s, (n - 1) // BS]) * BS + (n - 1) % BS
            kc[slots[s] // BS, :, slots[s] % BS, :] = synth.CANARY[dtype]
            vc[slots[s] // BS, :, slots[s] % BS, :] = synth.CANARY[dtype]
    kn = synth.round_to_bits(rng.standard_normal((len(lens), Hkv, D), dtype=np.float32), dtype)
    vn = synth.round_to_bits(rng.standard_normal((len(lens), Hkv, D), dtype=np.float32), dtype)
    return q, kc, vc, bt, lens, max_len, slots, kn, vn


def step_ws(q, kc, max_len, P):
    B, Hq, D = q.shape
    _, Hkv, BS, _ = kc.shape
    n = pkv.pkv_decode_step_workspace_size(B, Hq, Hkv, D, BS, max_len, P)
    return torch.zeros(n, dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("dtype", [synth.F16, synth.BF16])
@pytest.mark.parametrize("Hq,Hkv,D,BS,P", [(32, 8, 128, 16, 0), (32, 8, 128, 16, 64),
                                           (32, 8, 128, 16, 1024), (8, 2, 64, 32, 2048),
                                           (64, 8, 128, 32, 128), (8, 8, 64, 8, 64),
                                           (16, 1, 128, 16, 0), (6, 2, 64, 16, 192),
                                           (12, 4, 128, 8, 64)])
def test_step_equals_cache_write_then_decode(cuda_device, dtype, Hq, Hkv, D, BS, P):
    """Several partitions (merged in the step launch) and, with P >= the longest context,
    one partition (the write-and-decode kernel alone)."""
    rng = np.random.default_rng(Hq + 3 * Hkv + D + BS + P + dtype)
    lens = list(rng.integers(1, 700, 29)) + [0, 1, BS, BS + 1, 64, 65, 512, 513]
    q, kc, vc, bt, lens, max_len, slots, kn, vn = step_case(rng, lens, Hq, Hkv, D, BS, dtype)
    qd, knd, vnd = to_dev(q, dtype), to_dev(kn, dtype), to_dev(vn, dtype)
    btd, lensd = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    # unfused: cache write, then decode
    kc1, vc1 = to_dev(kc, dtype), to_dev(vc, dtype)
    pkv.pkv_reshape_and_cache(knd, vnd, kc1, vc1, torch.from_numpy(slots).cuda())
    out1 = torch.empty_like(qd)
    pkv.pkv_paged_attention_decode(out1, qd, kc1, vc1, btd, lensd, max_len, scale=0.11,
                                   partition_size=P)
    # fused
    kc2, vc2 = to_dev(kc, dtype), to_dev(vc, dtype)
    out2 = torch.empty_like(qd)
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_paged_decode_step(out2, qd, knd, vnd, kc2, vc2, btd, lensd, max_len,
                              step_ws(q, kc, max_len, P), scale=0.11, partition_size=P)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status() == 0
    assert torch.equal(kc1.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc1.view(torch.int16), vc2.view(torch.int16))
    assert np.array_equal(to_bits(out1), to_bits(out2))
    # and against the oracle
    ek, ev = C.reshape_and_cache(kn, vn, kc, vc, slots)
    ref = A.paged_decode_attention(q, ek, ev, bt, lens, 0.11, dtype)
    assert_close(to_bits(out2), ref, dtype, f"P={P}")


def test_full_step_append_then_layers_matches_oracle(cuda_device):
    """Device append, then three layers of decode steps (own caches, shared tables),
    against the oracle model's append and the fp64 oracle per layer."""
    rng = np.random.default_rng(31)
    dtype, Hq, Hkv, D, BS, L = synth.BF16, 16, 4, 128, 16, 3
    nseq, mb = 24, 40
    nb = nseq * mb + 16
    m = model_state(rng, nb, BS, mb, nseq, 30 * BS)
    bt, lens = upload_model(m, nseq)
    fl = np.array(m.free_list(), np.int32)
    for s in range(nseq):
        m.append(s, 1)
    ebt, elens = upload_model(m, nseq)
    eslots = np.array([int(ebt[s, (n - 1) // BS]) * BS + (n - 1) % BS for s, n in enumerate(elens)])
    max_len = mb * BS
    btd, lensd = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    used = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_device_append(btd, lensd, torch.from_numpy(fl).cuda(), used, nb, max_len, BS)
    ws = None
    for layer in range(L):
        kc = synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
        vc = synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
        q = synth.round_to_bits(rng.standard_normal((nseq, Hq, D), dtype=np.float32), dtype)
        kn = synth.round_to_bits(rng.standard_normal((nseq, Hkv, D), dtype=np.float32), dtype)
        vn = synth.round_to_bits(rng.standard_normal((nseq, Hkv, D), dtype=np.float32), dtype)
        kcd, vcd, qd = to_dev(kc, dtype), to_dev(vc, dtype), to_dev(q, dtype)
        if ws is None:
            ws = step_ws(q, kc, max_len, 64)
        out = torch.empty_like(qd)
        pkv.pkv_paged_decode_step(out, qd, to_dev(kn, dtype), to_dev(vn, dtype), kcd, vcd, btd,
                                  lensd, max_len, ws, partition_size=64)
        torch.cuda.synchronize()
        ek, ev = C.reshape_and_cache(kn, vn, kc, vc, eslots)
        assert np.array_equal(to_bits(kcd), ek) and np.array_equal(to_bits(vcd), ev)
        ref = A.paged_decode_attention(q, ek, ev, ebt, elens, 1 / np.sqrt(D), dtype)
        assert_close(to_bits(out), ref, dtype, f"layer {layer}")
    assert pkv.pkv_get_device_status() == 0
    np.testing.assert_array_equal(btd.cpu().numpy(), ebt)
    np.testing.assert_array_equal(lensd.cpu().numpy(), elens)


def test_workspace_reused_across_shapes(cuda_device):
    """One zero-filled workspace through 12 launches of different batch sizes, grids and
    partition counts: each launch leaves the header ready for the next."""
    rng = np.random.default_rng(44)
    dtype = synth.F16
    ws = torch.zeros(64 << 20, dtype=torch.uint8, device="cuda")
    pkv.pkv_get_device_status(clear=True)
    for i in range(12):
        nseq = int(rng.choice([1, 5, 64, 300]))
        P = int(rng.choice([64, 128, 0]))
        lens = rng.integers(1, 1200, nseq)
        q, kc, vc, bt, lens, max_len, slots, kn, vn = step_case(rng, lens, 8, 2, 64, 16, dtype)
        qd = to_dev(q, dtype)
        out = torch.empty_like(qd)
        kcd, vcd = to_dev(kc, dtype), to_dev(vc, dtype)
        pkv.pkv_paged_decode_step(out, qd, to_dev(kn, dtype), to_dev(vn, dtype), kcd, vcd,
                                  torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(),
                                  max_len, ws, scale=0.2, partition_size=P)
        torch.cuda.synchronize()
        assert pkv.pkv_get_device_status() == 0, i
        ek, ev = C.reshape_and_cache(kn, vn, kc, vc, slots)
        ref = A.paged_decode_attention(q, ek, ev, bt, lens, 0.2, dtype)
        assert_close(to_bits(out), ref, dtype, f"launch {i}")


def test_foreign_workspace_is_refused(cuda_device):
    rng = np.random.default_rng(45)
    dtype = synth.BF16
    q, kc, vc, bt, lens, max_len, slots, kn, vn = step_case(rng, [900, 40, 2000], 16, 4, 128, 16,
                                                            dtype)
    qd = to_dev(q, dtype)
    ws = step_ws(q, kc, max_len, 64)
    ws.fill_(0x5A)                              # never zeroed: not a step workspace
    out = torch.full_like(qd, 7.0)
    kcd = to_dev(kc, dtype)
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_paged_decode_step(out, qd, to_dev(kn, dtype), to_dev(vn, dtype), kcd,
                              to_dev(vc, dtype), torch.from_numpy(bt).cuda(),
                              torch.from_numpy(lens).cuda(), max_len, ws, partition_size=64)
    assert pkv.pkv_get_device_status() & WORKSPACE
    assert (out == 7.0).all()
    assert np.array_equal(to_bits(kcd), kc)     # no write either


@pytest.mark.slow
def test_gqa_workload_step_full_size(cuda_device):
    """The GQA workload (256 sequences, 1 layer) as the benchmark's fused step runs it:
    sampled sequences against the oracle, all of them against the unfused path."""
    wl = synth.make_workload("llama3_8b_gqa", values_on="cuda")
    sp = wl.spec
    dt = sp.dtype
    seqs = synth.sample_sequences(wl, 8, seed=5)
    kc, vc = wl.k_cache[0], wl.v_cache[0]
    ref = sampled_oracle(to_bits(wl.q[0]), kc, vc, wl.block_tables, wl.context_lens, seqs,
                         wl.scale, dt, to_bits(wl.k_new[0]), to_bits(wl.v_new[0]),
                         wl.slot_mapping)
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    kc2, vc2 = kc.clone(), vc.clone()
    out_f = torch.empty_like(wl.q[0])
    ws = torch.zeros(pkv.pkv_decode_step_workspace_size(wl.num_seqs, sp.num_heads,
                                                        sp.num_kv_heads, sp.head_dim,
                                                        sp.block_size, sp.max_len),
                     dtype=torch.uint8, device="cuda")
    kn = wl.k_new[0].view(wl.num_seqs, sp.num_kv_heads, sp.head_dim)
    vn = wl.v_new[0].view(wl.num_seqs, sp.num_kv_heads, sp.head_dim)
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_paged_decode_step(out_f, wl.q[0], kn, vn, kc2, vc2, bt, lens, sp.max_len, ws,
                              scale=wl.scale)
    pkv.pkv_reshape_and_cache(wl.k_new[0], wl.v_new[0], kc, vc,
                              torch.from_numpy(wl.slot_mapping).cuda())
    out_u = torch.empty_like(wl.q[0])
    pkv.pkv_paged_attention_decode(out_u, wl.q[0], kc, vc, bt, lens, sp.max_len, scale=wl.scale)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status() == 0
    assert torch.equal(kc.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), vc2.view(torch.int16))
    assert np.array_equal(to_bits(out_f), to_bits(out_u))
    assert_close(to_bits(out_f)[seqs], ref, dt, "fused step, sampled")


def fused_full_size(wl, layer, nsample, seed):
    """The benchmark's fused step on a full-size workload layer: sampled sequences against
    the oracle, every sequence bit for bit against cache write + decode."""
    sp = wl.spec
    dt = sp.dtype
    B = wl.num_seqs
    seqs = synth.sample_sequences(wl, nsample, seed=seed)
    kc, vc = wl.k_cache[layer], wl.v_cache[layer]
    ref = sampled_oracle(to_bits(wl.q[layer]), kc, vc, wl.block_tables, wl.context_lens, seqs,
                         wl.scale, dt, to_bits(wl.k_new[layer]), to_bits(wl.v_new[layer]),
                         wl.slot_mapping)
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    kc2, vc2 = kc.clone(), vc.clone()
    ws = torch.zeros(pkv.pkv_decode_step_workspace_size(B, sp.num_heads, sp.num_kv_heads,
                                                        sp.head_dim, sp.block_size, sp.max_len),
                     dtype=torch.uint8, device="cuda")
    out_f = torch.empty_like(wl.q[layer])
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_paged_decode_step(out_f, wl.q[layer],
                              wl.k_new[layer].view(B, sp.num_kv_heads, sp.head_dim),
                              wl.v_new[layer].view(B, sp.num_kv_heads, sp.head_dim), kc2, vc2,
                              bt, lens, sp.max_len, ws, scale=wl.scale)
    pkv.pkv_reshape_and_cache(wl.k_new[layer], wl.v_new[layer], kc, vc,
                              torch.from_numpy(wl.slot_mapping).cuda())
    out_u = torch.empty_like(wl.q[layer])
    pkv.pkv_paged_attention_decode(out_u, wl.q[layer], kc, vc, bt, lens, sp.max_len,
                                   scale=wl.scale)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status() == 0
    assert torch.equal(kc.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), vc2.view(torch.int16))
    assert np.array_equal(to_bits(out_f), to_bits(out_u))
    assert_close(to_bits(out_f)[seqs], ref, dt, f"{sp.name} layer {layer}, fused step")


@pytest.mark.slow
def test_llama7b_mha_fused_step_full_size(cuda_device):
    """The default workload's layers: write-and-decode kernel + reduce (2048 pairs)."""
    wl = synth.make_workload("llama7b_mha", values_on="cuda", num_layers=2)
    for layer in range(2):
        fused_full_size(wl, layer, 6, seed=11 + layer)


@pytest.mark.slow
@pytest.mark.parametrize("bs", [8, 32])
def test_long_context_fused_step_full_size(cuda_device, bs):
    """Long contexts: the step kernel merges in its own launch (512 pairs, longest-first
    item order)."""
    wl = synth.make_workload("long_context", values_on="cuda", block_size=bs)
    B, sp = wl.num_seqs, wl.spec
    assert pkv.pkv_decode_step_launches(B, sp.num_heads, sp.num_kv_heads, sp.head_dim, bs,
                                        sp.max_len) == 1
    fused_full_size(wl, 0, 2, seed=13)


@pytest.mark.parametrize("nseq,Hq,P", [(12, 8, 64), (64, 32, 64)])
def test_fused_step_replays_in_a_cuda_graph(cuda_device, nseq, Hq, P):
    """Device append + two fused layers captured once in a CUDA graph and replayed three
    times equal the same three steps run eagerly, bit for bit (tables, lengths, free-list
    cursor, caches, outputs). Small batches merge in the step launch (cooperative), larger
    ones launch the reduce kernel."""
    rng = np.random.default_rng(70 + nseq)
    dtype, Hkv, D, BS, L = synth.F16, 4, 64, 16, 2
    mb = 24
    nb = nseq * mb + 32
    m = model_state(rng, nb, BS, mb, nseq, 12 * BS)
    bt0, lens0 = upload_model(m, nseq)
    fl = np.array(m.free_list(), np.int32)
    max_len = mb * BS
    kc0 = [synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
           for _ in range(L)]
    vc0 = [synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
           for _ in range(L)]
    q = [to_dev(synth.round_to_bits(rng.standard_normal((nseq, Hq, D), dtype=np.float32), dtype),
                dtype) for _ in range(L)]
    kn = [to_dev(synth.round_to_bits(rng.standard_normal((nseq, Hkv, D), dtype=np.float32),
                                     dtype), dtype) for _ in range(L)]
    vn = [to_dev(synth.round_to_bits(rng.standard_normal((nseq, Hkv, D), dtype=np.float32),
                                     dtype), dtype) for _ in range(L)]

    def fresh():
        st = dict(bt=torch.from_numpy(bt0).cuda(), lens=torch.from_numpy(lens0).cuda(),
                  free=torch.from_numpy(fl).cuda(), used=torch.zeros(1, dtype=torch.int32,
                                                                     device="cuda"),
                  kc=[to_dev(x, dtype) for x in kc0], vc=[to_dev(x, dtype) for x in vc0],
                  out=[torch.empty_like(x) for x in q],
                  ws=torch.zeros(pkv.pkv_decode_step_workspace_size(nseq, Hq, Hkv, D, BS,
                                                                    max_len, P),
                                 dtype=torch.uint8, device="cuda"))
        return st

    def step(st):
        pkv.pkv_device_append(st["bt"], st["lens"], st["free"], st["used"], nb, max_len, BS)
        for l in range(L):
            pkv.pkv_paged_decode_step(st["out"][l], q[l], kn[l], vn[l], st["kc"][l], st["vc"][l],
                                      st["bt"], st["lens"], max_len, st["ws"], scale=0.125,
                                      partition_size=P)

    pkv.pkv_get_device_status(clear=True)
    eager = fresh()
    for _ in range(3):
        step(eager)
    torch.cuda.synchronize()
    graphed = fresh()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=side):
        step(graphed)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status() == 0
    for key in ("bt", "lens", "used"):
        assert torch.equal(eager[key], graphed[key]), key
    for l in range(L):
        assert torch.equal(eager["kc"][l].view(torch.int16), graphed["kc"][l].view(torch.int16))
        assert torch.equal(eager["vc"][l].view(torch.int16), graphed["vc"][l].view(torch.int16))
        assert torch.equal(eager["out"][l].view(torch.int16), graphed["out"][l].view(torch.int16))
    del g


def test_device_append_refuses_a_shared_partial_block(cuda_device):
    """A shared page is copied before it is changed ("分页 KV Cache 分析" §3.2). After a fork,
    parent and child share a partly filled last block; given the host manager's reference
    counts, the device append refuses the step (nothing written: tables, lengths, cursor
    and slots as they were) instead of writing into the page the sibling still reads.
    Sequences forked at a block boundary write into new blocks: that step is accepted and
    equals the host manager's own append."""
    bs, mb, nb = 16, 8, 64
    mgr = pkv.BlockManager(nb, bs, mb, np.arange(nb, dtype=np.int32)[::-1].copy())
    assert mgr.pkv_seq_append(0, 20)[0] == 0          # 16 + 4: partly filled last block
    assert mgr.pkv_seq_append(1, 32)[0] == 0          # two full blocks
    assert mgr.pkv_seq_fork(0, 2) == 0
    assert mgr.pkv_seq_fork(1, 3) == 0
    refc = torch.from_numpy(mgr.pkv_alloc_refcounts()).cuda()
    free = torch.from_numpy(mgr.pkv_alloc_free_list()).cuda()

    def upload(ids):
        st, tables, lens = mgr.pkv_block_tables(np.array(ids, np.int64))
        assert st == 0
        return torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()

    bt, lens = upload([0, 1, 2, 3])
    bt0, lens0 = bt.clone(), lens.clone()
    used = torch.zeros(1, dtype=torch.int32, device="cuda")
    slots = torch.full((4,), -7, dtype=torch.int64, device="cuda")
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_device_append(bt, lens, free, used, nb, mb * bs, bs, slots_out=slots,
                          block_refcounts=refc)
    st = pkv.pkv_get_device_status(clear=True)
    assert st & NO_BLOCKS and st & SHARED, st
    assert torch.equal(bt, bt0) and torch.equal(lens, lens0)
    assert used.item() == 0 and bool((slots == -7).all())

    # block-aligned forks: both sequences take a fresh block, as the host manager does
    bt, lens = upload([1, 3])
    pkv.pkv_device_append(bt, lens, free, used, nb, mb * bs, bs, slots_out=slots[:2],
                          block_refcounts=refc)
    assert pkv.pkv_get_device_status(clear=True) == 0
    st, done, sl, cows = mgr.pkv_seq_append_batch(np.array([1, 3], np.int64), 1)
    assert st == 0 and len(cows) == 0
    _, tables, lens_h = mgr.pkv_block_tables(np.array([1, 3], np.int64))
    assert np.array_equal(bt.cpu().numpy(), tables) and np.array_equal(lens.cpu().numpy(), lens_h)
    assert slots[:2].cpu().numpy().tolist() == sl[:, 0].tolist()
    assert used.item() == 2
    mgr.close()


K_SCHED_ARMED = int(np.array([0x9A6EDC0D], np.uint32).view(np.int32)[0])
K_STEP_ARMED = int(np.array([0x57E9A11D], np.uint32).view(np.int32)[0])


def header(ws):
    """The step workspace header's words: armed, next, arrive, gen, exit."""
    return ws[:20].view(torch.int32)


def in_launch_merge_case(seed):
    """Three sequences of several 64-token partitions, merged inside the step launch."""
    rng = np.random.default_rng(seed)
    dtype = synth.BF16
    case = step_case(rng, [900, 40, 2000], 16, 4, 128, 16, dtype)
    q, kc = case[0], case[1]
    assert pkv.pkv_decode_step_launches(len(case[4]), 16, 4, 128, 16, case[5], 64) == 1
    return dtype, case


def run_step(dtype, case, ws, out):
    q, kc, vc, bt, lens, max_len, slots, kn, vn = case
    kcd, vcd = to_dev(kc, dtype), to_dev(vc, dtype)
    pkv.pkv_paged_decode_step(out, to_dev(q, dtype), to_dev(kn, dtype), to_dev(vn, dtype), kcd,
                              vcd, torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(),
                              max_len, ws, partition_size=64)
    return kcd, vcd


def oracle_step(dtype, case):
    q, kc, vc, bt, lens, max_len, slots, kn, vn = case
    ek, ev = C.reshape_and_cache(kn, vn, kc, vc, slots)
    return ek, ev, A.paged_decode_attention(q, ek, ev, bt, lens, 1 / np.sqrt(128), dtype)


def test_header_with_a_stale_exit_count_is_refused(cuda_device):
    """A header armed by the reduce kernel must come with cleared counters: one whose
    exit count is not 0 (no CTA would ever see itself last, the work counter would never
    be reset and later launches would skip items) is refused before any write."""
    dtype, case = in_launch_merge_case(46)
    q, kc = case[0], case[1]
    ws = step_ws(q, kc, case[5], 64)
    h = header(ws)
    h[0] = K_SCHED_ARMED
    h[4] = 5
    before = ws[:256].clone()
    out = torch.full((len(case[4]), 16, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    pkv.pkv_get_device_status(clear=True)
    kcd, vcd = run_step(dtype, case, ws, out)
    assert pkv.pkv_get_device_status(clear=True) & WORKSPACE
    assert (out == 7.0).all()
    assert np.array_equal(to_bits(kcd), kc)            # no cache write either
    assert torch.equal(ws[:256], before)


def test_workspace_of_a_plain_decode_serves_the_step(cuda_device):
    """A workspace never zero-filled, used first by the plain decode (whose reduce kernel
    re-arms it and clears the step counters), is a valid step workspace afterwards."""
    dtype, case = in_launch_merge_case(47)
    q, kc, vc, bt, lens, max_len, slots, kn, vn = case
    ws = step_ws(q, kc, max_len, 64)
    ws.fill_(0x5A)
    qd = to_dev(q, dtype)
    out = torch.empty_like(qd)
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_paged_attention_decode(out, qd, to_dev(kc, dtype), to_dev(vc, dtype),
                                   torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(),
                                   max_len, partition_size=64, workspace=ws)
    torch.cuda.synchronize()
    h = header(ws).cpu().numpy()
    assert h[0] == K_SCHED_ARMED and h[1] == 0 and h[2] == 0 and h[4] == 0
    kcd, vcd = run_step(dtype, case, ws, out)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status(clear=True) == 0
    ek, ev, ref = oracle_step(dtype, case)
    assert np.array_equal(to_bits(kcd), ek) and np.array_equal(to_bits(vcd), ev)
    assert_close(to_bits(out), ref, dtype, "step after a plain decode")
    assert header(ws)[0].item() == K_STEP_ARMED


def test_grid_barrier_gives_up_and_the_workspace_recovers(cuda_device):
    """The bounded grid barrier of the in-launch merge runs out: an arrival count left in
    the header (as if by an interrupted launch) means no CTA is ever the last to arrive,
    so every CTA gives up after its poll limit. The launch returns with
    PKV_STATUS_WAIT_TIMEOUT (and PKV_STATUS_WORKSPACE for the stale count) set, skips the
    merge, and the last CTA out leaves the header re-armed with its counters cleared; the
    next step on the same workspace is correct."""
    dtype, case = in_launch_merge_case(48)
    q, kc = case[0], case[1]
    ws = step_ws(q, kc, case[5], 64)
    header(ws)[2] = -(1 << 31)                         # arrive = 0x80000000
    out = torch.empty((len(case[4]), 16, 128), dtype=torch.bfloat16, device="cuda")
    pkv.pkv_get_device_status(clear=True)
    run_step(dtype, case, ws, out)
    st = pkv.pkv_get_device_status(clear=True)
    assert st & TIMEOUT and st & WORKSPACE, st
    h = header(ws).cpu().numpy()
    assert h[0] == K_STEP_ARMED and h[1] == 0 and h[2] == 0 and h[4] == 0
    out2 = torch.empty_like(out)
    kcd, vcd = run_step(dtype, case, ws, out2)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status(clear=True) == 0
    ek, ev, ref = oracle_step(dtype, case)
    assert np.array_equal(to_bits(kcd), ek) and np.array_equal(to_bits(vcd), ev)
    assert_close(to_bits(out2), ref, dtype, "step after a barrier timeout")


@pytest.mark.parametrize("Hq,Hkv,D,BS,P", [(32, 8, 128, 16, 64), (16, 16, 128, 16, 512),
                                           (8, 2, 64, 32, 128)])
def test_step_partitions_then_merge_equal_the_step(cuda_device, Hq, Hkv, D, BS, P):
    """The write-and-decode launch alone, then the merge, on one workspace, step after
    step: the bits of the fused step call (which for these shapes may merge in its own
    launch) and the same cache writes."""
    rng = np.random.default_rng(Hq * 7 + BS + P)
    dtype = synth.F16
    lens = list(rng.integers(1, 1300, 37))
    q, kc, vc, bt, lens, max_len, slots, kn, vn = step_case(rng, lens, Hq, Hkv, D, BS, dtype)
    qd, knd, vnd = to_dev(q, dtype), to_dev(kn, dtype), to_dev(vn, dtype)
    btd, lensd = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    kc1, vc1 = to_dev(kc, dtype), to_dev(vc, dtype)
    out1 = torch.empty_like(qd)
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_paged_decode_step(out1, qd, knd, vnd, kc1, vc1, btd, lensd, max_len,
                              step_ws(q, kc, max_len, P), partition_size=P)
    ws = step_ws(q, kc, max_len, P)
    for rep in range(3):
        kc2, vc2 = to_dev(kc, dtype), to_dev(vc, dtype)
        out2 = torch.full_like(qd, float("nan"))
        pkv.pkv_paged_decode_step_partitions(out2, qd, knd, vnd, kc2, vc2, btd, lensd, max_len,
                                             ws, partition_size=P)
        pkv.pkv_paged_attention_merge(out2, lensd, Hkv, BS, max_len, ws, partition_size=P)
        torch.cuda.synchronize()
        assert pkv.pkv_get_device_status() == 0
        assert np.array_equal(to_bits(out1), to_bits(out2)), rep
        assert torch.equal(kc1.view(torch.int16), kc2.view(torch.int16))
        assert torch.equal(vc1.view(torch.int16), vc2.view(torch.int16))


def test_one_partition_steps_arm_and_reuse_the_header(cuda_device):
    """Contexts that are one partition each (the automatic choice for up to 64 sequences of
    short contexts with at least 1024 items): the first launch on a zero-filled workspace
    runs the static schedule and arms the header, the next ones take their items from the
    work counter; every launch equals the cache write + decode and the oracle."""
    rng = np.random.default_rng(77)
    dtype, Hq, Hkv, D, BS = synth.F16, 32, 32, 128, 16
    lens = list(rng.integers(1, 1500, 40))
    q, kc, vc, bt, lens, max_len, slots, kn, vn = step_case(rng, lens, Hq, Hkv, D, BS, dtype)
    P = pkv.pkv_decode_partition_size(len(lens), Hq, Hkv, D, BS, max_len)
    assert P >= max_len                                   # one partition per context
    assert pkv.pkv_decode_step_launches(len(lens), Hq, Hkv, D, BS, max_len) == 1
    ws = step_ws(q, kc, max_len, 0)
    assert ws.numel() == 256                              # the header alone
    ek, ev = C.reshape_and_cache(kn, vn, kc, vc, slots)
    ref = A.paged_decode_attention(q, ek, ev, bt, lens, 1 / np.sqrt(D), dtype)
    qd, knd, vnd = to_dev(q, dtype), to_dev(kn, dtype), to_dev(vn, dtype)
    btd, lensd = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    pkv.pkv_get_device_status(clear=True)
    first = None
    for launch in range(4):
        kcd, vcd = to_dev(kc, dtype), to_dev(vc, dtype)
        out = torch.full_like(qd, float("nan"))
        pkv.pkv_paged_decode_step(out, qd, knd, vnd, kcd, vcd, btd, lensd, max_len, ws)
        torch.cuda.synchronize()
        assert pkv.pkv_get_device_status() == 0
        assert header(ws)[0].item() == K_SCHED_ARMED and header(ws)[1].item() == 0
        assert np.array_equal(to_bits(kcd), ek) and np.array_equal(to_bits(vcd), ev)
        if first is None:
            first = to_bits(out)
            assert_close(first, ref, dtype, "one-partition step")
        else:
            assert np.array_equal(to_bits(out), first), launch
