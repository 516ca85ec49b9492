"""GPU parity of paged decode attention (partition kernel + log-sum-exp reduce)
against the fp64 oracle, elementwise within 4e-3 + 1e-2*|ref|.

Small cases are compared in full; the full-size workloads (in the launch
configuration the benchmark uses) on sampled sequences — the longest, the
shortest and a seeded random remainder — whose oracle runs from host copies of
only their pages. Also: edge cases (one-token context, zero length, lengths at
block and partition boundaries, GQA 1..16, block sizes 8/16/32, head_dim 64/128,
fp16/bf16), NaN canaries in unused slots, placement invariance, and out-of-pool
block ids reported (read as zeros) instead of faulting."""
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_320_b200 as pkv
from oracle import attention as A
from oracle import cache_ops as C
from paged_kv_cache_320_b200 import synth
from tests.gpu_util import assert_close, sampled_oracle, to_bits, to_dev

pytestmark = pytest.mark.gpu


def decode_dev(q, kc, vc, bt, lens, max_len, scale, partition=0):
    out = torch.empty_like(q)
    pkv.pkv_paged_attention_decode(out, q, kc, vc, bt, lens, max_len, scale=scale,
                                   partition_size=partition)
    torch.cuda.synchronize()
    return out


def random_case(rng, lens, Hq, Hkv, D, BS, dtype, extra=5):
    """A pool with random placement; unused rows hold the NaN canary."""
    lens = np.asarray(lens, np.int32)
    nblk = [-(-int(n) // BS) for n in lens]
    nb = sum(nblk) + extra
    mb = max(max(nblk), 1) + 2
    perm = rng.permutation(nb).astype(np.int32)
    bt = np.full((len(lens), mb), -1, np.int32)
    off = 0
    kc = synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
    vc = synth.round_to_bits(rng.standard_normal((nb, Hkv, BS, D), dtype=np.float32), dtype)
    used = np.zeros((nb, BS), bool)
    for s, n in enumerate(lens):
        bt[s, :nblk[s]] = perm[off:off + nblk[s]]
        off += nblk[s]
        for t in range(int(n)):
            used[bt[s, t // BS], t % BS] = True
    kc.transpose(0, 2, 1, 3)[~used] = synth.CANARY[dtype]
    vc.transpose(0, 2, 1, 3)[~used] = synth.CANARY[dtype]
    q = synth.round_to_bits(rng.standard_normal((len(lens), Hq, D), dtype=np.float32), dtype)
    return q, kc, vc, bt, lens, mb * BS


def check_case(q, kc, vc, bt, lens, max_len, dtype, scale, partition=0, what=""):
    out = decode_dev(to_dev(q, dtype), to_dev(kc, dtype), to_dev(vc, dtype),
                     torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(), max_len, scale,
                     partition)
    ref = A.paged_decode_attention(q, kc, vc, bt, lens, scale, dtype)
    assert pkv.pkv_get_device_status() == 0
    return out, assert_close(to_bits(out), ref, dtype, what)


def test_tiny_workload_full_step(cuda_device):
    """One decode step of the tiny workload: cache write of 4 tokens, then attention."""
    wl = synth.make_workload("tiny")
    dt = wl.spec.dtype
    kc, vc = to_dev(wl.k_cache[0], dt), to_dev(wl.v_cache[0], dt)
    pkv.pkv_reshape_and_cache(to_dev(wl.k_new[0], dt), to_dev(wl.v_new[0], dt), kc, vc,
                              torch.from_numpy(wl.slot_mapping).cuda())
    out = decode_dev(to_dev(wl.q[0], dt), kc, vc, torch.from_numpy(wl.block_tables).cuda(),
                     torch.from_numpy(wl.context_lens).cuda(), 128, wl.scale)
    ek, ev = C.reshape_and_cache(wl.k_new[0], wl.v_new[0], wl.k_cache[0], wl.v_cache[0],
                                 wl.slot_mapping)
    ref = A.paged_decode_attention(wl.q[0], ek, ev, wl.block_tables, wl.context_lens, wl.scale, dt)
    assert_close(to_bits(out), ref, dt, "tiny")
    assert pkv.pkv_get_device_status() == 0


@pytest.mark.parametrize("partition", [64, 128])
def test_tiny_forced_partitions_exercise_reduce(cuda_device, partition):
    wl = synth.make_workload("tiny")
    dt = wl.spec.dtype
    check_case(wl.q[0], wl.k_cache[0], wl.v_cache[0], wl.block_tables,
               np.maximum(wl.context_lens - 1, 0).astype(np.int32), 128, dt, wl.scale,
               partition, f"tiny P={partition}")


@pytest.mark.parametrize("dtype", [synth.F16, synth.BF16])
@pytest.mark.parametrize("Hq,Hkv,D,BS", [
    (8, 8, 64, 16), (8, 2, 128, 16), (8, 2, 128, 8), (8, 2, 128, 32), (32, 8, 128, 16),
    (64, 8, 128, 32), (16, 1, 128, 16), (6, 2, 64, 8), (3, 1, 64, 32), (4, 4, 128, 8)])
def test_boundary_lengths(cuda_device, dtype, Hq, Hkv, D, BS):
    rng = np.random.default_rng(Hq * 131 + Hkv * 17 + D + BS + dtype)
    lens = [1, 2, BS - 1, BS, BS + 1, 15, 16, 17, 63, 64, 65, 127, 128, 129, 200, 511, 512, 513]
    q, kc, vc, bt, lens, max_len = random_case(rng, lens, Hq, Hkv, D, BS, dtype)
    check_case(q, kc, vc, bt, lens, max_len, dtype, 1 / math.sqrt(D), 0, "auto")
    check_case(q, kc, vc, bt, lens, max_len, dtype, 1 / math.sqrt(D), 64, "P=64")
    check_case(q, kc, vc, bt, lens, max_len, dtype, 0.3, 128, "P=128 scale=0.3")


def test_one_token_context_returns_v_row_exactly(cuda_device):
    rng = np.random.default_rng(50)
    dtype = synth.BF16
    q, kc, vc, bt, lens, max_len = random_case(rng, [1] * 7, 16, 2, 128, 16, dtype)
    out, _ = check_case(q, kc, vc, bt, lens, max_len, dtype, 0.088)
    got = to_bits(out)
    for s in range(7):
        for h in range(16):
            np.testing.assert_array_equal(got[s, h], vc[bt[s, 0], h // 8, 0])


def test_zero_length_context_gives_zero(cuda_device):
    rng = np.random.default_rng(51)
    dtype = synth.F16
    q, kc, vc, bt, lens, max_len = random_case(rng, [0, 5, 0, 300], 8, 2, 64, 16, dtype)
    out, _ = check_case(q, kc, vc, bt, lens, max_len, dtype, 0.125, 64)
    got = to_bits(out)
    assert (got[0] == 0).all() and (got[2] == 0).all()


def test_placement_invariance_on_gpu(cuda_device):
    rng = np.random.default_rng(52)
    dtype = synth.BF16
    q, kc, vc, bt, lens, max_len = random_case(rng, rng.integers(1, 900, 24), 32, 8, 128, 16,
                                               dtype)
    out1, _ = check_case(q, kc, vc, bt, lens, max_len, dtype, 0.088)
    newpos = rng.permutation(kc.shape[0])
    kc2 = np.empty_like(kc); vc2 = np.empty_like(vc)
    kc2[newpos] = kc; vc2[newpos] = vc
    bt2 = np.where(bt >= 0, newpos[np.maximum(bt, 0)], -1).astype(np.int32)
    out2, _ = check_case(q, kc2, vc2, bt2, lens, max_len, dtype, 0.088)
    np.testing.assert_array_equal(to_bits(out1), to_bits(out2))


def test_out_of_pool_block_id_is_reported_not_faulted(cuda_device):
    rng = np.random.default_rng(53)
    dtype = synth.BF16
    q, kc, vc, bt, lens, max_len = random_case(rng, [40, 40], 8, 2, 128, 16, dtype)
    bt_bad = bt.copy()
    bt_bad[1, 1] = kc.shape[0] + 1000        # past the pool
    pkv.pkv_get_device_status(clear=True)
    out = decode_dev(to_dev(q, dtype), to_dev(kc, dtype), to_dev(vc, dtype),
                     torch.from_numpy(bt_bad).cuda(), torch.from_numpy(lens).cuda(), max_len,
                     0.1)
    st = pkv.pkv_get_device_status(clear=True)
    assert st & pkv._binding.STATUS_BAD_BLOCK
    # the sequence with valid tables is unaffected
    ref = A.paged_decode_attention(q[:1], kc, vc, bt[:1], lens[:1], 0.1, dtype)
    assert_close(to_bits(out)[:1], ref, dtype, "valid sequence next to a bad one")
    assert np.isfinite(A.bits_to_f64(to_bits(out)[1], dtype)).all()


def test_context_len_above_bound_is_clamped_and_reported(cuda_device):
    rng = np.random.default_rng(54)
    dtype = synth.F16
    q, kc, vc, bt, lens, max_len = random_case(rng, [30, 64], 4, 4, 64, 16, dtype)
    lens_bad = lens.copy()
    lens_bad[0] = 10_000
    pkv.pkv_get_device_status(clear=True)
    out = decode_dev(to_dev(q, dtype), to_dev(kc, dtype), to_dev(vc, dtype),
                     torch.from_numpy(bt).cuda(), torch.from_numpy(lens_bad).cuda(), 64, 0.1)
    assert pkv.pkv_get_device_status(clear=True) & pkv._binding.STATUS_BAD_LEN
    ref = A.paged_decode_attention(q[1:], kc, vc, bt[1:], lens[1:], 0.1, dtype)
    assert_close(to_bits(out)[1:], ref, dtype, "unaffected sequence")


def test_workspace_too_small_is_rejected(cuda_device):
    q = torch.zeros(2, 8, 64, dtype=torch.float16, device="cuda")
    kc = torch.zeros(16, 8, 16, 64, dtype=torch.float16, device="cuda")
    bt = torch.zeros(2, 8, dtype=torch.int32, device="cuda")
    lens = torch.full((2,), 100, dtype=torch.int32, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.pkv_paged_attention_decode(torch.empty_like(q), q, kc, kc, bt, lens, 128,
                                       partition_size=64, workspace=ws)
    assert e.value.code == pkv._binding.PKV_ERR_WORKSPACE


# ----------------------------------------------------------------------------
# full-size workloads, sampled sequences
# ----------------------------------------------------------------------------
def full_step_and_sample(wl, layer, nsample, partition=0):
    sp = wl.spec
    dt = sp.dtype
    kc, vc = wl.k_cache[layer], wl.v_cache[layer]
    seqs = synth.sample_sequences(wl, nsample, seed=layer)
    q_bits = to_bits(wl.q[layer])
    kn_bits, vn_bits = to_bits(wl.k_new[layer]), to_bits(wl.v_new[layer])
    # oracle inputs: pages read BEFORE the GPU writes anything
    ref = sampled_oracle(q_bits, kc, vc, wl.block_tables, wl.context_lens, seqs, wl.scale, dt,
                         kn_bits, vn_bits, wl.slot_mapping)
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    pkv.pkv_reshape_and_cache(wl.k_new[layer], wl.v_new[layer], kc, vc,
                              torch.from_numpy(wl.slot_mapping).cuda())
    out = torch.empty_like(wl.q[layer])
    pkv.pkv_paged_attention_decode(out, wl.q[layer], kc, vc, bt, lens, sp.max_len,
                                   scale=wl.scale, partition_size=partition)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status() == 0
    got = to_bits(out)
    assert np.isfinite(A.bits_to_f64(got, dt)).all()
    return assert_close(got[seqs], ref, dt, f"{sp.name} layer {layer} seqs {seqs.tolist()}")


@pytest.mark.slow
def test_llama7b_mha_two_layers_sampled(cuda_device):
    wl = synth.make_workload("llama7b_mha", values_on="cuda", num_layers=2)
    for layer in range(2):
        full_step_and_sample(wl, layer, 6)


@pytest.mark.slow
def test_llama3_8b_gqa_sampled(cuda_device):
    wl = synth.make_workload("llama3_8b_gqa", values_on="cuda")
    full_step_and_sample(wl, 0, 8)


@pytest.mark.slow
def test_shared_prefix_decode_sampled(cuda_device):
    wl = synth.make_workload("shared_prefix", values_on="cuda")
    full_step_and_sample(wl, 0, 10)


@pytest.mark.slow
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_long_context_sampled(cuda_device, bs):
    wl = synth.make_workload("long_context", values_on="cuda", block_size=bs)
    full_step_and_sample(wl, 0, 2)


def test_one_workspace_reused_across_calls_and_batch_sizes(cuda_device):
    """One workspace serves calls of different batch sizes in turn: the work counter
    in its header is re-armed after every call and the partial rows of each call are
    written before they are read. Three rounds over three batch sizes."""
    rng = np.random.default_rng(55)
    dtype = synth.BF16
    cases = [random_case(rng, rng.integers(1, 700, n), 16, 4, 128, 16, dtype) for n in (5, 40, 17)]
    need = max(pkv.pkv_decode_workspace_size(len(c[4]), 16, 4, 128, 16, c[5], 64) for c in cases)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    refs = [A.paged_decode_attention(c[0], c[1], c[2], c[3], c[4], 0.09, dtype) for c in cases]
    dev = [tuple(to_dev(x, dtype) for x in c[:3]) + (torch.from_numpy(c[3]).cuda(),
                                                      torch.from_numpy(c[4]).cuda())
           for c in cases]
    for rnd in range(3):
        for i, (c, r, d) in enumerate(zip(cases, refs, dev)):
            out = torch.empty_like(d[0])
            pkv.pkv_paged_attention_decode(out, d[0], d[1], d[2], d[3], d[4], c[5], scale=0.09,
                                           partition_size=64, workspace=ws)
            torch.cuda.synchronize()
            assert_close(to_bits(out), r, dtype, f"round {rnd} case {i}")
    assert pkv.pkv_get_device_status() == 0


def test_many_partitions_merge(cuda_device):
    """Contexts of up to 5000 tokens at 64-token partitions: up to 79 partials merged."""
    rng = np.random.default_rng(56)
    dtype = synth.F16
    q, kc, vc, bt, lens, max_len = random_case(rng, [5000, 4097, 64, 65, 1], 8, 1, 128, 32, dtype)
    check_case(q, kc, vc, bt, lens, max_len, dtype, 0.088, 64, "P=64 long")


@pytest.mark.parametrize("nseq", [31, 32, 33, 1100])
def test_both_item_orders(cuda_device, nseq):
    """Up to 32 sequences the work items go out longest first; above, in sequence order.
    Both orders cover every item once: short, empty and multi-partition contexts mixed."""
    rng = np.random.default_rng(57 + nseq)
    dtype = synth.BF16
    lens = rng.integers(0, 300, nseq)
    lens[::7] = rng.integers(300, 3000, len(lens[::7]))
    lens[1] = 0
    q, kc, vc, bt, lens, max_len = random_case(rng, lens, 8, 2, 64, 16, dtype)
    for P in (64, 0):
        check_case(q, kc, vc, bt, lens, max_len, dtype, 0.125, P, f"B={nseq} P={P}")


@pytest.mark.parametrize("BS,P", [(8, 2048), (16, 4096)])
def test_items_of_256_blocks(cuda_device, BS, P):
    """Partitions of the largest size an item takes (256 blocks): eight table entries per
    producer lane."""
    rng = np.random.default_rng(58 + BS)
    dtype = synth.BF16
    q, kc, vc, bt, lens, max_len = random_case(rng, [9000, P, P + 1, 300, 2 * P - 5], 16, 2, 128,
                                               BS, dtype)
    check_case(q, kc, vc, bt, lens, max_len, dtype, 0.09, P, f"BS={BS} P={P}")


@pytest.mark.parametrize("nseq,Hq,Hkv,D,BS,P,dtype", [
    (40, 32, 8, 128, 16, 64, synth.BF16),      # sequence-major order, many partitions
    (20, 16, 16, 128, 32, 128, synth.F16),     # longest-first order (<= 32 sequences)
    (300, 8, 2, 64, 8, 256, synth.F16),
    (7, 64, 8, 128, 16, 0, synth.BF16)])
def test_partitions_then_merge_equal_the_decode(cuda_device, nseq, Hq, Hkv, D, BS, P, dtype):
    """The two launches of the decode as separate calls give its bits; the partitions
    call repeated on one workspace without a merge in between (each launch re-arms the
    work counter it used) gives the same partials, and the oracle agrees."""
    rng = np.random.default_rng(nseq + Hq + D + BS + P)
    lens = list(rng.integers(1, 1500, nseq))
    q, kc, vc, bt, lens, max_len = random_case(rng, lens, Hq, Hkv, D, BS, dtype)
    qd, kcd, vcd = to_dev(q, dtype), to_dev(kc, dtype), to_dev(vc, dtype)
    btd, lensd = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    ref_out = decode_dev(qd, kcd, vcd, btd, lensd, max_len, 0.07, P)
    need = pkv.pkv_decode_workspace_size(nseq, Hq, Hkv, D, BS, max_len, P)
    ws = torch.full((max(need, 16),), 0x5A, dtype=torch.uint8, device="cuda")
    pkv.pkv_get_device_status(clear=True)
    for rep in range(3):
        out = torch.full_like(qd, float("nan"))
        for _ in range(rep + 1):
            pkv.pkv_paged_attention_decode_partitions(out, qd, kcd, vcd, btd, lensd, max_len, ws,
                                                      scale=0.07, partition_size=P)
        pkv.pkv_paged_attention_merge(out, lensd, Hkv, BS, max_len, ws, partition_size=P)
        torch.cuda.synchronize()
        assert pkv.pkv_get_device_status() == 0
        assert np.array_equal(to_bits(out), to_bits(ref_out)), rep
    ref = A.paged_decode_attention(q, kc, vc, bt, lens, 0.07, dtype)
    assert_close(to_bits(out), ref, dtype, "partitions + merge")
