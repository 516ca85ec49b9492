"""GPU parity of the cache write and the block copy against the oracle: bit-exact,
every untouched byte unchanged (pools pre-filled with a NaN canary or random bits),
out-of-pool indices skipped and reported through the device status word."""
import numpy as np
import pytest
import torch

import paged_kv_cache_320_b200 as pkv
from oracle import cache_ops as C
from paged_kv_cache_320_b200 import synth
from tests.gpu_util import to_bits, to_dev

pytestmark = pytest.mark.gpu


def run_reshape(kn, vn, kc, vc, slots, dtype):
    kn_d, vn_d = to_dev(kn, dtype), to_dev(vn, dtype)
    kc_d, vc_d = to_dev(kc, dtype), to_dev(vc, dtype)
    sl_d = torch.from_numpy(np.asarray(slots, np.int64)).cuda()
    pkv.pkv_reshape_and_cache(kn_d, vn_d, kc_d, vc_d, sl_d)
    torch.cuda.synchronize()
    return to_bits(kc_d), to_bits(vc_d)


def test_reshape_and_cache_tiny_workload(cuda_device):
    wl = synth.make_workload("tiny")
    dt = wl.spec.dtype
    k, v = run_reshape(wl.k_new[0], wl.v_new[0], wl.k_cache[0], wl.v_cache[0], wl.slot_mapping, dt)
    ek, ev = C.reshape_and_cache(wl.k_new[0], wl.v_new[0], wl.k_cache[0], wl.v_cache[0],
                                 wl.slot_mapping)
    np.testing.assert_array_equal(k, ek)
    np.testing.assert_array_equal(v, ev)
    assert pkv.pkv_get_device_status() == 0


@pytest.mark.parametrize("dtype", [synth.F16, synth.BF16])
@pytest.mark.parametrize("D,BS", [(64, 8), (128, 16), (128, 32), (64, 32)])
def test_reshape_and_cache_edges(cuda_device, dtype, D, BS):
    rng = np.random.default_rng(40 + D + BS)
    NB, Hkv, T = 37, 3, 50
    kc = np.full((NB, Hkv, BS, D), synth.CANARY[dtype], np.uint16)
    vc = kc.copy()
    kn = synth.round_to_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32), dtype)
    vn = synth.round_to_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32), dtype)
    sl = rng.choice(np.arange(BS, NB * BS - 1), size=T, replace=False).astype(np.int64)
    sl[[0, 1, 2]] = [0, NB * BS - 1, BS - 1]   # first / last row of the pool, last row of a block
    sl[[5, 9, 30]] = -1                        # padding tokens
    k, v = run_reshape(kn, vn, kc, vc, sl, dtype)
    ek, ev = C.reshape_and_cache(kn, vn, kc, vc, sl)
    np.testing.assert_array_equal(k, ek)
    np.testing.assert_array_equal(v, ev)
    assert pkv.pkv_get_device_status() == 0


def test_reshape_and_cache_out_of_pool_slot_is_skipped_and_reported(cuda_device):
    rng = np.random.default_rng(41)
    dtype = synth.BF16
    NB, Hkv, BS, D = 8, 2, 16, 128
    kc = rng.integers(0, 1 << 16, (NB, Hkv, BS, D), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, (NB, Hkv, BS, D), dtype=np.uint16)
    kn = synth.round_to_bits(rng.standard_normal((3, Hkv, D), dtype=np.float32), dtype)
    vn = synth.round_to_bits(rng.standard_normal((3, Hkv, D), dtype=np.float32), dtype)
    sl = np.array([5, NB * BS, 17], dtype=np.int64)         # middle one is past the pool
    pkv.pkv_get_device_status(clear=True)
    k, v = run_reshape(kn, vn, kc, vc, sl, dtype)
    assert pkv.pkv_get_device_status(clear=True) & pkv._binding.STATUS_BAD_SLOT
    ek, ev = C.reshape_and_cache(kn, vn, kc, vc, np.array([5, -1, 17], np.int64))
    np.testing.assert_array_equal(k, ek)
    np.testing.assert_array_equal(v, ev)


def test_reshape_and_cache_full_gqa_workload(cuda_device):
    """256 new tokens into the Llama-3-8B-shaped pool (as the benchmark step does)."""
    wl = synth.make_workload("llama3_8b_gqa", values_on="cuda")
    kc, vc = wl.k_cache[0], wl.v_cache[0]
    before_k, before_v = to_bits(kc), to_bits(vc)
    kn, vn = wl.k_new[0], wl.v_new[0]
    sl = torch.from_numpy(wl.slot_mapping).cuda()
    pkv.pkv_reshape_and_cache(kn, vn, kc, vc, sl)
    torch.cuda.synchronize()
    ek, ev = C.reshape_and_cache(to_bits(kn), to_bits(vn), before_k, before_v, wl.slot_mapping)
    np.testing.assert_array_equal(to_bits(kc), ek)
    np.testing.assert_array_equal(to_bits(vc), ev)
    assert pkv.pkv_get_device_status() == 0


@pytest.mark.parametrize("layers,D,BS", [(1, 128, 16), (3, 128, 16), (2, 64, 8), (2, 128, 32)])
def test_copy_blocks_bit_exact(cuda_device, layers, D, BS):
    rng = np.random.default_rng(42 + layers + D)
    NB, Hkv = 60, 8
    dtype = synth.BF16
    kcs = [rng.integers(0, 1 << 16, (NB, Hkv, BS, D), dtype=np.uint16) for _ in range(layers)]
    vcs = [rng.integers(0, 1 << 16, (NB, Hkv, BS, D), dtype=np.uint16) for _ in range(layers)]
    blocks = rng.permutation(NB)
    pairs = np.stack([blocks[:14], blocks[14:28]], axis=1).astype(np.int32)   # distinct dsts
    kd = [to_dev(c, dtype) for c in kcs]
    vd = [to_dev(c, dtype) for c in vcs]
    kp = torch.tensor([t.data_ptr() for t in kd], dtype=torch.int64, device="cuda")
    vp = torch.tensor([t.data_ptr() for t in vd], dtype=torch.int64, device="cuda")
    pd = torch.from_numpy(pairs).cuda()
    pkv.pkv_copy_blocks(kp, vp, pd, Hkv, D, BS, NB, pkv.PKV_BF16)
    torch.cuda.synchronize()
    ek, ev = C.copy_blocks(kcs, vcs, pairs)
    for layer in range(layers):
        np.testing.assert_array_equal(to_bits(kd[layer]), ek[layer])
        np.testing.assert_array_equal(to_bits(vd[layer]), ev[layer])
    assert pkv.pkv_get_device_status() == 0


def test_copy_blocks_bad_pair_skipped_and_reported(cuda_device):
    rng = np.random.default_rng(43)
    NB, Hkv, BS, D = 10, 2, 16, 64
    kc = rng.integers(0, 1 << 16, (NB, Hkv, BS, D), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, (NB, Hkv, BS, D), dtype=np.uint16)
    kd, vd = to_dev(kc, synth.F16), to_dev(vc, synth.F16)
    kp = torch.tensor([kd.data_ptr()], dtype=torch.int64, device="cuda")
    vp = torch.tensor([vd.data_ptr()], dtype=torch.int64, device="cuda")
    pairs = np.array([[1, 2], [3, NB], [-1, 4], [5, 6]], dtype=np.int32)
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_copy_blocks(kp, vp, torch.from_numpy(pairs).cuda(), Hkv, D, BS, NB, pkv.PKV_F16)
    assert pkv.pkv_get_device_status(clear=True) & pkv._binding.STATUS_BAD_PAIR
    ek, ev = C.copy_blocks([kc], [vc], pairs[[0, 3]])
    np.testing.assert_array_equal(to_bits(kd), ek[0])
    np.testing.assert_array_equal(to_bits(vd), ev[0])
