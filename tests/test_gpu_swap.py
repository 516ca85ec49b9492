"""GPU parity of pkv_swap_blocks (whole blocks of every layer between the caches and
pinned host memory) against the oracle: bit-exact, untouched blocks unchanged, bad
ids reported, buffers that are not pinned host memory rejected before any launch."""
import numpy as np
import pytest
import torch

import paged_kv_cache_320_b200 as pkv
from oracle import cache_ops as C
from paged_kv_cache_320_b200 import synth
from tests.gpu_util import to_bits, to_dev

pytestmark = pytest.mark.gpu


def setup(rng, L, NB, Hkv, BS, D, dtype):
    kcs = [rng.integers(0, 1 << 16, (NB, Hkv, BS, D), dtype=np.uint16) for _ in range(L)]
    vcs = [rng.integers(0, 1 << 16, (NB, Hkv, BS, D), dtype=np.uint16) for _ in range(L)]
    kd = [to_dev(c, dtype) for c in kcs]
    vd = [to_dev(c, dtype) for c in vcs]
    kp = torch.tensor([t.data_ptr() for t in kd], dtype=torch.int64, device="cuda")
    vp = torch.tensor([t.data_ptr() for t in vd], dtype=torch.int64, device="cuda")
    return kcs, vcs, kd, vd, kp, vp


@pytest.mark.parametrize("L,D,BS", [(1, 128, 16), (3, 128, 8), (2, 64, 32)])
def test_swap_out_and_in_bit_exact(cuda_device, L, D, BS):
    rng = np.random.default_rng(80 + L + D + BS)
    NB, Hkv, dtype = 40, 8, synth.BF16
    kcs, vcs, kd, vd, kp, vp = setup(rng, L, NB, Hkv, BS, D, dtype)
    out_ids = np.array(rng.choice(NB, size=13, replace=False), np.int32)
    buf = torch.empty((L, 2, 13, Hkv, BS, D), dtype=torch.int16).pin_memory()
    pkv.pkv_swap_blocks(kp, vp, torch.from_numpy(out_ids).cuda(), buf, 1, Hkv, D, BS, NB,
                        pkv.PKV_BF16)
    torch.cuda.synchronize()
    expect = C.swap_out(kcs, vcs, out_ids)
    np.testing.assert_array_equal(buf.numpy().view(np.uint16), expect)
    # swap back into other blocks of the same pool
    in_ids = np.array([b for b in range(NB) if b not in out_ids][:13], np.int32)
    pkv.pkv_swap_blocks(kp, vp, torch.from_numpy(in_ids).cuda(), buf, 0, Hkv, D, BS, NB,
                        pkv.PKV_BF16)
    torch.cuda.synchronize()
    ek, ev = C.swap_in(kcs, vcs, in_ids, expect)
    for layer in range(L):
        np.testing.assert_array_equal(to_bits(kd[layer]), ek[layer])
        np.testing.assert_array_equal(to_bits(vd[layer]), ev[layer])
    assert pkv.pkv_get_device_status() == 0


def test_swap_rejects_buffers_that_are_not_pinned_host_memory(cuda_device):
    rng = np.random.default_rng(81)
    NB, Hkv, BS, D = 8, 2, 16, 64
    kcs, vcs, kd, vd, kp, vp = setup(rng, 1, NB, Hkv, BS, D, synth.F16)
    ids = torch.tensor([1, 2], dtype=torch.int32, device="cuda")
    for buf in (torch.empty((1, 2, 2, Hkv, BS, D), dtype=torch.int16),            # pageable
                torch.empty((1, 2, 2, Hkv, BS, D), dtype=torch.int16, device="cuda"),  # device
                torch.empty((1, 2, 1, Hkv, BS, D), dtype=torch.int16).pin_memory()):   # small
        with pytest.raises(pkv.PagedKVError) as e:
            pkv.pkv_swap_blocks(kp, vp, ids, buf, 1, Hkv, D, BS, NB, pkv.PKV_F16)
        assert e.value.code == pkv._binding.PKV_ERR_INVALID_ARG


def test_swap_bad_id_skipped_and_reported(cuda_device):
    rng = np.random.default_rng(82)
    NB, Hkv, BS, D = 8, 2, 16, 64
    kcs, vcs, kd, vd, kp, vp = setup(rng, 1, NB, Hkv, BS, D, synth.F16)
    buf = torch.zeros((1, 2, 3, Hkv, BS, D), dtype=torch.int16).pin_memory()
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_swap_blocks(kp, vp, torch.tensor([2, NB + 5, 4], dtype=torch.int32, device="cuda"),
                        buf, 1, Hkv, D, BS, NB, pkv.PKV_F16)
    assert pkv.pkv_get_device_status(clear=True) & pkv._binding.STATUS_BAD_PAIR
    b = buf.numpy().view(np.uint16)
    np.testing.assert_array_equal(b[0, 0, 0], kcs[0][2])
    np.testing.assert_array_equal(b[0, 0, 2], kcs[0][4])
    assert (b[0, :, 1] == 0).all()


@pytest.mark.parametrize("L,D,BS,tiles", [(1, 128, 16, 2), (3, 128, 8, 5), (2, 64, 32, 64),
                                          (2, 128, 16, 7)])
def test_staged_swap_out_and_in_bit_exact(cuda_device, L, D, BS, tiles):
    """The staged swap (a device buffer of `tiles` tiles in two halves, one large copy per
    half-buffer chunk; 2 tiles: a copy per tile, 5 or 7: ragged last chunk, 64: one or two
    chunks) gives the oracle's host buffer and cache contents, and the same buffer as the
    one-kernel swap."""
    rng = np.random.default_rng(90 + L + D + BS + tiles)
    NB, Hkv, dtype = 40, 8, synth.BF16
    kcs, vcs, kd, vd, kp, vp = setup(rng, L, NB, Hkv, BS, D, dtype)
    out_ids = np.array(rng.choice(NB, size=13, replace=False), np.int32)
    tile = Hkv * BS * D * 2
    staging = torch.empty(tiles * tile + 16, dtype=torch.uint8, device="cuda")
    buf = torch.full((L, 2, 13, Hkv, BS, D), -1, dtype=torch.int16).pin_memory()
    ids_d = torch.from_numpy(out_ids).cuda()
    pkv.pkv_swap_blocks_staged(kp, vp, ids_d, buf, 1, Hkv, D, BS, NB, pkv.PKV_BF16, staging)
    torch.cuda.synchronize()
    expect = C.swap_out(kcs, vcs, out_ids)
    np.testing.assert_array_equal(buf.numpy().view(np.uint16), expect)
    direct = torch.zeros_like(buf).pin_memory()
    pkv.pkv_swap_blocks(kp, vp, ids_d, direct, 1, Hkv, D, BS, NB, pkv.PKV_BF16)
    torch.cuda.synchronize()
    assert torch.equal(direct, buf)
    in_ids = np.array([b for b in range(NB) if b not in out_ids][:13], np.int32)
    pkv.pkv_swap_blocks_staged(kp, vp, torch.from_numpy(in_ids).cuda(), buf, 0, Hkv, D, BS, NB,
                               pkv.PKV_BF16, staging)
    torch.cuda.synchronize()
    ek, ev = C.swap_in(kcs, vcs, in_ids, expect)
    for layer in range(L):
        np.testing.assert_array_equal(to_bits(kd[layer]), ek[layer])
        np.testing.assert_array_equal(to_bits(vd[layer]), ev[layer])
    assert pkv.pkv_get_device_status() == 0


def test_staged_swap_rejects_bad_buffers_and_zeroes_bad_ids(cuda_device):
    rng = np.random.default_rng(91)
    NB, Hkv, BS, D = 8, 2, 16, 64
    kcs, vcs, kd, vd, kp, vp = setup(rng, 1, NB, Hkv, BS, D, synth.F16)
    tile = Hkv * BS * D * 2
    ids = torch.tensor([1, 2], dtype=torch.int32, device="cuda")
    buf = torch.empty((1, 2, 2, Hkv, BS, D), dtype=torch.int16).pin_memory()
    # staging smaller than two tiles (one per half)
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.pkv_swap_blocks_staged(kp, vp, ids, buf, 1, Hkv, D, BS, NB, pkv.PKV_F16,
                                   torch.empty(2 * tile - 16, dtype=torch.uint8, device="cuda"))
    assert e.value.code == pkv._binding.PKV_ERR_WORKSPACE
    # staging in host memory: refused by the binding
    with pytest.raises(ValueError):
        pkv.pkv_swap_blocks_staged(kp, vp, ids, buf, 1, Hkv, D, BS, NB, pkv.PKV_F16,
                                   torch.empty(4 * tile, dtype=torch.uint8))
    staging = torch.empty(4 * tile, dtype=torch.uint8, device="cuda")
    # host buffer pageable, or too small
    for bad in (torch.empty((1, 2, 2, Hkv, BS, D), dtype=torch.int16),
                torch.empty((1, 2, 1, Hkv, BS, D), dtype=torch.int16).pin_memory()):
        with pytest.raises(pkv.PagedKVError) as e:
            pkv.pkv_swap_blocks_staged(kp, vp, ids, bad, 1, Hkv, D, BS, NB, pkv.PKV_F16,
                                       staging)
        assert e.value.code == pkv._binding.PKV_ERR_INVALID_ARG
    # an out-of-pool id: its tiles are zero in the host buffer, the others exact
    buf3 = torch.full((1, 2, 3, Hkv, BS, D), 7, dtype=torch.int16).pin_memory()
    pkv.pkv_get_device_status(clear=True)
    pkv.pkv_swap_blocks_staged(kp, vp, torch.tensor([2, NB + 5, 4], dtype=torch.int32,
                                                    device="cuda"),
                               buf3, 1, Hkv, D, BS, NB, pkv.PKV_F16, staging)
    assert pkv.pkv_get_device_status(clear=True) & pkv._binding.STATUS_BAD_PAIR
    b = buf3.numpy().view(np.uint16)
    np.testing.assert_array_equal(b[0, 0, 0], kcs[0][2])
    np.testing.assert_array_equal(b[0, 1, 2], vcs[0][4])
    assert (b[0, :, 1] == 0).all()


def test_staged_swap_replays_in_a_cuda_graph(cuda_device):
    """The staged swap's copies run on a stream of the library's, joined to the caller's by
    events: recorded into a CUDA graph on the caller's stream, a replay gives the oracle's
    host buffer (the copy stream is part of the graph)."""
    rng = np.random.default_rng(92)
    L, NB, Hkv, BS, D = 2, 24, 4, 16, 128
    kcs, vcs, kd, vd, kp, vp = setup(rng, L, NB, Hkv, BS, D, synth.BF16)
    ids = np.array(rng.choice(NB, size=9, replace=False), np.int32)
    ids_d = torch.from_numpy(ids).cuda()
    tile = Hkv * BS * D * 2
    staging = torch.empty(4 * tile, dtype=torch.uint8, device="cuda")   # 2 tiles per half
    buf = torch.zeros((L, 2, 9, Hkv, BS, D), dtype=torch.int16).pin_memory()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):   # eager first call: creates the library's copy stream
        pkv.pkv_swap_blocks_staged(kp, vp, ids_d, buf, 1, Hkv, D, BS, NB, pkv.PKV_BF16, staging,
                                   stream=side)
    side.synchronize()
    buf.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        pkv.pkv_swap_blocks_staged(kp, vp, ids_d, buf, 1, Hkv, D, BS, NB, pkv.PKV_BF16, staging,
                                   stream=side)
    torch.cuda.synchronize()
    assert (buf.numpy() == 0).all()          # recording moved nothing
    g.replay()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(buf.numpy().view(np.uint16), C.swap_out(kcs, vcs, ids))
    del g
    assert pkv.pkv_get_device_status() == 0
