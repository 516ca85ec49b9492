"""Pins of the cache-write and block-copy oracles (CPU only): read-back of every
written slot equals the new token, every other byte is unchanged (NaN canary),
padding slots are skipped, copied pages equal their sources in every layer."""
import numpy as np
import pytest

from oracle import cache_ops, c_oracle
from paged_kv_cache_320_b200 import synth


@pytest.mark.parametrize("dtype", [synth.F16, synth.BF16])
def test_reshape_and_cache_read_back_and_canary(dtype):
    rng = np.random.default_rng(30)
    NB, Hkv, bs, d, T = 12, 3, 8, 16, 20
    kc = np.full((NB, Hkv, bs, d), synth.CANARY[dtype], np.uint16)
    vc = kc.copy()
    kn = synth.round_to_bits(rng.standard_normal((T, Hkv, d), dtype=np.float32), dtype)
    vn = synth.round_to_bits(rng.standard_normal((T, Hkv, d), dtype=np.float32), dtype)
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
    slots[[3, 11]] = -1                                   # padding tokens
    k2, v2 = cache_ops.reshape_and_cache(kn, vn, kc, vc, slots)
    k3, v3 = c_oracle.reshape_and_cache(kn, vn, kc, vc, slots)
    np.testing.assert_array_equal(k2, k3)
    np.testing.assert_array_equal(v2, v3)
    touched = np.zeros((NB, bs), bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        np.testing.assert_array_equal(k2[s // bs, :, s % bs], kn[t])
        np.testing.assert_array_equal(v2[s // bs, :, s % bs], vn[t])
        touched[s // bs, s % bs] = True
    untouched = ~touched
    assert (k2.transpose(0, 2, 1, 3)[untouched] == synth.CANARY[dtype]).all()
    assert (v2.transpose(0, 2, 1, 3)[untouched] == synth.CANARY[dtype]).all()
    # inputs are not modified
    assert (kc == synth.CANARY[dtype]).all()


def test_copy_blocks_every_layer_and_nothing_else():
    rng = np.random.default_rng(31)
    L, NB, Hkv, bs, d = 3, 10, 2, 4, 8
    kcs = [rng.integers(0, 1 << 16, (NB, Hkv, bs, d), dtype=np.uint16) for _ in range(L)]
    vcs = [rng.integers(0, 1 << 16, (NB, Hkv, bs, d), dtype=np.uint16) for _ in range(L)]
    pairs = np.array([[0, 5], [2, 7], [2, 9]], dtype=np.int32)
    k2, v2 = cache_ops.copy_blocks(kcs, vcs, pairs)
    for layer in range(L):
        for src, dst in pairs:
            assert k2[layer][dst].tobytes() == kcs[layer][src].tobytes()
            assert v2[layer][dst].tobytes() == vcs[layer][src].tobytes()
        others = [b for b in range(NB) if b not in pairs[:, 1]]
        np.testing.assert_array_equal(k2[layer][others], kcs[layer][others])
        np.testing.assert_array_equal(v2[layer][others], vcs[layer][others])


def test_swap_round_trip_is_a_block_copy():
    """swap_out then swap_in to other ids equals copy_blocks of the same pairs; the
    buffer holds each layer's pages in list order; other blocks are untouched."""
    rng = np.random.default_rng(32)
    L, NB, Hkv, bs, d = 2, 12, 2, 8, 16
    kcs = [rng.integers(0, 1 << 16, (NB, Hkv, bs, d), dtype=np.uint16) for _ in range(L)]
    vcs = [rng.integers(0, 1 << 16, (NB, Hkv, bs, d), dtype=np.uint16) for _ in range(L)]
    src = np.array([3, 7, 0], np.int32)
    dst = np.array([9, 1, 11], np.int32)
    buf = cache_ops.swap_out(kcs, vcs, src)
    assert buf.shape == (L, 2, 3, Hkv, bs, d)
    for layer in range(L):
        for i, b in enumerate(src):
            assert buf[layer, 0, i].tobytes() == kcs[layer][b].tobytes()
            assert buf[layer, 1, i].tobytes() == vcs[layer][b].tobytes()
    k2, v2 = cache_ops.swap_in(kcs, vcs, dst, buf)
    k3, v3 = cache_ops.copy_blocks(kcs, vcs, np.stack([src, dst], 1))
    for layer in range(L):
        np.testing.assert_array_equal(k2[layer], k3[layer])
        np.testing.assert_array_equal(v2[layer], v3[layer])
