"""Host checks of the seeded workload generator (CPU only)."""
import numpy as np
import pytest

from paged_kv_cache_320_b200 import synth


def test_same_seed_same_workload():
    a = synth.make_workload("tiny")
    b = synth.make_workload("tiny")
    for f in ("context_lens", "perm", "block_tables", "slot_mapping", "q", "k_cache", "v_cache", "k_new", "v_new"):
        np.testing.assert_array_equal(getattr(a, f), getattr(b, f))


def test_tiny_shapes_and_canary():
    wl = synth.make_workload("tiny")
    sp = wl.spec
    assert list(wl.context_lens) == [7, 16, 33, 100]
    assert wl.num_blocks == 64
    assert wl.q.shape == (1, 4, 8, 64)
    assert wl.k_cache.shape == (1, 64, 8, 16, 64)
    used = wl.block_tables[wl.block_tables >= 0]
    assert len(set(used.tolist())) == len(used) == 1 + 1 + 3 + 7
    # the slot of this step's token still holds the canary; history holds values
    for s, n in enumerate(wl.context_lens):
        slot = wl.slot_mapping[s]
        assert (wl.k_cache[0, slot // 16, :, slot % 16] == synth.CANARY[sp.dtype]).all()
        for t in range(n - 1):
            b = wl.block_tables[s, t // 16]
            assert not (wl.k_cache[0, b, :, t % 16] == synth.CANARY[sp.dtype]).any()
    unused = np.setdiff1d(np.arange(64), used)
    assert (wl.k_cache[0, unused] == synth.CANARY[sp.dtype]).all()


@pytest.mark.parametrize("name,lo,hi", [("llama7b_mha", 16, 2048), ("llama3_8b_gqa", 8, 8192),
                                        ("long_context", 32768, 131072)])
def test_length_ranges_and_pool(name, lo, hi):
    wl = synth.make_workload(name, values_on="none")
    assert wl.context_lens.min() >= lo and wl.context_lens.max() <= hi
    need = sum(-(-int(n) // wl.spec.block_size) for n in wl.context_lens)
    assert wl.num_blocks == int(np.ceil(1.2 * need))
    assert wl.max_blocks_per_seq * wl.spec.block_size >= hi


def test_shared_prefix_tables_share_prefix_blocks():
    wl = synth.make_workload("shared_prefix", values_on="none")
    bt = wl.block_tables
    for p in range(16):
        rows = bt[p * 8:(p + 1) * 8, :64]
        assert (rows == rows[0]).all()
    assert ((wl.context_lens >= 1025) & (wl.context_lens <= 1281)).all()
    private = bt[:, 64:]
    used = private[private >= 0]
    assert len(set(used.tolist())) == len(used)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, np.nan], dtype=np.float32)
    b = synth.round_to_bits(x, synth.BF16)
    assert b[0] == 0x3F80
    assert b[1] == 0x3F80          # tie -> even
    assert b[2] == 0x3F82          # tie -> even (up)
    assert b[3] == 0xC020
    assert b[4] == synth.CANARY[synth.BF16]
