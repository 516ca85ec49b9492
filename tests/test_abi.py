"""The C-ABI library loads and exports every entry point its header declares, and
host-side argument checks reject bad sizes before any device work (CPU only)."""
import ctypes
import os
import re

import pytest

import paged_kv_cache_320_b200 as pkv
from paged_kv_cache_320_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for must in ("pkv_paged_attention_decode", "pkv_reshape_and_cache", "pkv_copy_blocks",
                 "pkv_alloc_create", "pkv_seq_append", "pkv_seq_fork", "pkv_seq_free",
                 "pkv_block_tables", "pkv_stats"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(B.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


@pytest.mark.parametrize("args", [
    (4, 8, 8, 96, 16, 128, 0),       # head_dim
    (4, 8, 8, 64, 12, 128, 0),       # block_size
    (4, 8, 3, 64, 16, 128, 0),       # Hq % Hkv
    (4, 64, 2, 64, 16, 128, 0),      # group > 16
    (4, 8, 8, 64, 16, 128, 100),     # partition not a multiple of 64
    (4, 8, 8, 64, 8, 128, 4096),     # partition > 256 blocks
    (-1, 8, 8, 64, 16, 128, 0),      # negative batch
])
def test_decode_size_checks(args):
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.pkv_decode_workspace_size(*args)
    assert e.value.code == B.PKV_ERR_INVALID_ARG


def test_workspace_size_formula():
    # single partition -> no workspace
    assert pkv.pkv_decode_workspace_size(4, 8, 8, 64, 16, 100, 128) == 0
    # B=2, Hq=4, D=64, max_len=300, P=128 -> 3 partitions;
    # scheduler header + first item per sequence + (max, sum) rows + output rows
    rows = 2 * 4 * 3
    expect = 256 + 256 + ((rows * 8 + 255) // 256) * 256 + rows * 64 * 4
    assert pkv.pkv_decode_workspace_size(2, 4, 2, 64, 16, 300, 128) == expect


def test_auto_partition_choices():
    assert pkv.pkv_decode_partition_size(256, 32, 8, 128, 16, 8192) == 512     # G = 4
    assert pkv.pkv_decode_partition_size(8, 64, 8, 128, 16, 131072) == 2048    # G = 8
    assert pkv.pkv_decode_partition_size(8, 64, 8, 128, 8, 131072) == 2048     # 256 blocks of 8
    assert pkv.pkv_decode_partition_size(8, 64, 8, 128, 16, 131072, 4096) == 4096  # 256 of 16
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_decode_partition_size(8, 64, 8, 128, 8, 131072, 4096)            # 512 of 8
    assert pkv.pkv_decode_partition_size(4, 8, 8, 64, 16, 128) == 64          # tiny batch
    # every context one item: at most 64 sequences (longest-first order), >= 1024 items
    assert pkv.pkv_decode_partition_size(64, 32, 32, 128, 16, 2100) == 2112
    assert pkv.pkv_decode_partition_size(64, 32, 32, 128, 16, 4097) == 512    # > 256 blocks
    assert pkv.pkv_decode_partition_size(65, 32, 32, 128, 16, 2100) == 512    # > 64 sequences
    assert pkv.pkv_decode_partition_size(31, 32, 32, 128, 16, 2100) == 512    # < 1024 items


def test_pair_count_must_fit_an_int():
    # 2^27 sequences x 16 query heads = 2^31 (sequence, head) pairs: refused on the host
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_decode_partition_size(1 << 27, 16, 1, 64, 16, 16)
    assert pkv.pkv_decode_partition_size((1 << 27) - 1, 16, 1, 64, 16, 16) == 2048


def test_shared_prefix_auto_partition_choices():
    f = pkv.pkv_decode_shared_prefix_partition_size
    assert f(128, 32, 8, 128, 16, 1300) == 2048        # G = 4: prefix and suffixes in one item
    assert f(8, 64, 8, 128, 16, 131072) == 2048        # G = 8
    assert f(128, 32, 8, 128, 8, 1300) == 2048         # 256 blocks of 8
    assert f(4, 8, 8, 64, 16, 128) == 64               # tiny batch: halved like the plain path
    assert f(128, 32, 8, 128, 16, 1300, 256) == 256    # an explicit size is kept
    with pytest.raises(pkv.PagedKVError):
        f(8, 64, 8, 128, 8, 131072, 4096)               # 512 blocks of 8
    assert pkv.pkv_decode_shared_prefix_workspace_size(128, 32, 8, 128, 16, 1300) == \
        pkv.pkv_decode_shared_prefix_workspace_size(128, 32, 8, 128, 16, 1300, 2048)


def test_decode_rejects_bad_args_without_a_device():
    L = B.lib()
    # head_dim 96 -> rejected before any CUDA call
    rc = L.pkv_paged_attention_decode(None, None, None, None, None, None, 4, 8, 8, 96, 16, 8, 64,
                                      100, 0.1, 0, 0, None, 0, None)
    assert rc == B.PKV_ERR_INVALID_ARG
    # max_context_len above max_blocks_per_seq * block_size
    rc = L.pkv_paged_attention_decode(None, None, None, None, None, None, 4, 8, 8, 64, 16, 8, 64,
                                      129, 0.1, 0, 0, None, 0, None)
    assert rc == B.PKV_ERR_INVALID_ARG
    # bad dtype / non-finite scale
    rc = L.pkv_paged_attention_decode(None, None, None, None, None, None, 4, 8, 8, 64, 16, 8, 64,
                                      100, 0.1, 7, 0, None, 0, None)
    assert rc == B.PKV_ERR_INVALID_ARG
    rc = L.pkv_paged_attention_decode(None, None, None, None, None, None, 4, 8, 8, 64, 16, 8, 64,
                                      100, float("inf"), 0, 0, None, 0, None)
    assert rc == B.PKV_ERR_INVALID_ARG
    # zero sequences: nothing to do
    rc = L.pkv_paged_attention_decode(None, None, None, None, None, None, 0, 8, 8, 64, 16, 8, 64,
                                      100, 0.1, 0, 0, None, 0, None)
    assert rc == B.PKV_OK
    # null pointers with work to do
    rc = L.pkv_paged_attention_decode(None, None, None, None, None, None, 4, 8, 8, 64, 16, 8, 64,
                                      100, 0.1, 0, 0, None, 0, None)
    assert rc == B.PKV_ERR_INVALID_ARG


def test_cache_op_checks_without_a_device():
    L = B.lib()
    assert L.pkv_reshape_and_cache(None, None, None, None, None, 0, 8, 64, 16, 64, 0, None) == B.PKV_OK
    assert L.pkv_reshape_and_cache(None, None, None, None, None, 4, 8, 64, 16, 64, 0, None) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_reshape_and_cache(None, None, None, None, None, 4, 8, 80, 16, 64, 0, None) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_copy_blocks(None, None, 1, None, 0, 8, 64, 16, 64, 0, None) == B.PKV_OK
    assert L.pkv_copy_blocks(None, None, 1, None, 3, 8, 64, 16, 64, 0, None) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_copy_blocks(None, None, 0, None, 3, 8, 64, 16, 64, 0, None) == B.PKV_ERR_INVALID_ARG


def test_staged_swap_checks_without_a_device():
    L = B.lib()
    args = (None, None, 1, None)
    # nothing to move; bad head_dim; missing pointers (all before any CUDA call)
    assert L.pkv_swap_blocks_staged(*args, 0, None, 0, 1, 8, 128, 16, 64, 0, None, 0,
                                    None) == B.PKV_OK
    assert L.pkv_swap_blocks_staged(*args, 4, None, 0, 1, 8, 96, 16, 64, 0, None, 0,
                                    None) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_swap_blocks_staged(*args, 4, None, 0, 1, 8, 128, 16, 64, 0, None, 0,
                                    None) == B.PKV_ERR_INVALID_ARG


def test_status_strings():
    L = B.lib()
    for code in range(-10, 1):
        assert L.pkv_status_string(code) != b"unknown status", code


def test_step_and_shared_prefix_checks_without_a_device():
    """The device-step and shared-prefix entry points reject bad arguments on the host,
    before any CUDA call (no GPU here)."""
    L = B.lib()
    # decode step: bad head_dim, missing workspace, zero sequences
    args = [None] * 8
    assert L.pkv_paged_decode_step(*args, 4, 8, 8, 96, 16, 8, 64, 100, 0.1, 0, 0, None, 0,
                                   None) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_paged_decode_step(*args, 0, 8, 8, 64, 16, 8, 64, 100, 0.1, 0, 0, None, 0,
                                   None) == B.PKV_OK
    assert L.pkv_paged_decode_step(*args, 4, 8, 8, 64, 16, 8, 64, 100, 0.1, 0, 0, None, 0,
                                   None) == B.PKV_ERR_INVALID_ARG        # null tensors
    # workspace size query: at least the 256-byte header, more with several partitions
    one, many = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert L.pkv_decode_step_workspace_size(4, 8, 2, 64, 16, 64, 64, ctypes.byref(one)) == 0
    assert L.pkv_decode_step_workspace_size(4, 8, 2, 64, 16, 1024, 64, ctypes.byref(many)) == 0
    assert one.value == 256 and many.value > one.value
    # merge alone: nothing to merge without partitions or sequences; bad dtype; no workspace
    assert L.pkv_paged_attention_merge(None, None, 0, 8, 2, 64, 16, 1000, 64, 0, None, 0,
                                       None) == B.PKV_OK
    assert L.pkv_paged_attention_merge(None, None, 4, 8, 2, 64, 16, 64, 64, 0, None, 0,
                                       None) == B.PKV_OK
    assert L.pkv_paged_attention_merge(None, None, 4, 8, 2, 64, 16, 1000, 64, 3, None, 0,
                                       None) == B.PKV_ERR_INVALID_ARG
    buf = ctypes.create_string_buffer(64)
    assert L.pkv_paged_attention_merge(ctypes.addressof(buf), ctypes.addressof(buf), 4, 8, 2, 64,
                                       16, 1000, 64, 0, None, 0, None) == B.PKV_ERR_WORKSPACE
    # device append: negative sizes, missing cursor
    assert L.pkv_device_append(None, None, None, 0, None, None, None, 4, 8, 16, 64, 128,
                               None) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_device_append(None, None, None, -1, None, None, None, 4, 8, 16, 64, 128,
                               None) == B.PKV_ERR_INVALID_ARG
    # shared-prefix plan / planned decode: too many groups, zero sequences
    assert L.pkv_shared_prefix_plan(None, None, None, None, 5, 4, 8, 2, 64, 16, 8, 100, 0, None,
                                    0, None) == B.PKV_ERR_INVALID_ARG
    assert L.pkv_shared_prefix_plan(None, None, None, None, 1, 0, 8, 2, 64, 16, 8, 100, 0, None,
                                    0, None) == B.PKV_OK
    assert L.pkv_paged_attention_decode_shared_prefix_planned(
        None, None, None, None, None, None, 4, 8, 2, 64, 16, 8, 64, 100, 0.1, 3, 0, None, 0,
        None) == B.PKV_ERR_INVALID_ARG                                    # dtype 3
    # launch-count query needs the device (SM count) only when there is work
    n = ctypes.c_int(-1)
    assert L.pkv_decode_step_launches(0, 8, 2, 64, 16, 100, 0, ctypes.byref(n)) == 0
    assert n.value == 0
