"""Argument checks of the Python binding, on the host: a tensor whose address the library
would dereference must be a CUDA tensor of the declared element type with the rows the C
declaration reads. These cases raise before the library is called, so no GPU is needed
(the dtype and row checks on CUDA tensors are in test_gpu_binding_checks.py)."""
import pytest
import torch

import paged_kv_cache_320_b200 as pkv
from paged_kv_cache_320_b200 import _binding as B


def host_case(nseq=2, Hq=4, Hkv=2, D=64, NB=8, BS=16, MB=4):
    q = torch.zeros(nseq, Hq, D, dtype=torch.float16)
    kc = torch.zeros(NB, Hkv, BS, D, dtype=torch.float16)
    kn = torch.zeros(nseq, Hkv, D, dtype=torch.float16)
    bt = torch.zeros(nseq, MB, dtype=torch.int32)
    lens = torch.ones(nseq, dtype=torch.int32)
    return q, kc, kn, bt, lens


def test_host_tensors_never_reach_the_library():
    q, kc, kn, bt, lens = host_case()
    out = torch.empty_like(q)
    ws = torch.zeros(1024, dtype=torch.uint8)
    i32 = torch.zeros(4, dtype=torch.int32)
    i64 = torch.zeros(2, dtype=torch.int64)
    calls = {
        "decode": lambda: pkv.pkv_paged_attention_decode(out, q, kc, kc, bt, lens, 64),
        "noalloc": lambda: pkv.pkv_paged_attention_decode_noalloc(out, q, kc, kc, bt, lens, 64),
        "shared": lambda: pkv.pkv_paged_attention_decode_shared_prefix(
            out, q, kc, kc, bt, lens, torch.tensor([0, 2], dtype=torch.int32),
            torch.tensor([16], dtype=torch.int32), 64),
        "plan": lambda: pkv.pkv_shared_prefix_plan(
            bt, lens, torch.tensor([0, 2], dtype=torch.int32),
            torch.tensor([16], dtype=torch.int32), 4, 2, 64, 16, 64, ws),
        "planned": lambda: pkv.pkv_paged_attention_decode_shared_prefix_planned(
            out, q, kc, kc, bt, lens, 64, ws),
        "step": lambda: pkv.pkv_paged_decode_step(out, q, kn, kn, kc, kc, bt, lens, 64, ws),
        "append": lambda: pkv.pkv_device_append(bt, lens, i32, i32[:1], 8, 64, 16),
        "reshape": lambda: pkv.pkv_reshape_and_cache(kn, kn, kc, kc, i64),
        "copy": lambda: pkv.pkv_copy_blocks(i64[:1], i64[:1], i32.view(2, 2), 2, 64, 16, 8,
                                            pkv.PKV_F16),
        "swap": lambda: pkv.pkv_swap_blocks(i64[:1], i64[:1], i32[:2], ws, 1, 2, 64, 16, 8,
                                            pkv.PKV_F16),
    }
    for name, call in calls.items():
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()


def test_block_tables_need_two_dims_and_a_row_per_sequence():
    dev = torch.device("cpu")
    lens = torch.ones(3, dtype=torch.int32)
    with pytest.raises(ValueError, match="block_tables must be"):
        B._tables(torch.zeros(12, dtype=torch.int32), lens, 3, dev)        # flat
    with pytest.raises(ValueError, match="block_tables must be"):
        B._tables(torch.zeros(2, 6, dtype=torch.int32), lens, 3, dev)      # a row short


def test_decode_shapes_and_dtype_checked_first():
    q, kc, kn, bt, lens = host_case()
    with pytest.raises(ValueError, match="shape mismatch"):
        pkv.pkv_paged_attention_decode(torch.empty_like(q), q, kc[..., :32], kc[..., :32], bt,
                                       lens, 64)
    q32 = q.float()
    with pytest.raises(TypeError, match="unsupported dtype"):
        pkv.pkv_paged_attention_decode(torch.empty_like(q32), q32, kc, kc, bt, lens, 64)
    with pytest.raises(ValueError, match="k_new must be"):
        pkv.pkv_reshape_and_cache(kn[0], kn[0], kc, kc, torch.zeros(2, dtype=torch.int64))
    with pytest.raises(ValueError, match="block_pairs must be"):
        pkv.pkv_copy_blocks(torch.zeros(1, dtype=torch.int64), torch.zeros(1, dtype=torch.int64),
                            torch.zeros(6, dtype=torch.int32), 2, 64, 16, 8, pkv.PKV_F16)


def test_need_accepts_only_matching_cuda_tensors():
    with pytest.raises(ValueError, match="CUDA tensor"):
        B._need(torch.zeros(2), "x")
    with pytest.raises(ValueError, match="CUDA tensor"):
        B._need([1, 2], "x")
