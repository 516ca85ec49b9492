"""Argument checks of the Python binding on CUDA tensors: element types, rows and devices
the C declarations require. Every case raises before the library is called, so no kernel
is launched with a bad argument."""
import pytest
import torch

import paged_kv_cache_320_b200 as pkv

pytestmark = pytest.mark.gpu


def case(nseq=3, Hq=8, Hkv=2, D=64, NB=16, BS=16, MB=4, dtype=torch.float16):
    dev = torch.device("cuda", 0)
    q = torch.zeros(nseq, Hq, D, dtype=dtype, device=dev)
    kc = torch.zeros(NB, Hkv, BS, D, dtype=dtype, device=dev)
    kn = torch.zeros(nseq, Hkv, D, dtype=dtype, device=dev)
    bt = torch.zeros(nseq, MB, dtype=torch.int32, device=dev)
    lens = torch.ones(nseq, dtype=torch.int32, device=dev)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=dev)
    return q, kc, kn, bt, lens, ws


def test_decode_rejects_wrong_index_types_rows_and_devices(cuda_device):
    q, kc, kn, bt, lens, ws = case()
    out = torch.empty_like(q)
    pkv.pkv_get_device_status(clear=True)
    with pytest.raises(TypeError, match="context_lens"):
        pkv.pkv_paged_attention_decode(out, q, kc, kc, bt, lens.long(), 64, workspace=ws)
    with pytest.raises(TypeError, match="block_tables"):
        pkv.pkv_paged_attention_decode(out, q, kc, kc, bt.long(), lens, 64, workspace=ws)
    with pytest.raises(ValueError, match="block_tables must be"):
        pkv.pkv_paged_attention_decode(out, q, kc, kc, bt[:2], lens, 64, workspace=ws)
    with pytest.raises(ValueError, match="context_lens holds 2"):
        pkv.pkv_paged_attention_decode(out, q, kc, kc, bt, lens[:2], 64, workspace=ws)
    with pytest.raises(TypeError, match="k_cache"):
        pkv.pkv_paged_attention_decode(out, q, kc.bfloat16(), kc.bfloat16(), bt, lens, 64,
                                       workspace=ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.pkv_paged_attention_decode(out, q, kc, kc, bt, lens.cpu(), 64, workspace=ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.pkv_paged_attention_decode(out, q, kc, kc, bt, lens, 64, workspace=ws.cpu())
    with pytest.raises(TypeError, match="k_new"):
        pkv.pkv_paged_decode_step(out, q, kn.bfloat16(), kn.bfloat16(), kc, kc, bt, lens, 64, ws)
    assert pkv.pkv_get_device_status() == 0


def test_cache_ops_and_device_append_reject_wrong_types(cuda_device):
    q, kc, kn, bt, lens, ws = case()
    with pytest.raises(TypeError, match="slot_mapping"):
        pkv.pkv_reshape_and_cache(kn, kn, kc, kc, lens)                 # int32, not int64
    with pytest.raises(ValueError, match="slot_mapping holds 2"):
        pkv.pkv_reshape_and_cache(kn, kn, kc, kc,
                                  torch.zeros(2, dtype=torch.int64, device=kc.device))
    fl = torch.arange(8, 16, dtype=torch.int32, device=kc.device)
    used = torch.zeros(1, dtype=torch.int32, device=kc.device)
    with pytest.raises(TypeError, match="free_blocks"):
        pkv.pkv_device_append(bt, lens, fl.long(), used, 16, 64, 16)
    with pytest.raises(TypeError, match="slots_out"):
        pkv.pkv_device_append(bt, lens, fl, used, 16, 64, 16, slots_out=lens.clone())
    ptr = torch.tensor([kc.data_ptr()], dtype=torch.int64, device=kc.device)
    with pytest.raises(TypeError, match="block_pairs"):
        pkv.pkv_copy_blocks(ptr, ptr, torch.zeros(1, 2, dtype=torch.int64, device=kc.device),
                            2, 64, 16, 16, pkv.PKV_F16)
    with pytest.raises(ValueError, match="v_cache_ptrs holds 1"):
        pkv.pkv_copy_blocks(torch.cat([ptr, ptr]), ptr,
                            torch.zeros(1, 2, dtype=torch.int32, device=kc.device),
                            2, 64, 16, 16, pkv.PKV_F16)
    assert torch.equal(used, torch.zeros_like(used))
    assert pkv.pkv_get_device_status() == 0
