"""Helpers shared by the GPU parity tests: moving uint16 bit arrays to and from
torch fp16/bf16 tensors, the attention tolerance, and sampled-sequence oracles."""
import numpy as np
import torch

from oracle import attention as A
from oracle import cache_ops as C
from paged_kv_cache_320_b200 import synth

# spec tolerance for attention outputs (bf16/fp16 in, fp32 accumulate)
ATOL = 4e-3
RTOL = 1e-2


def tdtype(dtype):
    return torch.float16 if dtype == synth.F16 else torch.bfloat16


def to_dev(bits, dtype, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)
    return t.view(tdtype(dtype))


def to_bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def assert_close(gpu_bits, ref, dtype, what=""):
    got = A.bits_to_f64(gpu_bits, dtype)
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {bad.sum()} of {bad.size} outside 4e-3 + 1e-2|ref|; first {idx.tolist()} "
            f"got {got[bad][:5]} ref {ref[bad][:5]}; max err {err.max():.3g}")
    return float((err / bound).max())


def sampled_oracle(q_bits, kc_dev, vc_dev, bt, lens, seqs, scale, dtype, k_new_bits=None,
                   v_new_bits=None, slots=None):
    """fp64 oracle outputs for the sequences ``seqs`` from host copies of just their
    pages (read from the device BEFORE any GPU write), with this step's cache write
    applied by the oracle's own cache-write routine. Returns [len(seqs), Hq, d]."""
    outs = []
    bs = kc_dev.shape[2]
    for s in seqs:
        n = int(lens[s])
        nblk = -(-n // bs)
        pages = bt[s, :nblk].astype(np.int64)
        kc = to_bits(kc_dev[torch.from_numpy(pages).to(kc_dev.device)])
        vc = to_bits(vc_dev[torch.from_numpy(pages).to(vc_dev.device)])
        bt_local = np.full((1, max(nblk, 1)), -1, np.int32)
        bt_local[0, :nblk] = np.arange(nblk)
        if slots is not None and slots[s] >= 0:
            slot = int(slots[s])
            page = int(np.nonzero(pages == slot // bs)[0][0])
            local_slot = np.array([page * bs + slot % bs], dtype=np.int64)
            kc, vc = C.reshape_and_cache(k_new_bits[s:s + 1], v_new_bits[s:s + 1], kc, vc,
                                         local_slot)
        o = A.paged_decode_attention(q_bits[s:s + 1], kc, vc, bt_local,
                                     np.array([n], np.int32), scale, dtype)
        outs.append(o[0])
    return np.stack(outs)
