"""The allocation-free decode entry point, for callers that may not call cudaMalloc
(plugins whose host framework owns all device memory, serving loops that give all
HBM to the KV pool, latency-critical code where an allocation may synchronise the
device). It keeps its partition scratch in a fixed array inside the library.

Called through the C-ABI (ctypes, raw pointers) and compared, twice in a row, with
the workspace entry point on the same inputs and element by element with the fp64
oracle (one softmax per sequence and query head over the gathered pages), within the
attention tolerance used by the other GPU tests (4e-3 + 1e-2*|ref|). Self-contained
so that it passes alone in a fresh process as well as after every other test."""
import ctypes
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from paged_kv_cache_320_b200 import _binding as B

pytestmark = pytest.mark.gpu


def make_inputs(seed=70):
    """bf16 GQA case whose contexts span several partitions, so the scratch is used."""
    rng = np.random.default_rng(seed)
    Bn, Hq, Hkv, D, BS = 12, 16, 4, 128, 16
    lens = rng.integers(1, 900, size=Bn).astype(np.int32)
    lens[0], lens[1] = 1, 897
    nblk = [-(-int(n) // BS) for n in lens]
    NB = sum(nblk) + 7
    MB = 64
    perm = rng.permutation(NB).astype(np.int32)
    bt = np.full((Bn, MB), -1, np.int32)
    off = 0
    for s in range(Bn):
        bt[s, :nblk[s]] = perm[off:off + nblk[s]]
        off += nblk[s]
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    q = torch.randn(Bn, Hq, D, generator=g, device=dev).to(torch.bfloat16)
    kc = torch.randn(NB, Hkv, BS, D, generator=g, device=dev).to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, BS, D, generator=g, device=dev).to(torch.bfloat16)
    return dict(q=q, kc=kc, vc=vc, bt=torch.from_numpy(bt).to(dev),
                lens=torch.from_numpy(lens).to(dev), Bn=Bn, Hq=Hq, Hkv=Hkv, D=D, BS=BS, NB=NB,
                MB=MB, max_len=MB * BS, scale=1.0 / math.sqrt(D))


def call_noalloc(L, x, out, partition):
    return L.pkv_paged_attention_decode_noalloc(
        out.data_ptr(), x["q"].data_ptr(), x["kc"].data_ptr(), x["vc"].data_ptr(),
        x["bt"].data_ptr(), x["lens"].data_ptr(), x["Bn"], x["Hq"], x["Hkv"], x["D"], x["BS"],
        x["MB"], x["NB"], x["max_len"], x["scale"], B.PKV_BF16, partition,
        torch.cuda.current_stream().cuda_stream)


def test_noalloc_decode_matches_workspace_decode_twice(cuda_device):
    L = B.lib()
    x = make_inputs()
    partition = 64                          # 16 partitions at most: the reduce kernel runs
    need = ctypes.c_size_t()
    assert L.pkv_decode_workspace_size(x["Bn"], x["Hq"], x["Hkv"], x["D"], x["BS"], x["max_len"],
                                       partition, ctypes.byref(need)) == 0
    assert 0 < need.value <= (16 << 20)
    ws = torch.empty(need.value, dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(x["q"])
    rc = L.pkv_paged_attention_decode(
        ref.data_ptr(), x["q"].data_ptr(), x["kc"].data_ptr(), x["vc"].data_ptr(),
        x["bt"].data_ptr(), x["lens"].data_ptr(), x["Bn"], x["Hq"], x["Hkv"], x["D"], x["BS"],
        x["MB"], x["NB"], x["max_len"], x["scale"], B.PKV_BF16, partition, ws.data_ptr(),
        need.value, torch.cuda.current_stream().cuda_stream)
    assert rc == B.PKV_OK
    torch.cuda.synchronize()
    r = ref.float().cpu().numpy()

    def bits(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    oracle = A.paged_decode_attention(bits(x["q"]), bits(x["kc"]), bits(x["vc"]),
                                      x["bt"].cpu().numpy(), x["lens"].cpu().numpy(), x["scale"],
                                      A.BF16)
    for call in range(2):
        out = torch.full_like(x["q"], float("nan"))
        assert call_noalloc(L, x, out, partition) == B.PKV_OK
        torch.cuda.synchronize()
        o = out.float().cpu().numpy()
        err = np.abs(o - r)
        assert np.all(err <= 4e-3 + 1e-2 * np.abs(r)), (call, float(err.max()))
        got = A.bits_to_f64(bits(out), A.BF16)
        err_o = np.abs(got - oracle)
        assert np.all(err_o <= 4e-3 + 1e-2 * np.abs(oracle)), (call, float(err_o.max()))
    st = ctypes.c_uint32(1)
    assert L.pkv_get_device_status(ctypes.byref(st), 1, None) == B.PKV_OK
    assert st.value == 0


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    L = B.lib()
    x = make_inputs(71)
    # 4096 sequences x 16 heads x 16 partitions of fp32 rows is far past the array
    big = 4096
    out = torch.empty_like(x["q"])
    rc = L.pkv_paged_attention_decode_noalloc(
        out.data_ptr(), x["q"].data_ptr(), x["kc"].data_ptr(), x["vc"].data_ptr(),
        x["bt"].data_ptr(), x["lens"].data_ptr(), big, x["Hq"], x["Hkv"], x["D"], x["BS"],
        x["MB"], x["NB"], x["max_len"], x["scale"], B.PKV_BF16, 64,
        torch.cuda.current_stream().cuda_stream)
    assert rc == B.PKV_ERR_WORKSPACE
