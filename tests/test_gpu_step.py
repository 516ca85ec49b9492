"""A whole parallel-sampling decode step driven by the block manager (GPU).

16 prompts, each a parent whose last block is partly filled, forked into 8
samples; every sample appends one token, so the first 7 writers of each shared
block copy it (112 copy-on-write pairs) and the 8th writes in place. The GPU side
uses the C++ block manager -> copy_blocks -> reshape_and_cache -> decode; the
oracle side uses its own block-manager model and CPU routines. Block tables,
slots and pairs must agree exactly, the caches bit for bit, attention within the
tolerance."""
import numpy as np
import pytest
import torch

import paged_kv_cache_320_b200 as pkv
from oracle import attention as A
from oracle import block_manager as BM
from oracle import cache_ops as C
from paged_kv_cache_320_b200 import BlockManager, synth
from tests.gpu_util import assert_close, to_bits, to_dev

pytestmark = pytest.mark.gpu


def drive(mgr_append, mgr_fork, step, samples):
    """Same op sequence on either manager: parents, forks, then one token per sample."""
    slots, pairs = [], []
    B = len(step.parent_lens) * samples
    for p, n in enumerate(step.parent_lens):
        parent = p * samples
        st, _, cows = mgr_append(parent, int(n))
        assert st == 0 and len(cows) == 0
        for k in range(1, samples):
            assert mgr_fork(parent, parent + k) == 0
    for s in range(B):
        st, sl, cows = mgr_append(s, 1)
        assert st == 0
        slots.append(int(sl[0]))
        pairs += [list(map(int, c)) for c in cows]
    return np.array(slots, np.int64), np.array(pairs, np.int32).reshape(-1, 2)


def test_copy_on_write_step_matches_oracle(cuda_device):
    step = synth.make_cow_step(num_layers=2)
    sp = step.spec
    samples = sp.samples
    B = len(step.parent_lens) * samples
    dt = sp.dtype

    # oracle side: model of the block manager, then CPU cache ops and attention
    model = BM.BlockManagerModel(step.num_blocks, sp.block_size, step.max_blocks_per_seq,
                                 step.initial_order)
    m_slots, m_pairs = drive(lambda s, n: model.append(s, n), model.fork, step, samples)
    m_bt = np.array([model.block_table(s)[0] for s in range(B)], np.int32)
    m_lens = np.array([model.block_table(s)[1] for s in range(B)], np.int32)

    # GPU side: the library's block manager
    mgr = BlockManager(step.num_blocks, sp.block_size, step.max_blocks_per_seq,
                       step.initial_order)
    g_slots, g_pairs = drive(mgr.pkv_seq_append, mgr.pkv_seq_fork, step, samples)
    st, g_bt, g_lens = mgr.pkv_block_tables(np.arange(B))
    assert st == 0
    np.testing.assert_array_equal(g_slots, m_slots)
    np.testing.assert_array_equal(g_pairs, m_pairs)
    np.testing.assert_array_equal(g_bt, m_bt)
    np.testing.assert_array_equal(g_lens, m_lens)
    assert g_pairs.shape == (len(step.parent_lens) * (samples - 1), 2)

    # pools: rows never written by a parent carry the NaN canary (from the model's tables)
    L = step.num_layers
    kc = step.k_cache.copy()
    vc = step.v_cache.copy()
    written = np.zeros((step.num_blocks, sp.block_size), bool)
    # parents' history rows, from a fresh model holding only the parents
    pm = BM.BlockManagerModel(step.num_blocks, sp.block_size, step.max_blocks_per_seq,
                              step.initial_order)
    for p, n in enumerate(step.parent_lens):
        pm.append(p, int(n))
        row, _ = pm.block_table(p)
        for t in range(int(n)):
            written[row[t // sp.block_size], t % sp.block_size] = True
    for layer in range(L):
        kc[layer].transpose(0, 2, 1, 3)[~written] = synth.CANARY[dt]
        vc[layer].transpose(0, 2, 1, 3)[~written] = synth.CANARY[dt]

    ek, ev = C.copy_blocks(list(kc), list(vc), m_pairs)
    for layer in range(L):
        ek[layer], ev[layer] = C.reshape_and_cache(step.k_new, step.v_new, ek[layer], ev[layer],
                                                   m_slots)
    ref = A.paged_decode_attention(step.q, ek[0], ev[0], m_bt, m_lens, 1 / np.sqrt(sp.head_dim),
                                   dt)

    kd = [to_dev(kc[layer], dt) for layer in range(L)]
    vd = [to_dev(vc[layer], dt) for layer in range(L)]
    kp = torch.tensor([t.data_ptr() for t in kd], dtype=torch.int64, device="cuda")
    vp = torch.tensor([t.data_ptr() for t in vd], dtype=torch.int64, device="cuda")
    pkv.pkv_copy_blocks(kp, vp, torch.from_numpy(g_pairs).cuda(), sp.num_kv_heads, sp.head_dim,
                        sp.block_size, step.num_blocks, pkv.PKV_BF16)
    sl = torch.from_numpy(g_slots).cuda()
    kn, vn = to_dev(step.k_new, dt), to_dev(step.v_new, dt)
    for layer in range(L):
        pkv.pkv_reshape_and_cache(kn, vn, kd[layer], vd[layer], sl)
    q = to_dev(step.q, dt)
    out = torch.empty_like(q)
    pkv.pkv_paged_attention_decode(out, q, kd[0], vd[0], torch.from_numpy(g_bt).cuda(),
                                   torch.from_numpy(g_lens).cuda(), sp.max_len,
                                   scale=1 / np.sqrt(sp.head_dim))
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_status() == 0
    for layer in range(L):
        np.testing.assert_array_equal(to_bits(kd[layer]), ek[layer])
        np.testing.assert_array_equal(to_bits(vd[layer]), ev[layer])
    assert_close(to_bits(out), ref, dt, "copy-on-write step")
