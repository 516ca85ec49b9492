"""Cache write through a slot mapping, and copy-on-write block duplication.

Sources: "vLLM / PagedAttention — 分页 KV Cache 分析", §3.2 (a request that must
change a shared page copies it first, then changes the copy; a new token is
written into its page) and §2.3 (block table maps logical token positions to
physical pages).

Readings:
* Slot ``slot`` is row ``slot % bs`` of physical page ``slot // bs``; a token with
  slot < 0 is padding and is not written.
* ``copy_blocks`` copies every layer's K and V page ``src`` onto ``dst`` for all
  KV heads. All ``dst`` are distinct and no ``dst`` is a ``src`` of the same call,
  so the order of the pairs does not matter.
"""
from __future__ import annotations

import numpy as np


def reshape_and_cache(k_new, v_new, k_cache, v_cache, slot_mapping):
    """Return copies of k_cache / v_cache [NB, Hkv, bs, d] with each new token's
    K/V row [Hkv, d] placed at its slot."""
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    bs = kc.shape[2]
    for t, slot in enumerate(np.asarray(slot_mapping)):
        slot = int(slot)
        if slot < 0:
            continue
        b, r = slot // bs, slot % bs
        for h in range(kc.shape[1]):
            kc[b, h, r, :] = k_new[t, h, :]
            vc[b, h, r, :] = v_new[t, h, :]
    return kc, vc


def copy_blocks(k_caches, v_caches, block_pairs):
    """Return copies of every layer's caches with page dst replaced by page src."""
    out_k = [np.array(c, copy=True) for c in k_caches]
    out_v = [np.array(c, copy=True) for c in v_caches]
    for src, dst in np.asarray(block_pairs).reshape(-1, 2):
        for layer in range(len(out_k)):
            out_k[layer][int(dst)] = k_caches[layer][int(src)]
            out_v[layer][int(dst)] = v_caches[layer][int(src)]
    return out_k, out_v


def swap_out(k_caches, v_caches, block_ids):
    """Host buffer [L][2][n][Hkv, bs, d] holding every layer's K and V page of each listed
    block, in list order ("vLLM/PagedAttention — L3 Cross-Paper Synthesis" §3: a
    preempted request's pages are swapped out whole)."""
    ids = [int(b) for b in np.asarray(block_ids).reshape(-1)]
    L = len(k_caches)
    tile = k_caches[0].shape[1:]
    buf = np.empty((L, 2, len(ids)) + tuple(tile), dtype=k_caches[0].dtype)
    for layer in range(L):
        for i, b in enumerate(ids):
            buf[layer, 0, i] = k_caches[layer][b]
            buf[layer, 1, i] = v_caches[layer][b]
    return buf


def swap_in(k_caches, v_caches, block_ids, buf):
    """Copies of the caches with page block_ids[i] of every layer set from the buffer."""
    out_k = [np.array(c, copy=True) for c in k_caches]
    out_v = [np.array(c, copy=True) for c in v_caches]
    for layer in range(len(out_k)):
        for i, b in enumerate(np.asarray(block_ids).reshape(-1)):
            out_k[layer][int(b)] = buf[layer, 0, i]
            out_v[layer][int(b)] = buf[layer, 1, i]
    return out_k, out_v
