"""Paged single-query decode attention, written as its plain definition (fp64).

Source: "vLLM / PagedAttention — 分页 KV Cache 分析", §2.2 (the KV cache is cut
into fixed-size pages reached through a per-request block table) and §3.1 (the
attention kernel is changed only in how it reaches non-contiguous KV; the
simplified per-page loop there). Read as: paging changes where the bytes live,
not what attention computes, so the oracle gathers each sequence's pages into a
contiguous K and V and runs ordinary softmax attention over all of them.

Readings where the page's loop is garbled or silent:
* The printed loop normalises the softmax per page and sums the page results;
  its weights would sum to the number of pages. Read instead as ONE softmax per
  (sequence, query head) over all ``len`` tokens — the per-page loop is the
  streaming form of it. It has no scale; the scale is an argument (1/sqrt(d)).
* Tokens at positions >= len (the unfilled tail of the last page) are not part
  of the sequence and are never read.
* GQA (named on "vLLM/PagedAttention — L3 Cross-Paper Synthesis", §2, only as a
  model-level change): query head h reads KV head h // (Hq/Hkv).
* A zero-length context has no defined attention; its output is 0.
"""
from __future__ import annotations

import numpy as np

F16 = 0
BF16 = 1


def bits_to_f64(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Exact upcast of fp16 / bf16 bit patterns (uint16) to float64."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == F16:
        return bits.view(np.float16).astype(np.float64)
    if dtype == BF16:
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def gather_sequence(cache: np.ndarray, block_table_row: np.ndarray, length: int,
                    kv_head: int, dtype: int) -> np.ndarray:
    """Contiguous [length, d] K (or V) of one sequence and one KV head.

    Logical token t lives in physical page block_table_row[t // bs] at row t % bs
    (the block-table mapping of §2.2's diagram)."""
    bs = cache.shape[2]
    t = np.arange(length)
    pages = block_table_row[t // bs]
    return bits_to_f64(cache[pages, kv_head, t % bs, :], dtype)


def softmax_attention(qv: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """One query vector against contiguous K [n, d], V [n, d] (fp64)."""
    x = scale * (K @ qv)
    x = x - x.max()
    p = np.exp(x)
    return (p @ V) / p.sum()


def paged_decode_attention(q, k_cache, v_cache, block_tables, context_lens, scale, dtype,
                           seqs=None):
    """out[s, h, :] for every sequence s (or the listed ``seqs``) and query head h.

    q:            uint16 bits [B, Hq, d]
    k/v_cache:    uint16 bits [NB, Hkv, bs, d]
    block_tables: int32 [B, MB];  context_lens: int32 [B]
    Returns float64 [len(seqs), Hq, d]."""
    B, Hq, d = q.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    seqs = range(B) if seqs is None else seqs
    seqs = list(seqs)
    out = np.zeros((len(seqs), Hq, d), dtype=np.float64)
    for i, s in enumerate(seqs):
        n = int(context_lens[s])
        if n == 0:
            continue
        qf = bits_to_f64(q[s], dtype)
        for hk in range(Hkv):
            K = gather_sequence(k_cache, block_tables[s], n, hk, dtype)
            V = gather_sequence(v_cache, block_tables[s], n, hk, dtype)
            for g in range(G):
                h = hk * G + g
                out[i, h] = softmax_attention(qf[h], K, V, scale)
    return out


# ----------------------------------------------------------------------------
# split-context form: per-partition partials and their exact merge
# ----------------------------------------------------------------------------
def partition_partials(qv, K, V, scale, partition):
    """(m_p, l_p, o_p) for consecutive token ranges of ``partition`` tokens:
    m_p = max score, l_p = sum exp(score - m_p), o_p = normalised partial output."""
    parts = []
    n = K.shape[0]
    for a in range(0, n, partition):
        x = scale * (K[a:a + partition] @ qv)
        m = x.max()
        p = np.exp(x - m)
        parts.append((m, p.sum(), (p @ V[a:a + partition]) / p.sum()))
    return parts


def merge_partitions(parts):
    """Log-sum-exp merge: M = max m_p; w_p = l_p exp(m_p - M); out = sum w_p o_p / sum w_p."""
    M = max(m for m, _, _ in parts)
    w = np.array([l * np.exp(m - M) for m, l, _ in parts])
    o = np.stack([o for _, _, o in parts])
    return (w[:, None] * o).sum(0) / w.sum()
