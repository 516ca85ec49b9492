"""KV memory utilisation.

Source: "vLLM / PagedAttention — 分页 KV Cache 分析", §4.2: effective utilisation
is approximately the sum of sequence lengths over (number of blocks x page
size) — tokens actually used over tokens allocated. The "vLLM" entity page
(是什么) gives the contrast: contiguous preallocation keeps only 20.4%–38.2% of
KV memory holding token state.

Readings:
* "number of blocks" = blocks held (refcount > 0). Without sharing that is
  sum_s ceil(len_s / bs), so util = sum len / (sum ceil(len/bs) * bs) exactly.
  With sharing the same ratio counts logical tokens and may exceed 1.
* The contiguous analogue preallocates ``max_len`` slots per sequence.
"""
from __future__ import annotations


def paged_utilisation(lens, block_size):
    used = sum(int(n) for n in lens)
    alloc = sum(-(-int(n) // block_size) * block_size for n in lens)
    return used / alloc if alloc else 0.0


def utilisation_from_state(logical_tokens, held_blocks, block_size):
    return logical_tokens / (held_blocks * block_size) if held_blocks else 0.0


def contiguous_utilisation(lens, max_len):
    return sum(int(n) for n in lens) / (len(lens) * max_len) if len(lens) else 0.0


def waste_lower_bound(lens, block_size):
    """Each sequence wastes at most bs-1 slots of its last block, so
    util >= sum len / (sum len + B (bs - 1))."""
    used = sum(int(n) for n in lens)
    return used / (used + len(lens) * (block_size - 1)) if used else 0.0
