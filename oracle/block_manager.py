"""Model of the host KV block manager: free list, refcounts, fork, copy-on-write.

Sources:
* "vLLM" entity page, 是什么: each sequence is cut into fixed-size logical blocks
  mapped by a block table to any physical block; a request asks for a new block
  only when it needs one; the last, unfilled block is the only internal
  fragmentation; parallel sampling / beam search / common prompts share physical
  blocks through reference counts and copy-on-write.
* "vLLM / PagedAttention — 分页 KV Cache 分析", §2.3 (KV Block Manager: a global
  physical-page allocator; one block table per request; copy-on-write for shared
  prefixes) and §3.2 (a request that must change a shared page copies it first).
* §3.3 of the same page: finished requests release their pages at once.

The pages fix no order, so these are readings (identical in the C++ allocator):
* The free list is a LIFO stack, seeded so that successive pops return
  ``initial_order[0], initial_order[1], ...``.
* ``append`` of one token at length ``n``: if ``n % bs == 0`` pop a new block
  (refcount 1); else if the last block's refcount is > 1, pop ``b'``, record the
  copy-on-write pair (last, b'), drop one reference to the old block, put ``b'``
  in the table with refcount 1. The token's slot is
  ``table[n // bs] * bs + n % bs``; then ``n += 1``.
* ``append`` of k tokens is all-or-nothing: the blocks it needs are counted
  first; if too few are free, or the table would exceed ``max_blocks_per_seq``,
  nothing changes.
* ``fork`` copies the parent's table and length and adds a reference to every
  block; ``free`` walks the table from the last logical block to the first,
  drops one reference each, and pushes a block whose count reaches 0.
* When n sequences share a partial block, the first n-1 writers copy and the
  last writes in place (its count is 1 by then); the order is the call order.
"""
from __future__ import annotations

# status codes of the block-manager interface (same numeric values as the library)
OK = 0
ERR_INVALID_ARG = -1
ERR_OUT_OF_BLOCKS = -2
ERR_UNKNOWN_SEQ = -3
ERR_SEQ_EXISTS = -4
ERR_TABLE_FULL = -5


class BlockManagerModel:
    def __init__(self, num_blocks, block_size, max_blocks_per_seq, initial_order=None):
        if num_blocks <= 0 or block_size <= 0 or max_blocks_per_seq <= 0:
            raise ValueError("bad sizes")
        order = list(range(num_blocks)) if initial_order is None else [int(b) for b in initial_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("initial_order must be a permutation of 0..num_blocks-1")
        self.nb = num_blocks
        self.bs = block_size
        self.mb = max_blocks_per_seq
        self.free_stack = list(reversed(order))     # pop() takes from the end
        self.refcount = [0] * num_blocks
        self.tables = {}                            # seq id -> list of block ids
        self.lens = {}                              # seq id -> tokens

    # -- helpers -----------------------------------------------------------
    def _pop(self):
        b = self.free_stack.pop()
        self.refcount[b] = 1
        return b

    def blocks_needed(self, seq, n_tokens):
        n = self.lens.get(seq, 0)
        table = self.tables.get(seq, [])
        need = 0
        if n % self.bs != 0 and table and self.refcount[table[-1]] > 1 and n_tokens > 0:
            need += 1
        new = sum(1 for p in range(n, n + n_tokens) if p % self.bs == 0)
        return need + new, -(-(n + n_tokens) // self.bs)

    # -- interface -----------------------------------------------------------
    def append(self, seq, n_tokens):
        """Returns (status, slots, cow_pairs)."""
        if n_tokens < 0:
            return ERR_INVALID_ARG, [], []
        need, table_len = self.blocks_needed(seq, n_tokens)
        if table_len > self.mb:
            return ERR_TABLE_FULL, [], []
        if need > len(self.free_stack):
            return ERR_OUT_OF_BLOCKS, [], []
        table = self.tables.setdefault(seq, [])
        self.lens.setdefault(seq, 0)
        slots, cows = [], []
        for _ in range(n_tokens):
            n = self.lens[seq]
            if n % self.bs == 0:
                table.append(self._pop())
            elif self.refcount[table[-1]] > 1:
                old = table[-1]
                new = self._pop()
                cows.append((old, new))
                self.refcount[old] -= 1
                table[-1] = new
            slots.append(table[n // self.bs] * self.bs + n % self.bs)
            self.lens[seq] = n + 1
        return OK, slots, cows

    def fork(self, parent, child):
        if parent not in self.tables:
            return ERR_UNKNOWN_SEQ
        if child in self.tables:
            return ERR_SEQ_EXISTS
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.refcount[b] += 1
        return OK

    def free(self, seq):
        if seq not in self.tables:
            return ERR_UNKNOWN_SEQ
        for b in reversed(self.tables[seq]):
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free_stack.append(b)
        del self.tables[seq]
        del self.lens[seq]
        return OK

    def block_table(self, seq):
        row = list(self.tables[seq]) + [-1] * (self.mb - len(self.tables[seq]))
        return row, self.lens[seq]

    def stats(self):
        free = len(self.free_stack)
        held = self.nb - free
        tokens = sum(self.lens.values())
        util = tokens / (held * self.bs) if held else 0.0
        return free, held, tokens, util
