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

Prefix caching ("vLLM / PagedAttention — 分页 KV Cache 分析" §2.3 and §3.2: common
prefixes such as system prompts are detected automatically and their pages reused
across requests; §五: only an exactly identical token sequence may share). The pages
give no mechanism; readings (the same in the C++ allocator):
* Only full blocks are cached. Block j of a token list is identified by the 64-bit
  hash of the whole prefix ``tokens[: (j+1)*bs]``: start at 0 and fold every token
  in with ``h = splitmix64(h ^ token)``; a hit also requires the cached block's
  prefix to equal the query's exactly.
* A sequence takes part while every token it holds came with its id (created by
  ``append_tokens`` or ``share_prefix`` with the cache on); an ``append`` without
  ids stops it. When such a sequence fills a block whose prefix is not cached yet,
  that block becomes cached.
* A cached block whose count falls to 0 is kept (evictable), most recently released
  last. A new block comes from the free stack first, else the least recently
  released evictable block leaves the cache and is reused. Evictable blocks count
  as free.
* ``share_prefix(seq, tokens)`` creates ``seq`` on the longest run of cached full
  blocks matching ``tokens`` from the start (at most ``max_blocks_per_seq``), one
  reference more each, and reports the tokens covered.
* Turning the cache off forgets every entry; evictable blocks go to the free stack
  (in release order) and no sequence takes part any more.
"""
from __future__ import annotations

from collections import OrderedDict

_MASK64 = (1 << 64) - 1


def splitmix64(x):
    """One step of splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
    number generators", OOPSLA 2014): add the golden-ratio increment, then the
    variant-13 finaliser. Seeded with 0, the generator's outputs are
    splitmix64(0), splitmix64(gamma), ..."""
    z = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def prefix_hash(tokens):
    """Hash of a whole token prefix (token ids as unsigned 32-bit values)."""
    h = 0
    for t in tokens:
        h = splitmix64(h ^ (int(t) & 0xFFFFFFFF))
    return h

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
        # prefix cache
        self.prefix_cache = False
        self.cache = {}                             # hash -> (prefix tuple, block)
        self.block_hash = {}                        # cached block -> its hash
        self.evictable = OrderedDict()              # block -> None, oldest release first
        self.ids = {}                               # taking-part seq -> its token ids
        self.query_tokens = 0
        self.hit_tokens = 0

    # -- helpers -----------------------------------------------------------
    def _pop(self):
        if self.free_stack:
            b = self.free_stack.pop()
        else:
            b, _ = self.evictable.popitem(last=False)
            del self.cache[self.block_hash.pop(b)]
        self.refcount[b] = 1
        return b

    def _unref(self, b):
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            if b in self.block_hash:
                self.evictable[b] = None
            else:
                self.free_stack.append(b)

    def available(self):
        return len(self.free_stack) + len(self.evictable)

    def _placed(self, seq, token):
        """Token `token` (None: no id) was just placed at position lens[seq]-1."""
        if seq not in self.ids:
            return
        if token is None:
            del self.ids[seq]
            return
        ids = self.ids[seq]
        ids.append(int(token))
        n = len(ids)
        if n % self.bs:
            return
        h = prefix_hash(ids)
        if h not in self.cache:
            b = self.tables[seq][n // self.bs - 1]
            self.cache[h] = (tuple(ids), b)
            self.block_hash[b] = h

    def blocks_needed(self, seq, n_tokens):
        n = self.lens.get(seq, 0)
        table = self.tables.get(seq, [])
        need = 0
        if n % self.bs != 0 and table and self.refcount[table[-1]] > 1 and n_tokens > 0:
            need += 1
        new = sum(1 for p in range(n, n + n_tokens) if p % self.bs == 0)
        return need + new, -(-(n + n_tokens) // self.bs)

    # -- interface -----------------------------------------------------------
    def append(self, seq, n_tokens, token_ids=None):
        """Returns (status, slots, cow_pairs). ``token_ids``: the appended tokens' ids."""
        if n_tokens < 0:
            return ERR_INVALID_ARG, [], []
        need, table_len = self.blocks_needed(seq, n_tokens)
        if table_len > self.mb:
            return ERR_TABLE_FULL, [], []
        if need > self.available():
            return ERR_OUT_OF_BLOCKS, [], []
        if seq not in self.tables and self.prefix_cache and token_ids is not None:
            self.ids[seq] = []
        table = self.tables.setdefault(seq, [])
        self.lens.setdefault(seq, 0)
        slots, cows = [], []
        for i in range(n_tokens):
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
            self._placed(seq, None if token_ids is None else token_ids[i])
        return OK, slots, cows

    def append_tokens(self, seq, token_ids):
        return self.append(seq, len(token_ids), list(token_ids))

    def set_prefix_cache(self, enable):
        if self.prefix_cache and not enable:
            for b in self.evictable:
                self.free_stack.append(b)
            self.evictable.clear()
            self.cache.clear()
            self.block_hash.clear()
            self.ids.clear()
        self.prefix_cache = bool(enable)
        return OK

    def share_prefix(self, seq, token_ids):
        """Returns (status, tokens covered)."""
        if seq in self.tables:
            return ERR_SEQ_EXISTS, 0
        toks = [int(t) for t in token_ids]
        table = []
        if self.prefix_cache:
            j = 0
            while (j + 1) * self.bs <= len(toks) and j < self.mb:
                pre = tuple(toks[: (j + 1) * self.bs])
                hit = self.cache.get(prefix_hash(pre))
                if hit is None or hit[0] != pre:
                    break
                b = hit[1]
                if self.refcount[b] == 0:
                    del self.evictable[b]
                self.refcount[b] += 1
                table.append(b)
                j += 1
            self.query_tokens += len(toks)
            self.hit_tokens += len(table) * self.bs
            self.ids[seq] = toks[: len(table) * self.bs]
        self.tables[seq] = table
        self.lens[seq] = len(table) * self.bs
        return OK, self.lens[seq]

    def free_list(self):
        """The blocks the next allocations take, in order."""
        return list(reversed(self.free_stack)) + list(self.evictable)

    def prefix_cache_stats(self):
        return len(self.cache), len(self.evictable), self.query_tokens, self.hit_tokens

    def fork(self, parent, child):
        if parent not in self.tables:
            return ERR_UNKNOWN_SEQ
        if child in self.tables:
            return ERR_SEQ_EXISTS
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        if parent in self.ids:
            self.ids[child] = list(self.ids[parent])
        for b in self.tables[child]:
            self.refcount[b] += 1
        return OK

    def free(self, seq):
        if seq not in self.tables:
            return ERR_UNKNOWN_SEQ
        for b in reversed(self.tables[seq]):
            self._unref(b)
        del self.tables[seq]
        del self.lens[seq]
        self.ids.pop(seq, None)
        return OK

    def block_table(self, seq):
        row = list(self.tables[seq]) + [-1] * (self.mb - len(self.tables[seq]))
        return row, self.lens[seq]

    def prefix_groups(self, seqs):
        """Groups of sequences that share their prompt's pages ("分页 KV Cache 分析" §3.2;
        "vLLM" entity page, 是什么), as the shared-prefix decode takes them. Reading (the
        pages fix no rule): sequences whose first full block is the same physical block are
        one group, groups in order of their first member, members in the given order; a
        sequence without a full block is alone. A group's prefix is the number of leading
        blocks all members hold in common, each member counting only its full blocks, times
        the block size (0 alone). Returns (order, group_start, prefix_lens)."""
        seqs = [int(x) for x in seqs]
        if len(set(seqs)) != len(seqs):
            raise ValueError("a sequence listed twice")
        groups, by_first = [], {}
        for s_ in seqs:
            table, n = self.tables[s_], self.lens[s_]
            if n >= self.bs and table:
                key = table[0]
                if key in by_first:
                    groups[by_first[key]].append(s_)
                    continue
                by_first[key] = len(groups)
            groups.append([s_])
        order, starts, prefixes = [], [], []
        for members in groups:
            starts.append(len(order))
            order += members
            if len(members) == 1:
                prefixes.append(0)
                continue
            full = min(self.lens[m] // self.bs for m in members)
            common = 0
            while common < full and all(self.tables[m][common] == self.tables[members[0]][common]
                                        for m in members):
                common += 1
            prefixes.append(common * self.bs)
        starts.append(len(order))
        return order, starts, prefixes

    def stats(self):
        free = self.available()
        held = self.nb - free
        tokens = sum(self.lens.values())
        util = tokens / (held * self.bs) if held else 0.0
        return free, held, tokens, util
