"""Reference model of the block allocator -- TEST INFRASTRUCTURE ONLY.

A deliberately plain Python restatement of the memory-management layer the
pages describe, used to check the product's C++ allocator state bit for bit:

* KV cache split into fixed-size blocks (16 tokens), physical blocks need not
  be contiguous, a per-sequence block table maps logical to physical blocks,
  a new block is taken only when needed and a finished request's blocks go
  back ("vLLM explained", "PagedAttention：用分頁管理 KV cache", items 1-4;
  "LLM inference optimization", §三.1);
* sharing by reference count: forked sequences point at the same physical
  blocks with the count raised; a block is copied only when one branch is
  about to write a token the others do not share (copy-on-write)
  ("LLM inference optimization", §三.2; "vLLM explained", "帶來的好處");
* a block in use (count > 0) is never handed out again ("vLLM explained",
  "KV cache 什麼時候可以被覆蓋", first row of the table).

Readings where the pages are silent: free blocks are handed out in FIFO order
from an initial order (default 0..N-1) and freed blocks join the back of the
queue; a request that cannot be met in full changes nothing (all-or-nothing);
appending into a partially filled block that is shared is refused until
``prepare_write`` has split it.

Prefix caching ("vLLM explained", "Prefix Caching：相同前綴只算一次"), when
switched on: a block is in use (count > 0), free and empty, or free but still
holding cached content (count 0, content kept for reuse).  A full block whose
tokens are known is identified by its whole prefix -- every token from the
start of the sequence to the end of the block (the page's hash matching; this
model compares the token tuples themselves, no hash).  A new request reuses
the longest run of leading full blocks whose prefixes are held by a block in
use or cached, and needs no prefill for those tokens.  A new block comes from
the empty blocks first; only when there are none is a cached block evicted,
least recently used first; blocks in use are never taken.  When a request
ends, its registered blocks whose count reaches zero become cached instead of
empty.  Readings: a sequence's blocks are released from its last block to
its first, so of blocks freed together the prefix's tail is evicted before
its head; a second block with an already registered prefix (a duplicate)
stays unregistered and returns to the empty blocks when freed; the last
partial block of a sequence is never registered.
"""
from __future__ import annotations

import collections

OK, INVALID_ARG, UNSUPPORTED, OOM = 0, 1, 2, 3


class AllocModel:
    def __init__(self, num_blocks: int, block_size: int = 16, initial_free_order=None):
        order = list(range(num_blocks)) if initial_free_order is None else list(initial_free_order)
        assert sorted(order) == list(range(num_blocks))
        self.block_size = block_size
        self.free = collections.deque(order)
        self.rc = [0] * num_blocks
        self.tables = {}   # seq -> list of physical block ids (logical order)
        self.ntok = {}     # seq -> number of tokens written
        # prefix caching
        self.prefix_caching = False
        self.tokens = {}   # seq -> list of token ids, or None once unknown
        self.key = {}      # registered block -> its whole prefix (tuple of tokens)
        self.holder = {}   # prefix tuple -> the registered block holding it
        self.cached = collections.OrderedDict()  # free blocks with content, LRU first

    def set_prefix_caching(self, on: bool) -> int:
        if self.tables:
            return INVALID_ARG
        self.prefix_caching = bool(on)
        return OK

    # -- block supply -----------------------------------------------------------
    def num_allocatable(self) -> int:
        return len(self.free) + len(self.cached)

    def _take(self) -> int:
        """An empty block if there is one, else the least recently used cached
        block, whose content is forgotten."""
        if self.free:
            b = self.free.popleft()
        else:
            b, _ = self.cached.popitem(last=False)
            del self.holder[self.key.pop(b)]
        self.rc[b] = 1
        return b

    def _register_full_blocks(self, seq, first_block: int):
        """Register the sequence's full blocks from first_block on (known tokens only)."""
        toks = self.tokens.get(seq)
        if not self.prefix_caching or toks is None:
            return
        B = self.block_size
        blocks = self.tables[seq]
        for i in range(first_block, len(toks) // B):
            prefix = tuple(toks[:(i + 1) * B])
            b = blocks[i]
            if b in self.key or prefix in self.holder:
                continue  # already registered, or a duplicate of a registered block
            self.key[b] = prefix
            self.holder[prefix] = b

    # -- queries --------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def refcount(self, b: int) -> int:
        return self.rc[b]

    def block_table(self, seq):
        return list(self.tables[seq])

    def num_tokens(self, seq) -> int:
        return self.ntok.get(seq, -1)

    def free_list(self):
        return list(self.free)

    def cached_list(self):
        return list(self.cached)

    # -- operations -------------------------------------------------------------
    def append(self, seq, n_tokens: int):
        """Reserve slots for n_tokens new tokens; returns (status, slots)."""
        if n_tokens < 0:
            return INVALID_ARG, []
        blocks = self.tables.get(seq, [])
        n = self.ntok.get(seq, 0)
        B = self.block_size
        if n_tokens > 0 and n % B != 0 and self.rc[blocks[-1]] > 1:
            return INVALID_ARG, []
        have = -(-n // B)
        need = -(-(n + n_tokens) // B) - have
        if need > self.num_allocatable():
            return OOM, []
        blocks = list(blocks)
        for _ in range(need):
            blocks.append(self._take())
        slots = [blocks[p // B] * B + p % B for p in range(n, n + n_tokens)]
        if n_tokens > 0 or seq not in self.tables:
            self.tokens[seq] = None  # tokens without ids: this sequence is no longer known
        self.tables[seq] = blocks
        self.ntok[seq] = n + n_tokens
        return OK, slots

    def append_tokens(self, seq, tokens):
        """append() for tokens whose ids are known: full blocks get registered."""
        known = self.tokens.get(seq) if seq in self.tables else []
        st, slots = self.append(seq, len(tokens))
        if st != OK:
            return st, []
        B = self.block_size
        n0 = self.ntok[seq] - len(tokens)
        self.tokens[seq] = None if known is None else list(known) + list(tokens)
        self._register_full_blocks(seq, n0 // B)
        return OK, slots

    def admit(self, seq, tokens):
        """A new sequence with a prompt of known tokens.  Returns
        (status, slots, n_cached): the leading n_cached tokens' K/V are already
        in the cache (reused full blocks) and need no prefill."""
        if seq in self.tables:
            return INVALID_ARG, [], 0
        B = self.block_size
        n = len(tokens)
        hits = []
        if self.prefix_caching:
            for i in range(n // B):
                b = self.holder.get(tuple(tokens[:(i + 1) * B]))
                if b is None:
                    break
                hits.append(b)
        revived = sum(1 for b in hits if self.rc[b] == 0)
        need = -(-n // B) - len(hits)
        if need > self.num_allocatable() - revived:
            return OOM, [], 0
        for b in hits:
            if self.rc[b] == 0:
                del self.cached[b]
            self.rc[b] += 1
        blocks = list(hits)
        for _ in range(need):
            blocks.append(self._take())
        self.tables[seq] = blocks
        self.ntok[seq] = n
        self.tokens[seq] = list(tokens)
        self._register_full_blocks(seq, len(hits))
        slots = [blocks[p // B] * B + p % B for p in range(n)]
        return OK, slots, len(hits) * B

    def fork(self, parent, child) -> int:
        if parent not in self.tables or child in self.tables:
            return INVALID_ARG
        self.tables[child] = list(self.tables[parent])
        self.ntok[child] = self.ntok[parent]
        t = self.tokens.get(parent)
        self.tokens[child] = None if t is None else list(t)
        for b in self.tables[child]:
            self.rc[b] += 1
        return OK

    def prepare_write(self, seq):
        """Copy-on-write of a shared, partially filled last block.
        Returns (status, [(src, dst)]) -- at most one pair."""
        if seq not in self.tables:
            return INVALID_ARG, []
        blocks, n, B = self.tables[seq], self.ntok[seq], self.block_size
        if n % B == 0 or self.rc[blocks[-1]] <= 1:
            return OK, []
        if self.num_allocatable() == 0:
            return OOM, []
        old = blocks[-1]
        new = self._take()
        self.rc[old] -= 1
        blocks[-1] = new
        return OK, [(old, new)]

    def free_seq(self, seq) -> int:
        if seq not in self.tables:
            return INVALID_ARG
        for b in reversed(self.tables.pop(seq)):  # last block first
            self.rc[b] -= 1
            if self.rc[b] == 0:
                if b in self.key:
                    self.cached[b] = None      # most recently used end
                else:
                    self.free.append(b)
        del self.ntok[seq]
        self.tokens.pop(seq, None)
        return OK
