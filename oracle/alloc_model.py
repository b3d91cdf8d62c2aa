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
        if need > len(self.free):
            return OOM, []
        blocks = list(blocks)
        for _ in range(need):
            b = self.free.popleft()
            self.rc[b] = 1
            blocks.append(b)
        slots = [blocks[p // B] * B + p % B for p in range(n, n + n_tokens)]
        self.tables[seq] = blocks
        self.ntok[seq] = n + n_tokens
        return OK, slots

    def fork(self, parent, child) -> int:
        if parent not in self.tables or child in self.tables:
            return INVALID_ARG
        self.tables[child] = list(self.tables[parent])
        self.ntok[child] = self.ntok[parent]
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
        if not self.free:
            return OOM, []
        old = blocks[-1]
        new = self.free.popleft()
        self.rc[new] = 1
        self.rc[old] -= 1
        blocks[-1] = new
        return OK, [(old, new)]

    def free_seq(self, seq) -> int:
        if seq not in self.tables:
            return INVALID_ARG
        for b in self.tables.pop(seq):
            self.rc[b] -= 1
            if self.rc[b] == 0:
                self.free.append(b)
        del self.ntok[seq]
        return OK
