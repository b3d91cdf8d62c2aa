"""Pins of the allocator model's prefix caching ("vLLM explained",
"Prefix Caching：相同前綴只算一次"): a block is in use (count > 0), free and
empty, or free but keeping its content (count 0) for reuse; a new request
reuses the blocks of an identical prefix; new blocks come from the empty ones
first and only then from the cached ones, least recently used first; blocks in
use are never taken.

The scenario below is worked out by hand from those rules.  The randomised
test checks a property that does not depend on how the model finds a hit: a
simulated cache whose "K/V" are the token ids themselves, written only where
the caller would write (tokens past the reused prefix), must read back every
live sequence's own tokens through its block table.
"""
import random

from oracle.alloc_model import AllocModel, INVALID_ARG, OK, OOM

B = 16
SYS = list(range(1000, 1032))  # a 32-token system prompt: two full blocks


def test_worked_scenario():
    m = AllocModel(6, B)
    assert m.set_prefix_caching(True) == OK
    # A: system prompt + 8 tokens -> blocks 0, 1 (full, registered), 2 (partial)
    st, slots, nc = m.admit("A", SYS + list(range(2000, 2008)))
    assert st == OK and nc == 0 and slots == list(range(40))
    assert m.block_table("A") == [0, 1, 2]
    # B shares the system prompt: blocks 0 and 1 reused, 32 tokens need no prefill
    st, slots, nc = m.admit("B", SYS + list(range(3000, 3005)))
    assert st == OK and nc == 32
    assert m.block_table("B") == [0, 1, 3] and m.refcount(0) == m.refcount(1) == 2
    assert slots[:32] == list(range(32)) and slots[32:] == [48, 49, 50, 51, 52]
    # A ends: its partial block 2 is empty again; 0 and 1 stay in use by B
    assert m.free_seq("A") == OK
    assert m.free_list() == [4, 5, 2] and m.cached_list() == []
    # B ends: released last block first -> 3 empty, then 1, 0 cached (LRU order)
    assert m.free_seq("B") == OK
    assert m.free_list() == [4, 5, 2, 3] and m.cached_list() == [1, 0]
    # C (48 new tokens) takes empty blocks only; the cache is untouched
    C = list(range(4000, 4048))
    st, _, nc = m.admit("C", C)
    assert st == OK and nc == 0 and m.block_table("C") == [4, 5, 2]
    assert m.free_list() == [3] and m.cached_list() == [1, 0]
    # D (20 tokens) needs 2: the last empty block, then the LRU cached one (1)
    st, _, nc = m.admit("D", list(range(5000, 5020)))
    assert st == OK and nc == 0 and m.block_table("D") == [3, 1]
    assert m.free_list() == [] and m.cached_list() == [0]
    # E = system prompt + 1: block 0 still holds the first 16 tokens, but the
    # second block's content was evicted with block 1; E needs 2 new blocks and
    # only the revived block 0 is left -> refused, nothing changes
    E = SYS + [6000]
    st, slots, nc = m.admit("E", E)
    assert (st, slots, nc) == (OOM, [], 0)
    assert m.cached_list() == [0] and m.refcount(0) == 0
    # C ends: 2, 5, 4 become cached (last block first)
    assert m.free_seq("C") == OK
    assert m.cached_list() == [0, 2, 5, 4]
    # E again: revives 0 (16 tokens cached), evicts 2 then 5 for its other blocks
    st, _, nc = m.admit("E", E)
    assert st == OK and nc == 16 and m.block_table("E") == [0, 2, 5]
    assert m.cached_list() == [4] and m.free_list() == []
    assert [m.refcount(b) for b in range(6)] == [1, 1, 1, 1, 0, 1]
    # C's prompt now hits only its first block (4); its second went with 5
    m.free_seq("D")
    st, _, nc = m.admit("F", C)
    assert st == OK and nc == 16 and m.block_table("F")[0] == 4


def test_switch_only_without_sequences():
    m = AllocModel(4, B)
    m.append("x", 3)
    assert m.set_prefix_caching(True) == INVALID_ARG
    m.free_seq("x")
    assert m.set_prefix_caching(True) == OK


def test_tokens_without_ids_are_never_registered():
    m = AllocModel(8, B)
    m.set_prefix_caching(True)
    m.append("a", 16)                      # no ids: nothing to hash
    m.free_seq("a")
    assert m.cached_list() == [] and m.num_free() == 8
    st, _, _ = m.admit("b", SYS[:10])
    m.append("b", 6)                       # ids of these 6 unknown -> not registered
    m.free_seq("b")
    assert m.cached_list() == []


def _check_state(m, pool, live):
    nb = len(m.rc)
    # every block in exactly one state; counts = table references
    refs = [0] * nb
    for t in m.tables.values():
        for b in t:
            refs[b] += 1
    assert refs == m.rc
    in_use = {b for b in range(nb) if m.rc[b] > 0}
    free, cached = set(m.free_list()), set(m.cached_list())
    assert len(free) == len(m.free_list()) and len(cached) == len(m.cached_list())
    assert in_use.isdisjoint(free) and in_use.isdisjoint(cached) and free.isdisjoint(cached)
    assert in_use | free | cached == set(range(nb))
    assert cached <= set(m.key)            # a cached block keeps a registered prefix
    # every live sequence reads its own tokens back through its table
    for s, toks in live.items():
        table = m.block_table(s)
        for p, tok in enumerate(toks):
            assert pool.get(table[p // B] * B + p % B) == tok, (s, p)
    # a registered block in use or cached holds its prefix's last 16 tokens
    for b, prefix in m.key.items():
        assert [pool.get(b * B + o) for o in range(B)] == list(prefix[-B:])


def test_random_sequences_read_back_their_tokens():
    rng = random.Random(2024)
    prefixes = [[rng.randrange(1 << 20) for _ in range(rng.choice([16, 24, 40, 64]))]
                for _ in range(5)]
    hits = evictions = 0
    for trial in range(40):
        nb = rng.choice([10, 16, 24])
        m = AllocModel(nb, B, rng.sample(range(nb), nb))
        m.set_prefix_caching(True)
        pool, live, next_id = {}, {}, 0
        for _ in range(120):
            op = rng.random()
            if op < 0.35 or not live:
                toks = list(rng.choice(prefixes)) + [rng.randrange(1 << 20)
                                                     for _ in range(rng.randrange(0, 30))]
                cached_before = set(m.cached_list())
                st, slots, nc = m.admit(next_id, toks)
                if st == OK:
                    hits += nc > 0
                    evictions += len(cached_before - set(m.cached_list())
                                     - set(m.block_table(next_id)[:nc // B]))
                    assert nc % B == 0 and nc <= len(toks)
                    # the reused tokens are already there; the rest are written now
                    for p in range(nc):
                        assert pool[slots[p]] == toks[p]
                    for p in range(nc, len(toks)):
                        pool[slots[p]] = toks[p]
                    live[next_id] = toks
                next_id += 1
            elif op < 0.6:
                s = rng.choice(list(live))
                st, pairs = m.prepare_write(s)
                if st != OK:
                    continue
                for src, dst in pairs:
                    for o in range(B):
                        pool[dst * B + o] = pool.get(src * B + o)
                add = [rng.randrange(1 << 20) for _ in range(rng.randrange(1, 20))]
                st, slots = m.append_tokens(s, add)
                if st == OK:
                    for sl, tok in zip(slots, add):
                        pool[sl] = tok
                    live[s] = live[s] + add
            elif op < 0.7:
                s = rng.choice(list(live))
                if m.fork(s, next_id) == OK:
                    live[next_id] = list(live[s])
                next_id += 1
            else:
                s = rng.choice(list(live))
                assert m.free_seq(s) == OK
                del live[s]
            _check_state(m, pool, live)
    assert hits > 100 and evictions > 20  # the walk exercised reuse and eviction
