"""The product's C++ block allocator against the reference model: identical
state (tables, refcounts, token counts, FIFO free queue) after every call of
long random call sequences, plus the pages' worked example."""
import random

import pytest

from oracle.alloc_model import AllocModel


@pytest.fixture(scope="module")
def B():
    from pagedattention_paged_kv_pa_b200 import build
    build.build()
    from pagedattention_paged_kv_pa_b200 import binding
    return binding


def _same_state(a, m, seqs, n):
    assert a.free_list() == m.free_list()
    assert [a.refcount(b) for b in range(n)] == m.rc
    assert a.num_seqs() == len(m.tables)
    for s in seqs:
        if s in m.tables:
            assert a.block_table(s) == m.block_table(s)
            assert a.num_tokens(s) == m.ntok[s]
        else:
            assert a.num_tokens(s) == -1


def test_worked_example(B):
    order = [7, 2, 9, 5] + [i for i in range(12) if i not in (7, 2, 9, 5)]
    a = B.BlockAllocator(12, 16, order)
    assert a.append(1, 16)[0] == 0
    assert a.fork(1, 2) == 0
    assert a.append(1, 32)[0] == 0
    assert a.append(2, 16)[0] == 0
    assert a.block_table(1) == [7, 2, 9]
    assert a.block_table(2) == [7, 5]
    assert a.refcount(7) == 2


def test_create_rejects_bad_arguments(B):
    with pytest.raises(B.PAError):
        B.BlockAllocator(0)
    with pytest.raises(B.PAError):
        B.BlockAllocator(4, 32)
    with pytest.raises(B.PAError):
        B.BlockAllocator(3, 16, [0, 0, 1])


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_random_call_sequences_match_model(B, seed):
    rnd = random.Random(seed)
    N = rnd.choice([8, 33, 100])
    order = rnd.sample(range(N), N)
    a = B.BlockAllocator(N, 16, order)
    m = AllocModel(N, 16, order)
    seqs = list(range(60))
    for _ in range(2500):
        op = rnd.random()
        s = rnd.choice(seqs)
        if op < 0.45:
            n = rnd.choice([0, 1, 3, 15, 16, 17, 40])
            ra = a.append(s, n)
            rm = m.append(s, n)
            assert ra == (rm[0], rm[1])
        elif op < 0.6:
            c = rnd.choice(seqs)
            assert a.fork(s, c) == m.fork(s, c)
        elif op < 0.8:
            ra = a.prepare_write(s)
            rm = m.prepare_write(s)
            assert ra[0] == rm[0] and ra[1] == rm[1]
        else:
            assert a.free_seq(s) == m.free_seq(s)
        _same_state(a, m, seqs, N)


@pytest.mark.parametrize("seed", [11, 12, 13, 14])
def test_prefix_caching_call_sequences_match_model(B, seed):
    """Prefix caching on: admissions drawn from a few shared prompts, token
    appends, plain appends, forks, copy-on-write and frees; statuses, slots,
    reused-token counts, free queue and cached (LRU) list agree after every
    call."""
    rnd = random.Random(seed)
    N = rnd.choice([12, 24, 40])
    order = rnd.sample(range(N), N)
    a = B.BlockAllocator(N, 16, order)
    m = AllocModel(N, 16, order)
    assert a.set_prefix_caching(True) == m.set_prefix_caching(True) == 0
    prompts = [[rnd.randrange(1 << 30) for _ in range(rnd.choice([16, 32, 40, 70]))]
               for _ in range(6)]
    seqs = list(range(40))
    hits = 0
    for _ in range(2000):
        op = rnd.random()
        s = rnd.choice(seqs)
        if op < 0.3:
            toks = list(rnd.choice(prompts))[:rnd.choice([16, 20, 32, 48, 70])]
            toks += [rnd.randrange(1 << 30) for _ in range(rnd.choice([0, 1, 9, 16]))]
            ra, rm = a.admit(s, toks), m.admit(s, toks)
            assert ra == rm
            hits += ra[2] > 0
        elif op < 0.5:
            toks = [rnd.randrange(1 << 30) for _ in range(rnd.choice([1, 5, 16, 23]))]
            assert a.append_tokens(s, toks) == m.append_tokens(s, toks)
        elif op < 0.55:
            n = rnd.choice([1, 16])
            ra, rm = a.append(s, n), m.append(s, n)
            assert ra == (rm[0], rm[1])
        elif op < 0.65:
            c = rnd.choice(seqs)
            assert a.fork(s, c) == m.fork(s, c)
        elif op < 0.75:
            ra, rm = a.prepare_write(s), m.prepare_write(s)
            assert ra[0] == rm[0] and ra[1] == rm[1]
        else:
            assert a.free_seq(s) == m.free_seq(s)
        _same_state(a, m, seqs, N)
        assert a.cached_list() == m.cached_list()
        assert a.num_cached() == len(m.cached)
    assert hits > 20  # the walk exercised prefix reuse


def test_prefix_caching_switch_and_admit_errors(B):
    a = B.BlockAllocator(4, 16)
    a.append(1, 3)
    assert a.set_prefix_caching(True) == B.PA_ERR_INVALID_ARG
    a.free_seq(1)
    assert a.set_prefix_caching(True) == 0
    assert a.admit(5, list(range(20)))[0] == 0
    assert a.admit(5, list(range(20)))[0] == B.PA_ERR_INVALID_ARG   # id in use
    assert a.admit(6, list(range(100)))[0] == B.PA_ERR_OOM
