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
