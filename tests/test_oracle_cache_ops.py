"""Pins for the oracle's slot write, block copy and allocator model (CPU only)."""
import os
import random

import numpy as np
import pytest
import torch

import oracle as orc
from oracle.alloc_model import AllocModel, OK, OOM, INVALID_ARG

B = 16
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# reshape_and_cache
# ---------------------------------------------------------------------------

def test_slot_write_same_dtype_matches_numpy_fancy_index():
    rng = np.random.default_rng(1)
    nb, n_kv, d, T = 20, 4, 64, 50
    kp = rng.standard_normal((nb, n_kv, B, d)).astype(np.float16)
    vp = rng.standard_normal((nb, n_kv, B, d)).astype(np.float16)
    key = rng.standard_normal((T, n_kv, d)).astype(np.float16)
    val = rng.standard_normal((T, n_kv, d)).astype(np.float16)
    slots = rng.choice(nb * B, size=T, replace=False).astype(np.int64)
    slots[[3, 17]] = -1  # padding tokens: no slot
    ek, ev = kp.copy(), vp.copy()
    ok = slots >= 0
    ek[slots[ok] // B, :, slots[ok] % B, :] = key[ok]
    ev[slots[ok] // B, :, slots[ok] % B, :] = val[ok]
    bad = orc.reshape_and_cache(kp.view(np.uint16), vp.view(np.uint16), key.view(np.uint16),
                                val.view(np.uint16), slots, orc.F16, orc.F16)
    assert bad == 0
    assert np.array_equal(kp.view(np.uint16), ek.view(np.uint16))
    assert np.array_equal(vp.view(np.uint16), ev.view(np.uint16))


def test_slot_write_out_of_range_is_skipped_and_counted():
    kp = np.zeros((4, 1, B, 8), np.float32)
    vp = np.zeros((4, 1, B, 8), np.float32)
    key = np.ones((3, 1, 8), np.float32)
    slots = np.array([5, 4 * B, 4 * B + 7], np.int64)
    bad = orc.reshape_and_cache(kp, vp, key, key, slots, orc.F32, orc.F32)
    assert bad == 2
    assert kp.sum() == 8 and kp[0, 0, 5].sum() == 8


def test_slot_write_fp8_matches_torch_cast_of_f32_quotient():
    rng = np.random.default_rng(2)
    nb, n_kv, d, T = 10, 2, 128, 40
    x = torch.from_numpy(rng.standard_normal((T, n_kv, d)).astype(np.float32) * 3)
    key = x.to(torch.bfloat16)
    val = (-x).to(torch.bfloat16)
    ks, vs = np.float32(0.0137), np.float32(0.0211)
    kp = np.zeros((nb, n_kv, B, d), np.uint8)
    vp = np.zeros((nb, n_kv, B, d), np.uint8)
    slots = rng.choice(nb * B, size=T, replace=False).astype(np.int64)
    orc.reshape_and_cache(kp, vp, key, val, slots, orc.BF16, orc.FP8_E4M3, ks, vs)
    # independent statement: float32 quotient, torch's RNE cast, clamp to +-448
    qk = (key.float() / torch.tensor(ks)).clamp(-448, 448)
    qv = (val.float() / torch.tensor(vs)).clamp(-448, 448)
    ek = qk.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ev = qv.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(kp[slots // B, :, slots % B, :], ek)
    assert np.array_equal(vp[slots // B, :, slots % B, :], ev)
    # some quotients really were beyond 448 and saturated
    assert (key.float().abs() / float(ks) > 448).any()


# ---------------------------------------------------------------------------
# copy_blocks
# ---------------------------------------------------------------------------

def test_copy_blocks_copies_bytes_and_nothing_else():
    rng = np.random.default_rng(3)
    kp = rng.integers(0, 256, size=(16, 8, B, 128), dtype=np.uint8)
    vp = rng.integers(0, 256, size=(16, 8, B, 128), dtype=np.uint8)
    k0, v0 = kp.copy(), vp.copy()
    pairs = np.array([[2, 9], [5, 11], [2, 14]], np.int64)
    assert orc.copy_blocks(kp, vp, pairs, orc.FP8_E4M3) == 0
    for s, t in pairs:
        assert np.array_equal(kp[t], k0[s]) and np.array_equal(vp[t], v0[s])
    others = [i for i in range(16) if i not in (9, 11, 14)]
    assert np.array_equal(kp[others], k0[others]) and np.array_equal(vp[others], v0[others])
    assert orc.copy_blocks(kp, vp, np.array([[0, 16], [-1, 3]], np.int64), orc.FP8_E4M3) == 2


def test_swap_blocks_moves_blocks_between_pools():
    # a preempted request's blocks go from the GPU pool to the host pool and
    # back ("vLLM explained", "KV cache 什麼時候可以被覆蓋": swap to the CPU)
    rng = np.random.default_rng(4)
    for dt, shape, np_dt in ((orc.BF16, (12, 4, B, 64), np.uint16),
                             (orc.FP8_E4M3, (12, 8, B, 128), np.uint8),
                             (orc.F32, (12, 2, B, 64), np.uint32)):
        gk = rng.integers(0, np.iinfo(np_dt).max, size=shape, dtype=np_dt)
        gv = rng.integers(0, np.iinfo(np_dt).max, size=shape, dtype=np_dt)
        hk = np.zeros((7,) + shape[1:], np_dt)
        hv = np.zeros_like(hk)
        out_pairs = np.array([[3, 0], [11, 6], [0, 2]], np.int64)
        assert orc.swap_blocks(hk, hv, gk, gv, out_pairs, dt) == 0
        for s, t in out_pairs:
            assert np.array_equal(hk[t], gk[s]) and np.array_equal(hv[t], gv[s])
        untouched = [i for i in range(7) if i not in (0, 6, 2)]
        assert not hk[untouched].any() and not hv[untouched].any()
        # back into other GPU blocks: the round trip is exact
        back = np.array([[0, 5], [6, 9], [2, 1]], np.int64)
        g0k, g0v = gk.copy(), gv.copy()
        assert orc.swap_blocks(gk, gv, hk, hv, back, dt) == 0
        for (s, _), (_, t) in zip(out_pairs, back):
            assert np.array_equal(gk[t], g0k[s]) and np.array_equal(gv[t], g0v[s])
        others = [i for i in range(12) if i not in (5, 9, 1)]
        assert np.array_equal(gk[others], g0k[others]) and np.array_equal(gv[others], g0v[others])
        # ids are checked against each pool's own size
        assert orc.swap_blocks(hk, hv, gk, gv, np.array([[11, 7], [12, 0], [0, -1]]), dt) == 3


# ---------------------------------------------------------------------------
# allocator model
# ---------------------------------------------------------------------------

def test_allocator_model_reproduces_worked_example():
    # "LLM inference optimization", Figure 1 / §三.1: Req1 -> P7, P2, P9 with P9
    # taken on demand; Req2 forks Req1 (shares P7) and then takes P5.
    rows = [l.split() for l in open(os.path.join(GOLDEN, "worked_block_table.txt"))
            if l.strip() and not l.startswith("#")]
    want = {}
    for req, lb, pb in rows:
        want.setdefault(req, []).append(int(pb))
    order = [7, 2, 9, 5] + [i for i in range(12) if i not in (7, 2, 9, 5)]
    m = AllocModel(12, B, order)
    st, slots = m.append("req1", 16)
    assert st == OK and slots == [7 * B + i for i in range(16)]
    assert m.fork("req1", "req2") == OK
    assert m.refcount(7) == 2
    assert m.append("req1", 32)[0] == OK        # fills P2, then P9 on demand
    assert m.append("req2", 16)[0] == OK        # next free block: P5
    assert m.block_table("req1") == want["req1"]
    assert m.block_table("req2") == want["req2"]
    assert [m.refcount(b) for b in (7, 2, 9, 5)] == [2, 1, 1, 1]
    assert m.num_free() == 8


def test_copy_on_write_only_on_divergent_write():
    # "LLM inference optimization", §三.2: branches point at the same block
    # with the count raised; only a branch that writes a different token copies.
    m = AllocModel(8, B)
    m.append(0, 20)                             # blocks 0 (full) and 1 (4 tokens)
    for c in (1, 2, 3):
        assert m.fork(0, c) == OK
    assert m.refcount(1) == 4 and m.refcount(0) == 4
    assert m.append(1, 1)[0] == INVALID_ARG     # shared partial block: CoW first
    pairs = []
    for s in (1, 2, 3):
        st, p = m.prepare_write(s)
        assert st == OK and len(p) == 1 and p[0][0] == 1
        pairs += p
    st, p = m.prepare_write(0)                  # last sharer writes in place
    assert st == OK and p == []
    assert [q[1] for q in pairs] == [2, 3, 4]
    assert m.refcount(1) == 1 and m.refcount(0) == 4
    st, slots = m.append(2, 1)
    assert st == OK and slots == [3 * B + 4]


def test_free_returns_blocks_only_at_refcount_zero_fifo():
    m = AllocModel(6, B)
    m.append("a", 33)                           # 0, 1, 2
    m.fork("a", "b")
    assert m.free_seq("a") == OK
    assert m.num_free() == 3 and m.free_list() == [3, 4, 5]
    assert m.free_seq("b") == OK
    # a finished request's blocks are released from its last block to its first
    assert m.free_list() == [3, 4, 5, 2, 1, 0]
    assert m.free_seq("b") == INVALID_ARG


def test_oom_is_all_or_nothing():
    m = AllocModel(4, B)
    m.append("a", 40)                           # 3 blocks
    before = (m.free_list(), list(m.rc), dict(m.tables), dict(m.ntok))
    st, slots = m.append("b", 17)               # needs 2, only 1 free
    assert st == OOM and slots == []
    assert (m.free_list(), list(m.rc), dict(m.tables), dict(m.ntok)) == before
    m.fork("a", "c")
    m.append("d", 16)                           # takes the last block
    st, p = m.prepare_write("c")                # CoW needs a block: none left
    assert st == OOM and m.block_table("c") == m.block_table("a")


def test_random_ops_keep_invariants():
    """Brute force: refcounts equal the number of tables holding a block, the
    free queue holds exactly the unreferenced blocks, every slot handed out
    names a block the sequence owns, and no block in use is handed out."""
    rnd = random.Random(7)
    N = 40
    m = AllocModel(N, B, rnd.sample(range(N), N))
    live = []
    nxt = 0
    for _ in range(3000):
        op = rnd.random()
        if op < 0.45 or not live:
            s = rnd.choice(live) if live and rnd.random() < 0.7 else nxt
            if s == nxt:
                nxt += 1
            used_before = {b for t in m.tables.values() for b in t}
            st, slots = m.append(s, rnd.randint(0, 40))
            if st == INVALID_ARG:
                st, p = m.prepare_write(s)
                continue
            if st == OK:
                if s not in live:
                    live.append(s)
                new = set(m.tables[s]) - used_before
                assert not (new & used_before)
                for sl in slots:
                    assert sl // B in m.tables[s]
        elif op < 0.6:
            c = nxt
            nxt += 1
            assert m.fork(rnd.choice(live), c) == OK
            live.append(c)
        elif op < 0.75:
            m.prepare_write(rnd.choice(live))
        else:
            s = rnd.choice(live)
            assert m.free_seq(s) == OK
            live.remove(s)
        counts = [0] * N
        for t in m.tables.values():
            for b in t:
                counts[b] += 1
        assert counts == m.rc
        assert sorted(m.free_list()) == [b for b in range(N) if counts[b] == 0]
        for s, t in m.tables.items():
            assert len(t) == -(-m.ntok[s] // B)
