"""End-to-end flows through the whole path, GPU against oracle.

Shared-prefix parallel sampling: 16 prompts x 4 samples, bf16, 32 q / 8 kv
heads.  Each prompt (2048 + U{1..15} tokens, so its last block is partial) is
written once and forked to its 4 samples (reference count 4).  Each sample
then writes 0-512 divergent tokens; the first divergent write into the shared
partial block copies it first (copy-on-write: "LLM inference optimization",
§三.2), the last sharer writes in place.  Then every sequence decodes.

GPU side: the C++ allocator, pa_copy_blocks, pa_reshape_and_cache, pa_decode.
Oracle side: the Python allocator model, the oracle's block copy, slot write
and decode.  Checked: identical allocator state, bit-identical pools after
the writes, decode within tolerance, and -- the page's claim that sharing
changes nothing -- the oracle's output on the shared pool equal, bit for bit,
to its output on private per-sequence copies.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from oracle.alloc_model import AllocModel
from pagedattention_paged_kv_pa_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

N_PROMPTS, N_SAMPLES, N_Q, N_KV, D = 16, 4, 32, 8, 128


def _raw16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def test_shared_prefix_copy_on_write_flow(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding as B
    dev = cuda_device
    rng = np.random.default_rng(1004)
    prompt_len = 2048 + rng.integers(1, 16, size=N_PROMPTS)
    div = rng.integers(0, 513, size=(N_PROMPTS, N_SAMPLES))
    seqs = [(p, s) for p in range(N_PROMPTS) for s in range(N_SAMPLES)]
    sid = {ps: i for i, ps in enumerate(seqs)}
    need = int(sum(-(-int(l) // 16) for l in prompt_len) +
               sum(-(-int(d) // 16) + 1 for d in div.ravel()))
    num_blocks = need + 16
    order = np.random.default_rng(7).permutation(num_blocks).tolist()
    alloc = B.BlockAllocator(num_blocks, 16, order)
    model = AllocModel(num_blocks, 16, order)

    gen = torch.Generator().manual_seed(1004)
    pool_shape = (num_blocks, N_KV, 16, D)
    k_pool = torch.randn(pool_shape, generator=gen).to(torch.bfloat16)
    v_pool = torch.randn(pool_shape, generator=gen).to(torch.bfloat16)
    kd, vd = k_pool.to(dev), v_pool.to(dev)
    ko, vo = _raw16(k_pool).copy(), _raw16(v_pool).copy()
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def write(slots, key, val):
        s = torch.tensor(slots, dtype=torch.int64)
        B.pa_reshape_and_cache(kd, vd, key.to(dev), val.to(dev), s.to(dev), dev_err=err)
        orc.reshape_and_cache(ko, vo, key, val, s, W.BF16, W.BF16)

    # prompts: written once, then forked to the samples
    for p in range(N_PROMPTS):
        s0 = sid[(p, 0)]
        st, slots = alloc.append(s0, int(prompt_len[p]))
        st_m, slots_m = model.append(s0, int(prompt_len[p]))
        assert st == st_m == 0 and slots == slots_m
        key, val = W.make_new_kv(len(slots), N_KV, D, W.BF16, "cpu", seed=5000 + p)
        write(slots, key, val)
        for s in range(1, N_SAMPLES):
            assert alloc.fork(s0, sid[(p, s)]) == model.fork(s0, sid[(p, s)]) == 0
    last = [alloc.block_table(sid[(p, 0)])[-1] for p in range(N_PROMPTS)]
    assert all(alloc.refcount(b) == N_SAMPLES for b in last)

    # divergent tokens: copy-on-write of the shared partial block first
    n_pairs = 0
    for p in range(N_PROMPTS):
        for s in range(N_SAMPLES):
            q = sid[(p, s)]
            n = int(div[p, s])
            if n == 0:
                continue
            st, pairs = alloc.prepare_write(q)
            st_m, pairs_m = model.prepare_write(q)
            assert st == st_m == 0 and pairs == pairs_m
            if pairs:
                pr = torch.tensor(pairs, dtype=torch.int64)
                B.pa_copy_blocks(kd, vd, pr.to(dev), dev_err=err)
                orc.copy_blocks(ko, vo, pr.numpy(), W.BF16)
                n_pairs += 1
            st, slots = alloc.append(q, n)
            st_m, slots_m = model.append(q, n)
            assert st == st_m == 0 and slots == slots_m
            key, val = W.make_new_kv(n, N_KV, D, W.BF16, "cpu", seed=9000 + q)
            write(slots, key, val)
    assert n_pairs > 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # allocator state and pools agree bit for bit
    assert alloc.free_list() == model.free_list()
    assert [alloc.refcount(b) for b in range(num_blocks)] == model.rc
    assert np.array_equal(_raw16(kd), ko) and np.array_equal(_raw16(vd), vo)

    # decode every sequence
    ctx = np.array([model.num_tokens(i) for i in range(len(seqs))], np.int32)
    max_blocks = int(-(-ctx.max() // 16))
    bt = np.full((len(seqs), max_blocks), -1, np.int32)
    for i in range(len(seqs)):
        t = model.block_table(i)
        bt[i, :len(t)] = t
    q = torch.randn(len(seqs), N_Q, D, generator=gen).to(torch.bfloat16)
    out = torch.empty_like(q, device=dev)
    B.pa_decode(out, q.to(dev), kd, vd, torch.from_numpy(bt).to(dev),
                torch.from_numpy(ctx).to(dev), 1 / np.sqrt(D), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    scale = 1 / np.sqrt(D)
    ref = orc.paged_decode(q, ko, vo, bt, ctx, scale, W.BF16, W.BF16)
    P.assert_close(out.float().cpu().numpy(), ref, W.BF16, W.BF16, "shared-prefix decode")

    # sharing changes nothing: private copies of every sequence's blocks
    used = [b for row, c in zip(bt, ctx) for b in row[:-(-int(c) // 16)]]
    kp2 = np.empty((len(used),) + ko.shape[1:], ko.dtype)
    vp2 = np.empty_like(kp2)
    bt2 = np.full_like(bt, -1)
    pos = 0
    for i, (row, c) in enumerate(zip(bt, ctx)):
        n = -(-int(c) // 16)
        kp2[pos:pos + n] = ko[row[:n]]
        vp2[pos:pos + n] = vo[row[:n]]
        bt2[i, :n] = np.arange(pos, pos + n)
        pos += n
    ref_private = orc.paged_decode(q, kp2, vp2, bt2, ctx, scale, W.BF16, W.BF16)
    assert np.array_equal(ref, ref_private)


def test_preemption_by_swap_keeps_decode_bits(cuda_device):
    """Sequences are preempted by swapping their blocks to a pinned host pool
    ("vLLM explained", "KV cache 什麼時候可以被覆蓋": swap to the CPU when
    memory runs short); new sequences take and overwrite the freed GPU blocks;
    the preempted ones are swapped back into other GPU blocks and decode to
    the same bits as before (attention depends only on logical contents)."""
    from pagedattention_paged_kv_pa_b200 import binding as B
    dev = cuda_device
    n_q, n_kv, d = 32, 8, 128
    gpu = B.BlockAllocator(120, 16)
    cpu = B.BlockAllocator(96, 16)
    gen = torch.Generator(device="cpu").manual_seed(77)
    shape = (120, n_kv, 16, d)
    kp = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    vp = torch.zeros_like(kp)
    hk = torch.zeros((96, n_kv, 16, d), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    lens = [300, 17, 640, 129, 500, 64]

    def write(alloc, seq, n, seed):
        st, slots = alloc.append(seq, n)
        assert st == 0
        key, val = W.make_new_kv(n, n_kv, d, W.BF16, dev, seed=seed)
        B.pa_reshape_and_cache(kp, vp, key, val, torch.tensor(slots, device=dev), dev_err=err)

    for s, n in enumerate(lens):
        write(gpu, s, n, 100 + s)
    q = torch.randn(len(lens), n_q, d, generator=gen).to(torch.bfloat16).to(dev)

    def decode(seqs):
        mb = 48
        bt = torch.full((len(seqs), mb), -1, dtype=torch.int32)
        for r, s in enumerate(seqs):
            t = gpu.block_table(s)
            bt[r, :len(t)] = torch.tensor(t, dtype=torch.int32)
        cl = torch.tensor([gpu.num_tokens(s) for s in seqs], dtype=torch.int32)
        out = torch.empty(len(seqs), n_q, d, dtype=torch.bfloat16, device=dev)
        B.pa_decode(out, q[seqs], kp, vp, bt.to(dev), cl.to(dev), 1 / np.sqrt(d), dev_err=err)
        return out

    before = decode(list(range(len(lens))))
    # preempt sequences 0, 2, 4: host blocks for their tokens, copy out, free on the GPU
    swapped = [0, 2, 4]
    old_tables = {s: gpu.block_table(s) for s in swapped}
    pairs = []
    for s in swapped:
        st, _ = cpu.append(s, gpu.num_tokens(s))
        assert st == 0
        pairs += list(zip(gpu.block_table(s), cpu.block_table(s)))
    B.pa_swap_blocks(hk, hv, kp, vp, torch.tensor(pairs, dtype=torch.int64, device=dev),
                     dev_err=err)
    for s in swapped:
        assert gpu.free_seq(s) == 0
    # new sequences take the never-used blocks, then freed ones, overwriting
    # them; they finish before the preempted sequences come back
    reused = set()
    for s in range(10, 14):
        write(gpu, s, 200, 200 + s)
        reused |= set(gpu.block_table(s))
    assert reused & {b for t in old_tables.values() for b in t}
    for s in range(10, 14):
        assert gpu.free_seq(s) == 0
    # swap the preempted sequences back in, into whatever blocks are free now
    pairs = []
    for s in swapped:
        st, _ = gpu.append(s, cpu.num_tokens(s))
        assert st == 0
        pairs += list(zip(cpu.block_table(s), gpu.block_table(s)))
        assert cpu.free_seq(s) == 0
    B.pa_swap_blocks(kp, vp, hk, hv, torch.tensor(pairs, dtype=torch.int64).pin_memory(),
                     dev_err=err)
    after = decode(swapped)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert any(gpu.block_table(s) != old_tables[s] for s in swapped)
    assert torch.equal(after, before[swapped])
