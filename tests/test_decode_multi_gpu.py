"""GPU parity of pa_decode_multi (several new queries per sequence, as when a
target model verifies draft tokens in one pass) against the fp64 oracle.

Query i of a sequence with context c sits at position c - q_len + i and sees
keys 0 .. c - q_len + i: that is the oracle's causal chunk of q_len queries
over a history of c - q_len ("LLM inference optimization", §五; "Daily AI,
2026-07-31", 推測解碼).  When c < q_len the first q_len - c queries have no
keys and must come back as zero rows; the others form a chunk of c queries
over an empty history.  With head_dim 128 and group 1, 2, 4 or 8, bf16 or f16
queries over a cache of the same type run on the multi-query tensor-core kernel
(persistent CTAs with equal shares of the key tiles, split pairs merged), bf16
queries over an fp8 cache on the chunked-prefill tensor-core kernel; the other
cases on decode's partition and merge kernels.  All are held to the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from pagedattention_paged_kv_pa_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding
    return binding


def run_multi(B, inp, qm, device, dev_err=None):
    d = inp.to(device)
    q = qm.to(device)
    out = torch.empty_like(q)
    if dev_err is None:
        dev_err = torch.zeros(1, dtype=torch.int32, device=device)
    B.pa_decode_multi(out, q, d.k_pool, d.v_pool, d.block_tables, d.context_lens, d.scale,
                      d.k_scale, d.v_scale, dev_err=dev_err)
    torch.cuda.synchronize(device)
    return out.float().cpu().numpy().astype(np.float64), int(dev_err.item())


def oracle_multi(inp, qm):
    """[num_seqs, q_len, n_q, d] from the oracle's causal prefill, one chunk per
    sequence holding its queries at non-negative positions."""
    s = inp.spec
    ns, q_len, n_q, d = qm.shape
    ctx = inp.context_lens.cpu().numpy().astype(np.int64)
    ref = np.zeros((ns, q_len, n_q, d), np.float64)
    seqs, qs, qsl, cl = [], [], [0], []
    for i in range(ns):
        n = int(min(q_len, ctx[i]))  # queries with at least one key
        if n == 0:
            continue
        seqs.append(i)
        qs.append(qm[i, q_len - n:].cpu())
        qsl.append(qsl[-1] + n)
        cl.append(int(ctx[i]))      # history ctx - n plus the chunk of n
    if not seqs:
        return ref
    out = orc.paged_prefill(torch.cat(qs), inp.k_pool.cpu(), inp.v_pool.cpu(),
                            inp.block_tables[seqs].cpu(), np.array(qsl, np.int32),
                            np.array(cl, np.int32), inp.scale, s.q_dtype, s.kv_dtype,
                            inp.k_scale, inp.v_scale)
    for j, i in enumerate(seqs):
        n = qsl[j + 1] - qsl[j]
        ref[i, q_len - n:] = out[qsl[j]:qsl[j + 1]]
    return ref


def _check(B, inp, qm, device, what):
    gpu, err = run_multi(B, inp, qm, device)
    assert err == 0, f"{what}: dev_err={err}"
    ref = oracle_multi(inp, qm)
    return P.assert_close(gpu, ref, inp.spec.q_dtype, inp.spec.kv_dtype, what)


@pytest.mark.parametrize("q_dt,kv_dt", [(W.F16, W.F16), (W.BF16, W.BF16),
                                        (W.BF16, W.FP8_E4M3), (W.F16, W.FP8_E4M3)])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("q_len", [2, 5, 8])
def test_dtype_group_qlen_grid(B, cuda_device, q_dt, kv_dt, d, G, q_len):
    n_kv = 2
    # contexts shorter than q_len (queries without keys), block edges, and
    # two-partition contexts (1100: 1024-token partitions; 2049: fp8's 2048)
    ctx = np.array([0, 1, 3, 7, 15, 16, 17, 33, 500, 1100, 2049], np.int32)
    spec = W.DecodeSpec("mq", len(ctx), n_kv * G, n_kv, d, q_dt, kv_dt, "fixed", (ctx,),
                        max_ctx=2304, pool_factor=1.3, seed=300 + 10 * G + d + q_len)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    qm = W.make_multi_queries(inp, q_len, seed=400 + q_len)
    _check(B, inp, qm, cuda_device, f"q={q_dt} kv={kv_dt} d={d} G={G} q_len={q_len}")


def test_q_len_one_is_decode_bit_for_bit(B, cuda_device):
    spec = W.LLAMA3_70B_GQA_BF16.scaled(num_seqs=6)
    ctx = np.array([700, 16, 3000, 1025, 8000, 64], np.int32)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    one, err = run_multi(B, inp, inp.q[:, None], cuda_device)
    assert err == 0
    dec, err = P.run_decode(inp, cuda_device)
    assert err == 0
    assert np.array_equal(one[:, 0], dec)


def test_last_query_sees_the_whole_context(B, cuda_device):
    # the last of q_len queries attends to exactly what a decode query at the
    # same position would; the MMA column it occupies must not matter
    spec = W.LLAMA3_70B_GQA_BF16.scaled(num_seqs=5)
    ctx = np.array([40, 1024, 2500, 4097, 129], np.int32)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    qm = W.make_multi_queries(inp, 4, seed=9)
    multi, err = run_multi(B, inp, qm, cuda_device)
    assert err == 0
    last = W.DecodeInputs(inp.spec, qm[:, -1].contiguous(), inp.k_pool, inp.v_pool,
                          inp.block_tables, inp.context_lens, inp.scale, 1.0, 1.0)
    dec, err = P.run_decode(last, cuda_device)
    assert err == 0
    P.assert_close(multi[:, -1], dec, W.BF16, W.BF16, "last query vs decode")


def test_permuting_physical_blocks_gives_identical_bits(B, cuda_device):
    spec = W.MIXED_DECODE_FP8.scaled(num_seqs=6)
    ctx = np.array([700, 16, 3000, 2049, 8000, 5], np.int32)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    qm = W.make_multi_queries(inp, 6, seed=11)
    out1, _ = run_multi(B, inp, qm, cuda_device)
    g = torch.Generator().manual_seed(5)
    pi = torch.randperm(inp.num_blocks, generator=g)
    kp, vp = torch.empty_like(inp.k_pool), torch.empty_like(inp.v_pool)
    kp[pi] = inp.k_pool
    vp[pi] = inp.v_pool
    bt = inp.block_tables.clone()
    m = bt >= 0
    bt[m] = pi[bt[m].long()].to(torch.int32)
    inp2 = W.DecodeInputs(inp.spec, inp.q, kp, vp, bt, inp.context_lens, inp.scale,
                          inp.k_scale, inp.v_scale)
    out2, _ = run_multi(B, inp2, qm, cuda_device)
    assert np.array_equal(out1, out2)


def test_invalid_q_len_and_fp32_are_refused(B, cuda_device):
    spec = W.LLAMA3_70B_GQA_BF16.scaled(num_seqs=2)
    inp = W.make_decode_inputs(spec, ctx=np.array([32, 64], np.int32), device=cuda_device)
    for q_len in (9,):
        qm = W.make_multi_queries(inp, q_len, seed=1)
        with pytest.raises(B.PAError) as e:
            B.pa_decode_multi(torch.empty_like(qm), qm, inp.k_pool, inp.v_pool,
                              inp.block_tables, inp.context_lens, inp.scale)
        assert e.value.status == B.PA_ERR_INVALID_ARG
    tiny = W.make_decode_inputs(W.TINY_FP32, device=cuda_device)
    qm = W.make_multi_queries(tiny, 2, seed=1)
    with pytest.raises(B.PAError) as e:
        B.pa_decode_multi(torch.empty_like(qm), qm, tiny.k_pool, tiny.v_pool,
                          tiny.block_tables, tiny.context_lens, tiny.scale)
    assert e.value.status == B.PA_ERR_UNSUPPORTED


def test_full_size_spec_verify_sampled(B, cuda_device):
    """The draft-verification workload (Llama-3-70B GQA cache, 5 queries per
    sequence) in the benchmark's launch configuration; the oracle checks a
    sample of sequences (the longest, the shortest and random ones)."""
    spec, q_len = W.SPEC_VERIFY_BF16, W.SPEC_VERIFY_Q_LEN
    inp = W.make_decode_inputs(spec, device=cuda_device)
    qm = W.make_multi_queries(inp, q_len, seed=spec.seed + 1)
    out = torch.empty_like(qm)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    B.pa_decode_multi(out, qm, inp.k_pool, inp.v_pool, inp.block_tables, inp.context_lens,
                      inp.scale, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    cl = inp.context_lens.cpu().numpy()
    rng = np.random.default_rng(0)
    pick = sorted({int(np.argmax(cl)), int(np.argmin(cl))} |
                  set(rng.choice(len(cl), size=4, replace=False).tolist()))
    sub = P.subset_for_oracle(inp, pick)
    ref = oracle_multi(sub, qm[pick].cpu())
    gpu = out[pick].float().cpu().numpy().astype(np.float64)
    P.assert_close(gpu, ref, spec.q_dtype, spec.kv_dtype, "spec-verify sampled")


@pytest.mark.parametrize("dt", [W.BF16, W.F16])
def test_tensor_core_work_split(B, cuda_device, dt):
    """16-bit queries over a cache of the same type run on the multi-query
    kernel, whose persistent CTAs take equal shares of the key tiles: with this
    many sequences some (sequence, kv head) pairs are finished inside one CTA
    (one or several 1024-token partitions), others are split between CTAs and
    merged.  Every row is held to the oracle; the tails of the blocks the
    contexts end in hold NaN bit patterns, which must not reach the output, and
    empty contexts give zero rows."""
    rng = np.random.default_rng(77)
    ctx = rng.integers(1, 4200, size=24).astype(np.int32)
    ctx[:6] = (0, 3, 1024, 1025, 4096, 2049)
    spec = W.DecodeSpec("mq_split", len(ctx), 16, 4, 128, dt, dt, "fixed", (ctx,),
                        max_ctx=4224, pool_factor=1.2, seed=4242)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    for s, c in enumerate(ctx):
        if c % 16:
            last = int(inp.block_tables[s, (c - 1) // 16])
            inp.k_pool[last, :, c % 16:] = float("nan")
            inp.v_pool[last, :, c % 16:] = float("nan")
    qm = W.make_multi_queries(inp, 5, seed=78)
    _check(B, inp, qm, cuda_device, f"work split dt={dt}")
    # deterministic: the same call twice gives the same bits
    a, _ = run_multi(B, inp, qm, cuda_device)
    b, _ = run_multi(B, inp, qm, cuda_device)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("dt", [W.BF16, W.F16])
def test_tensor_core_bad_table_entries(B, cuda_device, dt):
    """On the multi-query kernel a block id outside the pool and a context
    longer than its table are flagged (PA_DEVERR_BLOCK_ID), never read, and
    leave the other sequences' rows as the oracle has them; the bad
    sequences' rows stay finite."""
    ctx = np.array([700, 1500, 300, 2100], np.int32)
    spec = W.DecodeSpec("mq_bad", len(ctx), 16, 4, 128, dt, dt, "fixed", (ctx,), max_ctx=2304,
                        pool_factor=1.2, seed=515)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    inp.block_tables[1, 50] = inp.num_blocks + 7           # inside sequence 1's context
    cl_bad = inp.context_lens.clone()
    cl_bad[3] = inp.block_tables.shape[1] * 16 + 40        # beyond sequence 3's table
    bad = W.DecodeInputs(inp.spec, inp.q, inp.k_pool, inp.v_pool, inp.block_tables, cl_bad,
                         inp.scale, inp.k_scale, inp.v_scale)
    qm = W.make_multi_queries(inp, 4, seed=516)
    gpu, err = run_multi(B, bad, qm, cuda_device)
    assert err & 1  # PA_DEVERR_BLOCK_ID
    assert np.isfinite(gpu).all()
    good = [0, 2]
    ref = oracle_multi(P.subset_for_oracle(inp, good), qm[good].cpu())
    P.assert_close(gpu[good], ref, dt, dt, "healthy sequences next to bad ones")


def test_tensor_core_many_sequences(B, cuda_device):
    """A batch of 1,000 short sequences (not a multiple of the 32 or 128 the
    kernel's share search takes at a time; a tenth of them empty) on the
    multi-query kernel: every row against the oracle."""
    rng = np.random.default_rng(1000)
    ctx = rng.integers(1, 600, size=1000).astype(np.int32)
    ctx[rng.choice(1000, size=100, replace=False)] = 0
    spec = W.DecodeSpec("mq_many", len(ctx), 8, 2, 128, W.BF16, W.BF16, "fixed", (ctx,),
                        max_ctx=640, pool_factor=1.1, seed=1001)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    qm = W.make_multi_queries(inp, 3, seed=1002)
    _check(B, inp, qm, cuda_device, "1,000 sequences")
