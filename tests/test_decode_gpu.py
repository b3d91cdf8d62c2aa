"""GPU parity of pa_decode against the fp64 oracle on the same seeded inputs.

Sizes are chosen so the oracle finishes in seconds while the GPU path still
crosses many 16-token tiles, several context partitions (1024 tokens with
16-bit caches, 2048 with fp8 caches, so the reduce kernel runs) and a ragged
last block.  Full-size workloads are checked on a
sample of sequences in the launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

from pagedattention_paged_kv_pa_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding
    return binding


def _check(inp, dev, what, expect_err=0):
    gpu, err = P.run_decode(inp, dev)
    ref = P.oracle_decode(inp)
    assert err == expect_err, f"{what}: dev_err={err}"
    return P.assert_close(gpu, ref, inp.spec.q_dtype, inp.spec.kv_dtype, what)


def test_tiny_fp32_workload(B, cuda_device):
    inp = W.make_decode_inputs(W.TINY_FP32)
    _check(inp, cuda_device, "tiny fp32")


def test_llama2_7b_fp16_reduced(B, cuda_device):
    spec = W.LLAMA2_7B_FP16.scaled(num_seqs=8)
    _check(W.make_decode_inputs(spec), cuda_device, "llama2-7b fp16")


def test_llama3_70b_gqa_bf16_reduced(B, cuda_device):
    spec = W.LLAMA3_70B_GQA_BF16.scaled(num_seqs=12)
    ctx = np.array([16, 17, 1023, 1024, 1025, 1000, 2048, 3001, 4096, 5555, 8191, 8192], np.int32)
    _check(W.make_decode_inputs(spec, ctx=ctx), cuda_device, "llama3-70b bf16")


def test_fp8_cache_reduced(B, cuda_device):
    spec = W.MIXED_DECODE_FP8.scaled(num_seqs=10)
    _check(W.make_decode_inputs(spec), cuda_device, "fp8 kv")


@pytest.mark.parametrize("q_dt,kv_dt", [(W.F32, W.F32), (W.F16, W.F16), (W.BF16, W.BF16),
                                        (W.BF16, W.FP8_E4M3), (W.F16, W.FP8_E4M3)])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_dtype_group_headdim_grid(B, cuda_device, q_dt, kv_dt, d, G):
    n_kv = 2
    # 1100 spans two 1024-token partitions, 2049 two 2048-token (fp8) ones
    ctx = np.array([0, 1, 2, 3, 5, 10, 15, 16, 17, 33, 500, 1100, 2049], np.int32)
    spec = W.DecodeSpec("grid", len(ctx), n_kv * G, n_kv, d, q_dt, kv_dt, "fixed", (ctx,),
                        max_ctx=2304, pool_factor=1.3, seed=77 + G + d)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    _check(inp, cuda_device, f"q={q_dt} kv={kv_dt} d={d} G={G}")


def test_empty_context_rows_are_zero(B, cuda_device):
    ctx = np.array([0, 40, 0], np.int32)
    spec = W.DecodeSpec("empty", 3, 8, 2, 128, W.BF16, W.BF16, "fixed", (ctx,), max_ctx=1024)
    gpu, err = P.run_decode(W.make_decode_inputs(spec, ctx=ctx), cuda_device)
    assert err == 0
    assert np.all(gpu[0] == 0) and np.all(gpu[2] == 0) and np.any(gpu[1] != 0)


def test_permuting_physical_blocks_gives_identical_bits(B, cuda_device):
    spec = W.LLAMA3_70B_GQA_BF16.scaled(num_seqs=6)
    ctx = np.array([700, 16, 3000, 1025, 8000, 64], np.int32)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    out1, _ = P.run_decode(inp, cuda_device)
    g = torch.Generator().manual_seed(5)
    pi = torch.randperm(inp.num_blocks, generator=g)
    kp, vp = torch.empty_like(inp.k_pool), torch.empty_like(inp.v_pool)
    kp[pi] = inp.k_pool
    vp[pi] = inp.v_pool
    bt = inp.block_tables.clone()
    m = bt >= 0
    bt[m] = pi[bt[m].long()].to(torch.int32)
    inp2 = W.DecodeInputs(inp.spec, inp.q, kp, vp, bt, inp.context_lens, inp.scale, 1.0, 1.0)
    out2, _ = P.run_decode(inp2, cuda_device)
    assert np.array_equal(out1, out2)
    # and the same call twice is deterministic
    out3, _ = P.run_decode(inp2, cuda_device)
    assert np.array_equal(out2, out3)


def test_garbage_in_unused_slots_is_ignored(B, cuda_device):
    # the tail of a sequence's last block may hold anything, NaN bit patterns
    # included; masked tokens must not leak into the output
    for kv_dt, q_dt in ((W.BF16, W.BF16), (W.FP8_E4M3, W.BF16)):
        ctx = np.array([17, 530, 9], np.int32)
        spec = W.DecodeSpec("nan", 3, 8, 2, 128, q_dt, kv_dt, "fixed", (ctx,), max_ctx=1024,
                            pool_factor=1.5)
        inp = W.make_decode_inputs(spec, ctx=ctx)
        for s, c in enumerate(ctx):
            last = int(inp.block_tables[s, (c - 1) // 16])
            off = c % 16
            if off:
                if kv_dt == W.FP8_E4M3:
                    inp.k_pool[last, :, off:] = 0x7F
                    inp.v_pool[last, :, off:] = 0xFF
                else:
                    inp.k_pool[last, :, off:] = float("nan")
                    inp.v_pool[last, :, off:] = float("nan")
        _check(inp, cuda_device, f"garbage tail kv={kv_dt}")


def test_out_of_range_block_id_is_flagged_not_read(B, cuda_device):
    ctx = np.array([40, 40], np.int32)
    spec = W.DecodeSpec("badid", 2, 4, 2, 128, W.BF16, W.BF16, "fixed", (ctx,), max_ctx=64)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    inp.block_tables[1, 1] = inp.num_blocks + 1000
    gpu, err = P.run_decode(inp, cuda_device)
    assert err & 1  # PA_DEVERR_BLOCK_ID
    ref = P.oracle_decode(W.DecodeInputs(spec.scaled(num_seqs=1), inp.q[:1], inp.k_pool,
                                         inp.v_pool, inp.block_tables[:1],
                                         inp.context_lens[:1], inp.scale, 1.0, 1.0))
    P.assert_close(gpu[:1], ref, W.BF16, W.BF16, "healthy row next to a bad one")
    assert np.isfinite(gpu[1]).all()


@pytest.mark.parametrize("spec", [W.LLAMA2_7B_FP16, W.LLAMA3_70B_GQA_BF16,
                                  W.LLAMA3_70B_GQA_BF16_CTX8K, W.MIXED_DECODE_FP8],
                         ids=lambda s: s.name)
def test_full_size_sampled(B, cuda_device, spec):
    """Full-size workload in the benchmark's launch configuration; the oracle
    checks a sample of sequences (the longest, the shortest and random ones)."""
    inp = W.make_decode_inputs(spec, device=cuda_device)
    out = torch.empty_like(inp.q)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    B.pa_decode(out, inp.q, inp.k_pool, inp.v_pool, inp.block_tables, inp.context_lens,
                inp.scale, inp.k_scale, inp.v_scale, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    cl = inp.context_lens.cpu().numpy()
    rng = np.random.default_rng(0)
    pick = sorted({int(np.argmax(cl)), int(np.argmin(cl))} |
                  set(rng.choice(len(cl), size=4, replace=False).tolist()))
    sub = P.subset_for_oracle(inp, pick)
    ref = P.oracle_decode(sub)
    gpu = out[pick].float().cpu().numpy().astype(np.float64)
    P.assert_close(gpu, ref, spec.q_dtype, spec.kv_dtype, f"{spec.name} sampled")


@pytest.mark.parametrize("kv_dt", [W.BF16, W.FP8_E4M3])
def test_long_contexts_many_partitions(B, cuda_device, kv_dt):
    # 100,000 and 65,537 tokens: 98 / 65 partitions of 1024 tokens (16-bit) or
    # 49 / 33 of 2048 (fp8) -- more partitions than a warp has lanes for the
    # merge kernel to fold, and a ragged last block
    ctx = np.array([100_000, 65_537, 5], np.int32)
    spec = W.DecodeSpec("long", 3, 8, 2, 128, W.BF16, kv_dt, "fixed", (ctx,),
                        max_ctx=100_016, pool_factor=1.05, seed=91)
    _check(W.make_decode_inputs(spec, ctx=ctx), cuda_device, f"long contexts kv={kv_dt}")


def test_largest_batch(B, cuda_device):
    # 65,535 sequences (the grid's z limit), one kv head, contexts 0..40
    n = 65_535
    ctx = (np.arange(n) % 41).astype(np.int32)
    spec = W.DecodeSpec("wide", n, 2, 1, 64, W.BF16, W.BF16, "fixed", (ctx,), max_ctx=48,
                        pool_factor=1.0, seed=92)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    gpu, err = P.run_decode(inp, cuda_device)
    assert err == 0
    ref = P.oracle_decode(inp)
    P.assert_close(gpu, ref, W.BF16, W.BF16, "65,535 sequences")
    assert np.all(gpu[ctx == 0] == 0)
