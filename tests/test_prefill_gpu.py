"""GPU parity of pa_prefill_paged (tcgen05 chunked prefill) against the oracle.

Small chunks are compared in full with the oracle's causal prefill; the
full-size mixed-step prefill (2 chunks x 512 queries over a 4096-token paged
history, fp8 cache) is compared on sampled (query, head) rows, each of which
the oracle computes as attention over that query's causal prefix.  Every case
runs both ways the call can go: without a workspace and with one.  With an
fp8 cache these are two kernels (each query tile widening the K/V it reads,
or the history widened once per chunk and kv head into the workspace) that
feed the tensor cores the same f16 K and V; the workspace kernel splits each
row's softmax over several warps, each deciding per part of a tile whether
masking is needed, so an exponent argument may come from one fused
multiply-add instead of a multiply and an add (flipping the f16 rounding of
that P now and then), and it adds the row sum in parts.  The two fp8 paths
therefore agree to a bound far inside the oracle tolerance, not bit for bit.
With a bf16 cache both calls run the same kernel (bf16 operands straight from
the pool; the workspace is not used) and agree bit for bit.
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


def _run(B, inp, dev, max_chunk_len, staged=False):
    d = dict(q=inp.q.to(dev), k=inp.k_pool.to(dev), v=inp.v_pool.to(dev),
             bt=inp.block_tables.to(dev), qsl=inp.query_start_loc.to(dev),
             cl=inp.context_lens.to(dev))
    out = torch.full_like(d["q"], float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = None
    if staged:  # poisoned, so rows the widening pass should write but skips show up
        ws = B.alloc_prefill_workspace(d["k"], d["bt"]).fill_(0xFF)
    B.pa_prefill_paged(out, d["q"], d["k"], d["v"], d["bt"], d["qsl"], d["cl"], inp.scale,
                       max_chunk_len, inp.k_scale, inp.v_scale, workspace=ws, dev_err=err)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), int(err.item())


def _paths_agree(a, b):
    """The two paths' outputs (bf16 values as float64): within one bf16 ulp
    plus 2^-12 (a P that rounds to the neighbouring f16 moves an output by
    far less), and mostly identical."""
    assert np.isfinite(a).all() and np.isfinite(b).all()
    assert (np.abs(a - b) <= np.abs(a) * 2.0 ** -7 + 2.0 ** -12).all()
    assert np.mean(a == b) > 0.5


def _oracle(inp):
    s = inp.spec
    return orc.paged_prefill(inp.q.cpu(), inp.k_pool.cpu(), inp.v_pool.cpu(),
                             inp.block_tables.cpu(), inp.query_start_loc.cpu(),
                             inp.context_lens.cpu(), inp.scale, s.q_dtype, s.kv_dtype,
                             inp.k_scale, inp.v_scale)


@pytest.mark.parametrize("staged", [False, True])
@pytest.mark.parametrize("kv_dt", [W.FP8_E4M3, W.BF16])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_small_chunks_against_oracle(B, cuda_device, kv_dt, G, staged):
    n_kv = 2
    spec = W.PrefillSpec("small", 3, 0, 0, n_kv * G, n_kv, 128, W.BF16, kv_dt, extra_blocks=5,
                         seed=300 + G)
    chunk_lens = [37, 130, 1]
    histories = [0, 291, 1000]
    inp = W.make_prefill_inputs(spec, chunk_lens=chunk_lens, histories=histories)
    gpu, err = _run(B, inp, cuda_device, max(chunk_lens), staged)
    assert err == 0
    P.assert_close(gpu, _oracle(inp), W.BF16, kv_dt, f"prefill G={G} kv={kv_dt}")


@pytest.mark.parametrize("staged", [False, True])
def test_history_zero_single_chunk_is_causal_self_attention(B, cuda_device, staged):
    spec = W.PrefillSpec("h0", 1, 200, 0, 32, 8, 128, W.BF16, W.BF16, seed=311)
    inp = W.make_prefill_inputs(spec)
    gpu, err = _run(B, inp, cuda_device, 200, staged)
    assert err == 0
    P.assert_close(gpu, _oracle(inp), W.BF16, W.BF16, "prefill H=0")


@pytest.mark.parametrize("staged", [False, True])
def test_chunk_lengths_at_tile_edges(B, cuda_device, staged):
    # G=4 packs 32 queries per CTA tile; keys come in tiles of 128
    spec = W.PrefillSpec("edges", 4, 0, 0, 32, 8, 128, W.BF16, W.FP8_E4M3, seed=312)
    chunk_lens = [32, 33, 64, 31]
    histories = [128, 127, 129, 16]
    inp = W.make_prefill_inputs(spec, chunk_lens=chunk_lens, histories=histories)
    gpu, err = _run(B, inp, cuda_device, 64, staged)
    assert err == 0
    P.assert_close(gpu, _oracle(inp), W.BF16, W.FP8_E4M3, "prefill tile edges")


@pytest.mark.parametrize("staged", [False, True])
def test_empty_chunks_between_others(B, cuda_device, staged):
    # a chunk with no queries (its history is still widened, nothing is
    # written), and an empty sequence (no history, no queries) at the end
    spec = W.PrefillSpec("empty", 4, 0, 0, 32, 8, 128, W.BF16, W.FP8_E4M3, seed=315)
    inp = W.make_prefill_inputs(spec, chunk_lens=[20, 0, 33, 0], histories=[100, 50, 0, 0])
    gpu, err = _run(B, inp, cuda_device, 33, staged)
    assert err == 0
    P.assert_close(gpu, _oracle(inp), W.BF16, W.FP8_E4M3, "prefill with empty chunks")


@pytest.mark.parametrize("staged", [False, True])
def test_long_chunk_many_query_tiles(B, cuda_device, staged):
    # 700 queries = 21 full query tiles of 32 (G = 4) and a ragged one, over
    # 1,033 keys (8 full key tiles and a ragged one)
    spec = W.PrefillSpec("long", 1, 0, 0, 32, 8, 128, W.BF16, W.BF16, seed=316)
    inp = W.make_prefill_inputs(spec, chunk_lens=[700], histories=[333])
    gpu, err = _run(B, inp, cuda_device, 700, staged)
    assert err == 0
    P.assert_close(gpu, _oracle(inp), W.BF16, W.BF16, "prefill, one long chunk")


@pytest.mark.parametrize("kv_dt", [W.FP8_E4M3, W.BF16])
def test_workspace_and_in_kernel_widening_agree(B, cuda_device, kv_dt):
    # contexts ending inside a block, on a 128-key tile edge and one past it
    spec = W.PrefillSpec("agree", 4, 0, 0, 16, 4, 128, W.BF16, kv_dt, extra_blocks=3, seed=313)
    chunk_lens = [100, 7, 128, 1]
    histories = [1333, 121, 0, 128]
    inp = W.make_prefill_inputs(spec, chunk_lens=chunk_lens, histories=histories)
    a, ea = _run(B, inp, cuda_device, 128, staged=False)
    b, eb = _run(B, inp, cuda_device, 128, staged=True)
    assert ea == eb == 0
    _paths_agree(a, b)


def test_out_of_range_block_id_is_flagged_on_both_paths(B, cuda_device):
    spec = W.PrefillSpec("badid", 2, 0, 0, 8, 2, 128, W.BF16, W.FP8_E4M3, seed=314)
    inp = W.make_prefill_inputs(spec, chunk_lens=[40, 20], histories=[300, 50])
    bt = inp.block_tables.clone()
    bt[0, 3] = inp.k_pool.shape[0] + 7  # keys 48..63 of chunk 0
    inp = W.PrefillInputs(inp.spec, inp.q, inp.k_pool, inp.v_pool, bt, inp.query_start_loc,
                          inp.context_lens, inp.scale, inp.k_scale, inp.v_scale)
    a, ea = _run(B, inp, cuda_device, 40, staged=False)
    b, eb = _run(B, inp, cuda_device, 40, staged=True)
    assert ea & 1 and eb & 1  # PA_DEVERR_BLOCK_ID
    assert np.isfinite(b).all()
    _paths_agree(a, b)


@pytest.mark.parametrize("staged", [False, True])
def test_mixed_step_prefill_full_size_sampled(B, cuda_device, staged):
    """2 chunks x 512 queries over a 4096-token history, 32 q / 8 kv heads,
    fp8 cache, in the launch configuration the mixed-step benchmark uses.
    Sampled rows: query i of chunk c equals decode attention over the first
    H + i + 1 keys of that chunk's sequence."""
    spec = W.MIXED_PREFILL_FP8
    inp = W.make_prefill_inputs(spec, device=cuda_device)
    gpu, err = _run(B, inp, cuda_device, spec.chunk_len, staged)
    assert err == 0
    rng = np.random.default_rng(1)
    qsl = inp.query_start_loc.cpu().numpy()
    cl = inp.context_lens.cpu().numpy()
    picks = [(c, i) for c in range(spec.n_chunks)
             for i in sorted(set(rng.choice(spec.chunk_len, 6, replace=False).tolist()) | {0, spec.chunk_len - 1})]
    rows = [qsl[c] + i for c, i in picks]
    ctx = np.array([cl[c] - spec.chunk_len + i + 1 for c, i in picks], np.int32)
    bt = inp.block_tables.cpu()[[c for c, _ in picks]]
    dec = W.DecodeInputs(W.MIXED_DECODE_FP8.scaled(num_seqs=len(rows)), inp.q[rows], inp.k_pool,
                         inp.v_pool, bt, torch.from_numpy(ctx), inp.scale, inp.k_scale,
                         inp.v_scale)
    sub = P.subset_for_oracle(dec, list(range(len(rows))))
    ref = P.oracle_decode(sub)
    P.assert_close(gpu[rows], ref, W.BF16, W.FP8_E4M3, "mixed-step prefill sampled")
    assert np.isfinite(gpu).all()
