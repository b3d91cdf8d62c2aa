"""The numerators of bench.py's throughput figures, checked by brute force on
tiny cases and against the full-size figures worked out by hand."""
import types

import numpy as np
import torch

import bench
from pagedattention_paged_kv_pa_b200 import workloads as W


def _prefill(chunk_lens, histories, n_q=32, d=128):
    qsl = np.concatenate([[0], np.cumsum(chunk_lens)]).astype(np.int32)
    cl = np.asarray(histories, np.int32) + np.asarray(chunk_lens, np.int32)
    spec = types.SimpleNamespace(head_dim=d, n_q_heads=n_q)
    return types.SimpleNamespace(spec=spec, query_start_loc=torch.from_numpy(qsl),
                                 context_lens=torch.from_numpy(cl))


def test_prefill_flops_count_visible_pairs():
    chunk_lens, histories = [3, 0, 2, 5], [4, 5, 0, 17]
    pairs = sum(h + i + 1 for h, L in zip(histories, chunk_lens) for i in range(L))
    # two products (QK^T and PV), each 2 flop per element of d, per q head
    assert bench.prefill_causal_flops(_prefill(chunk_lens, histories)) == 4 * 128 * 32 * pairs


def test_prefill_flops_mixed_step():
    # 2 chunks x 512 queries over 4096-token histories: 2,228,480 visible
    # (query, key) pairs per chunk -> 7.302e10 flop for 32 q heads, d = 128
    inp = _prefill([512, 512], [4096, 4096])
    assert bench.prefill_causal_flops(inp) == 4 * 128 * 32 * 2 * 2_228_480 == 73_022_832_640


def test_decode_bytes_brute_force():
    ctx = np.array([0, 1, 17, 300], np.int64)
    n_q, n_kv, d = 8, 2, 64
    kv = sum(int(c) * n_kv * d * 2 * 1 for c in ctx)        # K and V, 1-byte codes
    qo = len(ctx) * n_q * d * (2 + 2)                        # bf16 q in, bf16 out
    assert W.decode_algorithmic_bytes(ctx, n_q, n_kv, d, 2, 1) == kv + qo
    assert W.decode_algorithmic_bytes(ctx, n_q, n_kv, d, 2, 1, out_elem=4) == kv + len(ctx) * n_q * d * 6


def test_decode_bytes_llama3_workload():
    # the Llama-3-70B GQA layer as generated: 269,902 context tokens over 128
    # sequences, 8 kv / 64 q heads, d = 128, bf16
    spec = W.LLAMA3_70B_GQA_BF16
    ctx = W.context_lens_for(spec, W._rng(spec.seed))
    assert int(np.sum(ctx)) == 269_902
    assert W.decode_algorithmic_bytes(ctx, 64, 8, 128, 2, 2) == 1_109_712_896
