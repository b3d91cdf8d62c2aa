"""Helpers for the GPU parity tests: run the CUDA path through the C ABI, run
the oracle on the same bytes, and compare within the stated tolerances.

Tolerances (per element, against the fp64 oracle on the same stored inputs):
  fp32 inputs          |gpu - ref| <= 1e-5
  fp16 / bf16 inputs   |gpu - ref| <= 2e-3 + 1e-2 |ref|
  fp8-e4m3 KV          |gpu - ref| <= 3e-2
The 16-bit rule is the allclose reading of "abs <= 2e-3, rel <= 1e-2": the
output itself is rounded to bf16 (half an ulp is 3.9e-3 for |out| in [1, 2)),
so an absolute bound alone cannot hold for large outputs and a relative bound
alone cannot hold near zero.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
from pagedattention_paged_kv_pa_b200 import workloads as W

TOL = {W.F32: (1e-5, 0.0), W.F16: (2e-3, 1e-2), W.BF16: (2e-3, 1e-2)}
FP8_ATOL = 3e-2


def tolerance(q_dtype: int, kv_dtype: int):
    if kv_dtype == W.FP8_E4M3:
        return FP8_ATOL, 0.0
    return TOL[q_dtype]


def assert_close(gpu: np.ndarray, ref: np.ndarray, q_dtype: int, kv_dtype: int, what=""):
    atol, rtol = tolerance(q_dtype, kv_dtype)
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    err = np.abs(gpu - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} elements out of tolerance; "
                             f"worst at {i}: gpu={gpu[i]!r} ref={ref[i]!r} "
                             f"max_abs={err.max():.3e}")
    return float(err.max())


def run_decode(inp: W.DecodeInputs, device, dev_err=None):
    from pagedattention_paged_kv_pa_b200 import binding as B
    d = inp.to(device)
    out = torch.empty_like(d.q)
    if dev_err is None:
        dev_err = torch.zeros(1, dtype=torch.int32, device=device)
    B.pa_decode(out, d.q, d.k_pool, d.v_pool, d.block_tables, d.context_lens, d.scale,
                d.k_scale, d.v_scale, dev_err=dev_err)
    torch.cuda.synchronize(device)
    return out.float().cpu().numpy().astype(np.float64), int(dev_err.item())


def oracle_decode(inp: W.DecodeInputs, nthreads=None):
    s = inp.spec
    return orc.paged_decode(inp.q.cpu(), inp.k_pool.cpu(), inp.v_pool.cpu(),
                            inp.block_tables.cpu(), inp.context_lens.cpu(), inp.scale,
                            s.q_dtype, s.kv_dtype, inp.k_scale, inp.v_scale, nthreads)


def subset_for_oracle(inp: W.DecodeInputs, seqs) -> W.DecodeInputs:
    """The listed sequences with a compact pool holding only their blocks.

    Block ids are relabelled (a permutation-free renumbering), which the
    attention result does not depend on."""
    bt = inp.block_tables[seqs].cpu().numpy()
    cl = inp.context_lens[seqs].cpu().numpy()
    need = [-(-int(c) // 16) for c in cl]
    used = sorted({int(b) for r, n in zip(bt, need) for b in r[:n]})
    remap = {b: i for i, b in enumerate(used)}
    bt2 = np.full_like(bt, -1)
    for r, (row, n) in enumerate(zip(bt, need)):
        bt2[r, :n] = [remap[int(b)] for b in row[:n]]
    idx = torch.tensor(used, dtype=torch.long, device=inp.k_pool.device)
    spec = inp.spec.scaled(num_seqs=len(seqs))
    return W.DecodeInputs(spec, inp.q[seqs].cpu(), inp.k_pool[idx].cpu(), inp.v_pool[idx].cpu(),
                          torch.from_numpy(bt2), torch.from_numpy(cl), inp.scale, inp.k_scale,
                          inp.v_scale)
