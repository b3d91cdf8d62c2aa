"""Parity over the whole bf16 range.

Paging leaves the attention result unchanged ("vLLM explained", "兩層實作"), so
bf16 queries, keys and values far outside f16's range (|x| of 1e5 and more)
or deep in its subnormal range (1e-6) must give the oracle's result on every
path: chunked prefill with a bf16 cache (bf16 tensor-core operands) and with
an fp8 cache (E4M3 widened to f16, each bf16 query row scaled into f16's range
by a power of two), decode with either cache, and multi-query decode (its
tcgen05 kernel with a bf16 cache, the prefill kernel with an fp8 cache).

Three kinds of input, all on top of the usual seeded N(0,1) draws:
  * powers of two that cancel in the scores (q x 2^-a with k x 2^a, or with
    the fp8 k_scale x 2^a): the oracle's result is unchanged, and any operand
    rounded to f16 on the way would overflow or lose its low bits;
  * V scaled by 2^17 or 2^-20: the output scales with it, so the result is
    compared after dividing both sides by the same power of two (exact);
  * sparse planted values of +-1e5, +-3e4 and +-1e-6.  Query plants sit in
    dims where every key entry is zero and key plants in dims where every
    query entry is zero, so every planted value passes through the products
    (0 x 1e5 must stay 0, not become 0 x inf) while the scores stay those of
    the ordinary entries: a score of 1e5-sized products carries an fp32
    rounding of ~1e-2, and near-tied keys then move an output by more than
    2e-3 in any fp32-accumulating implementation, against an fp64 oracle.
    Value plants are checked with an extra 2^-14 of the weighted average of
    |V| (the oracle run on |V|): the forward-error bound of a weighted sum is
    relative to the magnitude of its terms, and 2^-14 of it is still 2^5
    times finer than a bf16 ulp.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as orc
from pagedattention_paged_kv_pa_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

PLANTS = (1e5, -1e5, 3e4, -3e4, 1e-6, -1e-6)


@pytest.fixture(scope="module")
def B(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding
    return binding


def _times(t, f):
    """t x f for a power of two f (exact in bf16 at these magnitudes)."""
    return (t.float() * f).to(t.dtype)


def _plant(t, dims, density, seed, zero_dims=()):
    """Copy of bf16 tensor t with a seeded fraction of the entries in the
    last-axis `dims` replaced by values from PLANTS, and `zero_dims` zeroed."""
    rng = np.random.default_rng(seed)
    x = t.float().numpy().copy()
    mask = rng.random(x.shape) < density
    keep = np.zeros(x.shape[-1], bool)
    keep[list(dims)] = True
    mask &= keep
    x[mask] = rng.choice(PLANTS, size=int(mask.sum()))
    if zero_dims:
        x[..., list(zero_dims)] = 0.0
    return torch.from_numpy(x).to(t.dtype)


Q_PLANT_DIMS = range(112, 120)  # every key entry zero
K_PLANT_DIMS = range(120, 128)  # every query entry zero


def _plant_qk(inp, seed):
    """Queries planted in Q_PLANT_DIMS (zero in K_PLANT_DIMS); bf16 keys
    planted in K_PLANT_DIMS, fp8 keys left as drawn; both zero where the
    other is planted."""
    q = _plant(inp.q, Q_PLANT_DIMS, 0.05, seed, zero_dims=K_PLANT_DIMS)
    if inp.k_pool.dtype == torch.uint8:  # E4M3 code 0 is +0
        k = inp.k_pool.clone()
        k[..., list(Q_PLANT_DIMS)] = 0
    else:
        k = _plant(inp.k_pool, K_PLANT_DIMS, 0.05, seed + 1, zero_dims=Q_PLANT_DIMS)
    return dataclasses.replace(inp, q=q, k_pool=k)


def _assert_close_mag(gpu, ref, ref_mag, what):
    """bf16 bound plus 2^-14 of the weighted average of |V| (see above)."""
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    err = np.abs(gpu - ref)
    bound = 2e-3 + 1e-2 * np.abs(ref) + 2.0 ** -14 * ref_mag
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {err.size} out of tolerance; worst "
                           f"excess {(err - bound).max():.3e}, max_abs {err.max():.3e}")


# ------------------------------------------------------------------ prefill

def _prefill(B, inp, dev, staged):
    d = dict(q=inp.q.to(dev), k=inp.k_pool.to(dev), v=inp.v_pool.to(dev),
             bt=inp.block_tables.to(dev), qsl=inp.query_start_loc.to(dev),
             cl=inp.context_lens.to(dev))
    out = torch.full_like(d["q"], float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = B.alloc_prefill_workspace(d["k"], d["bt"]).fill_(0xFF) if staged else None
    max_len = int((inp.query_start_loc[1:] - inp.query_start_loc[:-1]).max())
    B.pa_prefill_paged(out, d["q"], d["k"], d["v"], d["bt"], d["qsl"], d["cl"], inp.scale,
                       max_len, inp.k_scale, inp.v_scale, workspace=ws, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out.float().cpu().numpy().astype(np.float64)


def _prefill_oracle(inp):
    s = inp.spec
    return orc.paged_prefill(inp.q, inp.k_pool, inp.v_pool, inp.block_tables,
                             inp.query_start_loc, inp.context_lens, inp.scale, s.q_dtype,
                             s.kv_dtype, inp.k_scale, inp.v_scale)


def _prefill_inputs(kv_dt, seed):
    spec = W.PrefillSpec("range", 3, 0, 0, 16, 2, 128, W.BF16, kv_dt, extra_blocks=3, seed=seed)
    return W.make_prefill_inputs(spec, chunk_lens=[70, 130, 3], histories=[0, 200, 611])


@pytest.mark.parametrize("staged", [False, True])
def test_prefill_bf16_keys_beyond_f16_range(B, cuda_device, staged):
    # K up to ~5e5 (f16 overflows at 65504), q down to ~1e-5 (f16 subnormal)
    inp = _prefill_inputs(W.BF16, 401)
    inp = dataclasses.replace(inp, q=_times(inp.q, 2.0 ** -15),
                              k_pool=_times(inp.k_pool, 2.0 ** 15))
    P.assert_close(_prefill(B, inp, cuda_device, staged), _prefill_oracle(inp), W.BF16, W.BF16,
                   "prefill bf16, q x 2^-15, K x 2^15")


@pytest.mark.parametrize("staged", [False, True])
@pytest.mark.parametrize("e", [17, -20])
def test_prefill_bf16_values_scaled(B, cuda_device, staged, e):
    inp = _prefill_inputs(W.BF16, 402)
    inp = dataclasses.replace(inp, v_pool=_times(inp.v_pool, 2.0 ** e))
    gpu = _prefill(B, inp, cuda_device, staged)
    ref = _prefill_oracle(inp)
    P.assert_close(gpu * 2.0 ** -e, ref * 2.0 ** -e, W.BF16, W.BF16, f"prefill bf16, V x 2^{e}")


@pytest.mark.parametrize("staged", [False, True])
def test_prefill_bf16_planted_queries_and_keys(B, cuda_device, staged):
    inp = _plant_qk(_prefill_inputs(W.BF16, 403), 1)
    P.assert_close(_prefill(B, inp, cuda_device, staged), _prefill_oracle(inp), W.BF16, W.BF16,
                   "prefill bf16, planted queries and keys")


@pytest.mark.parametrize("staged", [False, True])
def test_prefill_bf16_planted_values(B, cuda_device, staged):
    inp = _prefill_inputs(W.BF16, 406)
    inp = dataclasses.replace(inp, v_pool=_plant(inp.v_pool, range(128), 0.002, 3))
    gpu = _prefill(B, inp, cuda_device, staged)
    ref = _prefill_oracle(inp)
    assert np.abs(ref).max() > 1e4  # the planted values reach the outputs
    mag = _prefill_oracle(dataclasses.replace(inp, v_pool=inp.v_pool.abs()))
    _assert_close_mag(gpu, ref, mag, "prefill bf16, planted values")


@pytest.mark.parametrize("staged", [False, True])
@pytest.mark.parametrize("e", [20, -20])
def test_prefill_fp8_query_rows_far_from_f16_range(B, cuda_device, staged, e):
    # q x 2^-e with k_scale x 2^e leaves every score unchanged
    inp = _prefill_inputs(W.FP8_E4M3, 404)
    inp = dataclasses.replace(inp, q=_times(inp.q, 2.0 ** -e), k_scale=inp.k_scale * 2.0 ** e)
    P.assert_close(_prefill(B, inp, cuda_device, staged), _prefill_oracle(inp), W.BF16,
                   W.FP8_E4M3, f"prefill fp8, q x 2^{-e}")


@pytest.mark.parametrize("staged", [False, True])
def test_prefill_fp8_planted_queries(B, cuda_device, staged):
    inp = _plant_qk(_prefill_inputs(W.FP8_E4M3, 405), 4)
    P.assert_close(_prefill(B, inp, cuda_device, staged), _prefill_oracle(inp), W.BF16,
                   W.FP8_E4M3, "prefill fp8, planted queries")


# ------------------------------------------------------------------- decode

# contexts across the 1024-token (16-bit) and 2048-token (fp8) partitions
CTX = np.array([1, 2, 9, 16, 17, 300, 1100, 2049, 3000], np.int32)


def _decode_inputs(kv_dt, seed):
    spec = W.DecodeSpec("range", len(CTX), 16, 2, 128, W.BF16, kv_dt, "fixed", (CTX,),
                        max_ctx=3072, pool_factor=1.2, seed=seed)
    return W.make_decode_inputs(spec, ctx=CTX)


def _decode_check(inp, dev, what, out_scale=1.0):
    gpu, err = P.run_decode(inp, dev)
    assert err == 0
    ref = P.oracle_decode(inp)
    P.assert_close(gpu * out_scale, ref * out_scale, inp.spec.q_dtype, inp.spec.kv_dtype, what)
    return ref


def test_decode_bf16_keys_beyond_f16_range(B, cuda_device):
    inp = _decode_inputs(W.BF16, 411)
    inp = dataclasses.replace(inp, q=_times(inp.q, 2.0 ** -15),
                              k_pool=_times(inp.k_pool, 2.0 ** 15))
    _decode_check(inp, cuda_device, "decode bf16, q x 2^-15, K x 2^15")


@pytest.mark.parametrize("e", [17, -20])
def test_decode_bf16_values_scaled(B, cuda_device, e):
    inp = _decode_inputs(W.BF16, 412)
    inp = dataclasses.replace(inp, v_pool=_times(inp.v_pool, 2.0 ** e))
    _decode_check(inp, cuda_device, f"decode bf16, V x 2^{e}", out_scale=2.0 ** -e)


def test_decode_bf16_planted_queries_and_keys(B, cuda_device):
    inp = _plant_qk(_decode_inputs(W.BF16, 413), 5)
    _decode_check(inp, cuda_device, "decode bf16, planted queries and keys")


def test_decode_bf16_planted_values(B, cuda_device):
    inp = _decode_inputs(W.BF16, 417)
    inp = dataclasses.replace(inp, v_pool=_plant(inp.v_pool, range(128), 0.002, 7))
    gpu, err = P.run_decode(inp, cuda_device)
    assert err == 0
    ref = P.oracle_decode(inp)
    assert np.abs(ref).max() > 1e4
    mag = P.oracle_decode(dataclasses.replace(inp, v_pool=inp.v_pool.abs()))
    _assert_close_mag(gpu, ref, mag, "decode bf16, planted values")


@pytest.mark.parametrize("e", [20, -20])
def test_decode_fp8_query_rows_far_from_f16_range(B, cuda_device, e):
    inp = _decode_inputs(W.FP8_E4M3, 414)
    inp = dataclasses.replace(inp, q=_times(inp.q, 2.0 ** -e), k_scale=inp.k_scale * 2.0 ** e)
    _decode_check(inp, cuda_device, f"decode fp8, q x 2^{-e}")


def test_decode_fp8_planted_queries(B, cuda_device):
    inp = _plant_qk(_decode_inputs(W.FP8_E4M3, 415), 8)
    _decode_check(inp, cuda_device, "decode fp8, planted queries")


def test_decode_multi_fp8_query_rows_far_from_f16_range(B, cuda_device):
    from tests.test_decode_multi_gpu import oracle_multi, run_multi
    inp = _decode_inputs(W.FP8_E4M3, 416)
    qm = W.make_multi_queries(inp, 3, seed=9)
    for e in (20, -20):
        sub = dataclasses.replace(inp, k_scale=inp.k_scale * 2.0 ** e)
        q = _times(qm, 2.0 ** -e)
        gpu, err = run_multi(B, sub, q, cuda_device)
        assert err == 0
        P.assert_close(gpu, oracle_multi(sub, q), W.BF16, W.FP8_E4M3,
                       f"multi-query decode fp8, q x 2^{-e}")


# --------------------------------------------- multi-query (tcgen05 kernel)

def _multi_check(B, inp, qm, dev, what, out_scale=1.0):
    from tests.test_decode_multi_gpu import oracle_multi, run_multi
    gpu, err = run_multi(B, inp, qm, dev)
    assert err == 0
    ref = oracle_multi(inp, qm)
    P.assert_close(gpu * out_scale, ref * out_scale, W.BF16, W.BF16, what)


def test_decode_multi_bf16_keys_beyond_f16_range(B, cuda_device):
    inp = _decode_inputs(W.BF16, 421)
    qm = W.make_multi_queries(inp, 3, seed=10)
    inp = dataclasses.replace(inp, k_pool=_times(inp.k_pool, 2.0 ** 15))
    _multi_check(B, inp, _times(qm, 2.0 ** -15), cuda_device,
                 "multi-query decode bf16, q x 2^-15, K x 2^15")


@pytest.mark.parametrize("e", [17, -20])
def test_decode_multi_bf16_values_scaled(B, cuda_device, e):
    inp = _decode_inputs(W.BF16, 422)
    qm = W.make_multi_queries(inp, 3, seed=11)
    inp = dataclasses.replace(inp, v_pool=_times(inp.v_pool, 2.0 ** e))
    _multi_check(B, inp, qm, cuda_device, f"multi-query decode bf16, V x 2^{e}",
                 out_scale=2.0 ** -e)


def test_decode_multi_bf16_planted_queries_and_keys(B, cuda_device):
    inp = _decode_inputs(W.BF16, 423)
    qm = W.make_multi_queries(inp, 3, seed=12)
    qm = _plant(qm, Q_PLANT_DIMS, 0.05, 13, zero_dims=K_PLANT_DIMS)
    inp = dataclasses.replace(inp, k_pool=_plant(inp.k_pool, K_PLANT_DIMS, 0.05, 14,
                                                 zero_dims=Q_PLANT_DIMS))
    _multi_check(B, inp, qm, cuda_device, "multi-query decode bf16, planted queries and keys")


def test_decode_multi_bf16_planted_values(B, cuda_device):
    from tests.test_decode_multi_gpu import oracle_multi, run_multi
    inp = _decode_inputs(W.BF16, 424)
    qm = W.make_multi_queries(inp, 3, seed=15)
    inp = dataclasses.replace(inp, v_pool=_plant(inp.v_pool, range(128), 0.002, 16))
    gpu, err = run_multi(B, inp, qm, cuda_device)
    assert err == 0
    ref = oracle_multi(inp, qm)
    assert np.abs(ref).max() > 1e4
    mag = oracle_multi(dataclasses.replace(inp, v_pool=inp.v_pool.abs()), qm)
    _assert_close_mag(gpu, ref, mag, "multi-query decode bf16, planted values")
