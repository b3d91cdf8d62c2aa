"""GPU parity of pa_reshape_and_cache and pa_copy_blocks: bit-exact against
the oracle (byte copies and E4M3 quantisation alike)."""
import numpy as np
import pytest
import torch

import oracle as orc
from pagedattention_paged_kv_pa_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding
    return binding


def _pools(nb, n_kv, d, dt, dev, seed=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    if dt == W.FP8_E4M3:
        k = torch.randint(0, 0x7E, (nb, n_kv, 16, d), dtype=torch.uint8, generator=g)
        v = torch.randint(0, 0x7E, (nb, n_kv, 16, d), dtype=torch.uint8, generator=g)
    else:
        k = torch.randn(nb, n_kv, 16, d, generator=g).to(W.TORCH_DTYPE[dt])
        v = torch.randn(nb, n_kv, 16, d, generator=g).to(W.TORCH_DTYPE[dt])
    return k, v


def _raw(t):
    t = t.cpu().contiguous()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    return t.numpy().copy()


def _scatter_both(B, dev, kp, vp, key, val, slots, src_dt, cache_dt, ks=1.0, vs=1.0):
    kg, vg = kp.to(dev), vp.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B.pa_reshape_and_cache(kg, vg, key.to(dev), val.to(dev), slots.to(dev), ks, vs, dev_err=err)
    torch.cuda.synchronize()
    ko, vo = _raw(kp), _raw(vp)
    bad = orc.reshape_and_cache(ko, vo, key, val, slots, src_dt, cache_dt, ks, vs)
    return _raw(kg), _raw(vg), ko, vo, int(err.item()), bad


@pytest.mark.parametrize("dt", [W.F32, W.F16, W.BF16])
@pytest.mark.parametrize("d", [64, 128])
def test_scatter_same_dtype_bit_exact(B, cuda_device, dt, d):
    nb, n_kv, T = 40, 8, 300
    kp, vp = _pools(nb, n_kv, d, dt, cuda_device)
    key, val = W.make_new_kv(T, n_kv, d, dt, "cpu", seed=3)
    rng = np.random.default_rng(4)
    slots = rng.choice(nb * 16, size=T, replace=False).astype(np.int64)
    slots[::37] = -1
    kg, vg, ko, vo, err, bad = _scatter_both(B, cuda_device, kp, vp, key, val,
                                             torch.from_numpy(slots), dt, dt)
    assert err == 0 and bad == 0
    assert np.array_equal(kg, ko) and np.array_equal(vg, vo)


@pytest.mark.parametrize("src_dt", [W.BF16, W.F16])
@pytest.mark.parametrize("scale", [1.0, 0.37, 0.0029])
def test_scatter_fp8_exhaustive_16bit_inputs(B, cuda_device, src_dt, scale):
    # every finite 16-bit pattern passes through the quantiser once (as K and,
    # negated, as V): CUDA's E4M3 conversion against the oracle's encoder
    codes = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = orc.decode_values(codes, src_dt)
    codes = codes[np.isfinite(vals)]
    T, n_kv, d = len(codes) // 128, 1, 128
    codes = codes[:T * 128]
    tdt = torch.bfloat16 if src_dt == W.BF16 else torch.float16
    key = torch.from_numpy(codes.view(np.int16).reshape(T, n_kv, d).copy()).view(tdt)
    val = torch.from_numpy(codes[::-1].view(np.int16).reshape(T, n_kv, d).copy()).view(tdt)
    nb = T // 16 + 1
    kp = torch.zeros(nb, n_kv, 16, d, dtype=torch.uint8)
    vp = torch.zeros_like(kp)
    slots = torch.from_numpy(np.random.default_rng(5).permutation(nb * 16)[:T].astype(np.int64))
    kg, vg, ko, vo, err, bad = _scatter_both(B, cuda_device, kp, vp, key, val, slots, src_dt,
                                             W.FP8_E4M3, scale, scale * 1.7)
    assert err == 0 and bad == 0
    assert np.array_equal(kg, ko)
    assert np.array_equal(vg, vo)


def test_scatter_fp8_from_f32(B, cuda_device):
    T, n_kv, d = 256, 4, 128
    g = torch.Generator().manual_seed(9)
    key = torch.randn(T, n_kv, d, generator=g) * 100
    val = torch.randn(T, n_kv, d, generator=g) * 1e-3
    kp = torch.zeros(20, n_kv, 16, d, dtype=torch.uint8)
    vp = torch.zeros_like(kp)
    slots = torch.arange(T, dtype=torch.int64) + 13
    kg, vg, ko, vo, err, bad = _scatter_both(B, cuda_device, kp, vp, key, val, slots, W.F32,
                                             W.FP8_E4M3, 0.21, 1e-5)
    assert np.array_equal(kg, ko) and np.array_equal(vg, vo)


def test_scatter_out_of_range_slot_flagged_and_skipped(B, cuda_device):
    kp, vp = _pools(4, 2, 64, W.BF16, cuda_device)
    key, val = W.make_new_kv(3, 2, 64, W.BF16, "cpu", seed=1)
    slots = torch.tensor([5, 4 * 16 + 1, -1], dtype=torch.int64)
    kg, vg, ko, vo, err, bad = _scatter_both(B, cuda_device, kp, vp, key, val, slots, W.BF16,
                                             W.BF16)
    assert err & 2 and bad == 1
    assert np.array_equal(kg, ko) and np.array_equal(vg, vo)


@pytest.mark.parametrize("dt", [W.BF16, W.FP8_E4M3, W.F32])
def test_copy_blocks_bit_exact(B, cuda_device, dt):
    nb, n_kv, d = 64, 8, 128
    kp, vp = _pools(nb, n_kv, d, dt, cuda_device, seed=11)
    pairs = torch.tensor([[3, 40], [3, 41], [7, 9], [63, 0]], dtype=torch.int64)
    kg, vg = kp.to(cuda_device), vp.to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    B.pa_copy_blocks(kg, vg, pairs.to(cuda_device), dev_err=err)
    torch.cuda.synchronize()
    ko, vo = _raw(kp), _raw(vp)
    orc.copy_blocks(ko, vo, pairs.numpy(), dt)
    assert int(err.item()) == 0
    assert np.array_equal(_raw(kg), ko) and np.array_equal(_raw(vg), vo)


def test_copy_blocks_bad_pair_flagged(B, cuda_device):
    kp, vp = _pools(8, 2, 64, W.F16, cuda_device)
    kg, vg = kp.to(cuda_device), vp.to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pairs = torch.tensor([[1, 2], [1, 99]], dtype=torch.int64, device=cuda_device)
    B.pa_copy_blocks(kg, vg, pairs, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & 2
    ko, vo = _raw(kp), _raw(vp)
    orc.copy_blocks(ko, vo, np.array([[1, 2]]), W.F16)
    assert np.array_equal(_raw(kg), ko)


# ---------------------------------------------------------------------------
# swap between a device pool and a pinned host pool
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dt", [W.BF16, W.FP8_E4M3, W.F32])
@pytest.mark.parametrize("pairs_on_host", [False, True])
def test_swap_round_trip_bit_exact(B, cuda_device, dt, pairs_on_host):
    dev = cuda_device
    n_kv, d = 8, 128
    gk, gv = _pools(40, n_kv, d, dt, "cpu", seed=21)
    gkd, gvd = gk.to(dev), gv.to(dev)
    hk = torch.zeros((24,) + tuple(gk.shape[1:]), dtype=gk.dtype).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    out_pairs = torch.tensor([[3, 0], [39, 23], [17, 5], [0, 11]], dtype=torch.int64)
    pr = out_pairs.pin_memory() if pairs_on_host else out_pairs.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B.pa_swap_blocks(hk, hv, gkd, gvd, pr, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rk, rv = np.zeros_like(_raw(hk)), np.zeros_like(_raw(hv))
    assert orc.swap_blocks(rk, rv, _raw(gk), _raw(gv), out_pairs.numpy(), dt) == 0
    assert np.array_equal(_raw(hk), rk) and np.array_equal(_raw(hv), rv)
    # back into other device blocks
    back = torch.tensor([[0, 7], [23, 30], [5, 1], [11, 2]], dtype=torch.int64)
    prb = back.pin_memory() if pairs_on_host else back.to(dev)
    B.pa_swap_blocks(gkd, gvd, hk, hv, prb, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ek, ev = _raw(gk), _raw(gv)
    assert orc.swap_blocks(ek, ev, rk, rv, back.numpy(), dt) == 0
    assert np.array_equal(_raw(gkd), ek) and np.array_equal(_raw(gvd), ev)


def test_swap_refuses_pageable_host_memory(B, cuda_device):
    dev = cuda_device
    gk, gv = (t.to(dev) for t in _pools(8, 2, 64, W.BF16, "cpu", seed=3))
    hk = torch.zeros((4,) + tuple(gk.shape[1:]), dtype=gk.dtype)   # not pinned
    hv = torch.zeros_like(hk)
    pairs = torch.tensor([[1, 0]], dtype=torch.int64, device=dev)
    with pytest.raises(B.PAError) as e:
        B.pa_swap_blocks(hk, hv, gk, gv, pairs)
    assert e.value.status == B.PA_ERR_INVALID_ARG
    assert not hk.any() and not hv.any()


def test_swap_out_of_range_ids_flagged(B, cuda_device):
    dev = cuda_device
    gk, gv = (t.to(dev) for t in _pools(8, 2, 64, W.BF16, "cpu", seed=5))
    hk = torch.zeros((4,) + tuple(gk.shape[1:]), dtype=gk.dtype).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    pairs = torch.tensor([[1, 0], [8, 1], [2, 4]], dtype=torch.int64, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B.pa_swap_blocks(hk, hv, gk, gv, pairs, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & 2  # PA_DEVERR_SLOT
    assert torch.equal(hk[0], gk[1].cpu()) and not hk[1:].any()
