"""CPU oracle for the paged-KV hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path never does, and nothing here
imports the product's CUDA library or shares code with it.

The arithmetic lives in ``pa_oracle.c`` (plain fp64 C, built with gcc by
``build.py``); this module only marshals NumPy arrays into it.  The
allocator's reference model is the pure-Python ``alloc_model``.

Every function here takes raw storage arrays (NumPy, or CPU torch tensors,
which are viewed as bytes) plus a dtype code with the numbering
F32=0, F16=1, BF16=2, FP8_E4M3=3.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

F32, F16, BF16, FP8_E4M3 = 0, 1, 2, 3
_ELEM = {F32: 4, F16: 2, BF16: 2, FP8_E4M3: 1}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P, I, D, F, I64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_float,
                           ctypes.c_int64)
        L.orc_paged_decode.argtypes = [P, P, I, P, P, I, P, P, D, D, D, I, I, I, I, I, I, I, I]
        L.orc_paged_decode.restype = I
        L.orc_paged_prefill.argtypes = [P, P, I, P, P, I, P, P, P, D, D, D, I, I, I, I, I, I,
                                        I, I]
        L.orc_paged_prefill.restype = I
        L.orc_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, F]
        L.orc_reshape_and_cache.restype = I
        L.orc_copy_blocks.argtypes = [P, P, P, I, I, I, I, I, I]
        L.orc_copy_blocks.restype = I
        L.orc_swap_blocks.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I]
        L.orc_swap_blocks.restype = I
        L.orc_decode_array.argtypes = [I, P, P, I64]
        L.orc_encode_e4m3_array.argtypes = [P, P, I64]
        L.orc_encode_bf16_array.argtypes = [P, P, I64]
        L.orc_encode_f16_array.argtypes = [P, P, I64]
        _lib = L
    return _lib


def _np(x) -> np.ndarray:
    """A C-contiguous NumPy view of an array or CPU torch tensor."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype in (torch.bfloat16, torch.float8_e4m3fn):
                x = x.view(torch.uint8 if x.element_size() == 1 else torch.int16)
            return x.numpy()
    except ImportError:
        pass
    return np.ascontiguousarray(x)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return os.cpu_count() or 1


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def paged_decode(q, k_pool, v_pool, block_tables, context_lens, scale, q_dtype, kv_dtype,
                 k_scale=1.0, v_scale=1.0, nthreads=None) -> np.ndarray:
    """fp64 decode attention over the paged pools; returns [num_seqs, n_q, d].

    Shapes: q [num_seqs, n_q, d]; pools [num_blocks, n_kv, 16, d];
    block_tables int32 [num_seqs, max_blocks]; context_lens int32 [num_seqs].
    """
    q, kp, vp = _np(q), _np(k_pool), _np(v_pool)
    bt = np.ascontiguousarray(_np(block_tables), dtype=np.int32)
    cl = np.ascontiguousarray(_np(context_lens), dtype=np.int32)
    num_seqs, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = kp.shape
    assert d == d2 and vp.shape == kp.shape
    out = np.zeros((num_seqs, n_q, d), dtype=np.float64)
    bad = lib().orc_paged_decode(_ptr(out), _ptr(q), q_dtype, _ptr(kp), _ptr(vp), kv_dtype,
                                 _ptr(bt), _ptr(cl), float(scale), float(k_scale),
                                 float(v_scale), num_seqs, n_q, n_kv, d, bs, bt.shape[1],
                                 num_blocks, nthreads or default_threads())
    if bad:
        raise ValueError(f"oracle: {bad} (seq, kv head) units hit an out-of-range block id")
    return out


def paged_prefill(q, k_pool, v_pool, block_tables, query_start_loc, context_lens, scale,
                  q_dtype, kv_dtype, k_scale=1.0, v_scale=1.0, nthreads=None) -> np.ndarray:
    """fp64 causal chunked-prefill attention; returns [total_q, n_q, d]."""
    q, kp, vp = _np(q), _np(k_pool), _np(v_pool)
    bt = np.ascontiguousarray(_np(block_tables), dtype=np.int32)
    qsl = np.ascontiguousarray(_np(query_start_loc), dtype=np.int32)
    cl = np.ascontiguousarray(_np(context_lens), dtype=np.int32)
    total_q, n_q, d = q.shape
    num_blocks, n_kv, bs, _ = kp.shape
    out = np.zeros((total_q, n_q, d), dtype=np.float64)
    bad = lib().orc_paged_prefill(_ptr(out), _ptr(q), q_dtype, _ptr(kp), _ptr(vp), kv_dtype,
                                  _ptr(bt), _ptr(qsl), _ptr(cl), float(scale), float(k_scale),
                                  float(v_scale), len(cl), n_q, n_kv, d, bs, bt.shape[1],
                                  num_blocks, nthreads or default_threads())
    if bad:
        raise ValueError(f"oracle: {bad} (chunk, kv head) units were invalid")
    return out


# --------------------------------------------------------------------------
# slot write / block copy (in place on NumPy pools)
# --------------------------------------------------------------------------

def reshape_and_cache(k_pool: np.ndarray, v_pool: np.ndarray, key, value, slot_mapping,
                      src_dtype: int, cache_dtype: int, k_scale=1.0, v_scale=1.0) -> int:
    """Writes new K/V rows into their slots of the NumPy pools, in place.
    Returns the number of tokens skipped for an out-of-range slot."""
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    key, value = _np(key), _np(value)
    sm = np.ascontiguousarray(_np(slot_mapping), dtype=np.int64)
    num_blocks, n_kv, bs, d = k_pool.shape
    r = lib().orc_reshape_and_cache(_ptr(k_pool), _ptr(v_pool), _ptr(key), _ptr(value),
                                    _ptr(sm), len(sm), n_kv, d, bs, num_blocks, src_dtype,
                                    cache_dtype, float(k_scale), float(v_scale))
    if r < 0:
        raise ValueError("oracle: unsupported dtype pair")
    return r


def copy_blocks(k_pool: np.ndarray, v_pool: np.ndarray, pairs, dtype: int) -> int:
    """Copies whole blocks (src -> dst for every pair), in place."""
    pr = np.ascontiguousarray(_np(pairs), dtype=np.int64).reshape(-1, 2)
    num_blocks, n_kv, bs, d = k_pool.shape
    return lib().orc_copy_blocks(_ptr(k_pool), _ptr(v_pool), _ptr(pr), len(pr), n_kv, d, bs,
                                 num_blocks, dtype)


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

def swap_blocks(dst_k: np.ndarray, dst_v: np.ndarray, src_k, src_v, pairs, dtype: int) -> int:
    """Copies block src of the source pools to block dst of the destination
    pools for every (src, dst) pair, in place on dst; returns the number of
    pairs skipped for an out-of-range id."""
    assert dst_k.flags.c_contiguous and dst_v.flags.c_contiguous
    sk, sv = _np(src_k), _np(src_v)
    pr = np.ascontiguousarray(_np(pairs), dtype=np.int64).reshape(-1, 2)
    dn, n_kv, bs, d = dst_k.shape
    return lib().orc_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(sk), _ptr(sv), _ptr(pr), len(pr),
                                 n_kv, d, bs, sk.shape[0], dn, dtype)


def decode_values(codes, dtype: int) -> np.ndarray:
    a = _np(codes)
    n = a.size
    out = np.empty(n, dtype=np.float64)
    lib().orc_decode_array(dtype, _ptr(a), _ptr(out), n)
    return out.reshape(a.shape)


def encode_e4m3(values_f32) -> np.ndarray:
    a = np.ascontiguousarray(values_f32, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint8)
    lib().orc_encode_e4m3_array(_ptr(a), _ptr(out), a.size)
    return out


def encode_bf16(values_f64) -> np.ndarray:
    a = np.ascontiguousarray(values_f64, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().orc_encode_bf16_array(_ptr(a), _ptr(out), a.size)
    return out


def encode_f16(values_f64) -> np.ndarray:
    a = np.ascontiguousarray(values_f64, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().orc_encode_f16_array(_ptr(a), _ptr(out), a.size)
    return out
