"""Thin Python binding of libpa_b200.so (the C ABI in include/pa.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  Functions keep the C names and take torch tensors (device
memory) for the device pointers; shapes and dtypes are read off the tensors,
the stream is torch's current stream unless one is given.  If the shared
library is missing this module raises on import -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa_b200.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_OOM, PA_ERR_CUDA = range(5)
PA_F32, PA_F16, PA_BF16, PA_FP8_E4M3 = range(4)
PA_DEVERR_BLOCK_ID, PA_DEVERR_SLOT, PA_DEVERR_TIMEOUT, PA_DEVERR_QUERY_LOC = 1, 2, 4, 8

# every symbol include/pa.h declares
EXPORTS = (
    "pa_abi_version", "pa_status_string", "pa_decode_workspace_size", "pa_decode",
    "pa_decode_partitions", "pa_decode_reduce", "pa_prefill_paged", "pa_reshape_and_cache",
    "pa_copy_blocks", "pa_alloc_create", "pa_alloc_destroy", "pa_alloc_append",
    "pa_alloc_fork", "pa_alloc_prepare_write", "pa_alloc_free_seq", "pa_alloc_block_table",
    "pa_alloc_free_list", "pa_alloc_num_tokens", "pa_alloc_refcount", "pa_alloc_num_free",
    "pa_alloc_num_seqs", "pa_decode_noalloc", "pa_decode_noalloc_scratch_bytes",
    "pa_decode_multi", "pa_alloc_set_prefix_caching", "pa_alloc_admit",
    "pa_alloc_append_tokens", "pa_alloc_cached_list", "pa_alloc_num_cached",
    "pa_swap_blocks", "pa_decode_shared_prefix", "pa_prefix_groups",
    "pa_prefill_workspace_size", "pa_test_decode_timeout",
)


class PAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m pagedattention_paged_kv_pa_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, Z, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_int64
    L.pa_abi_version.restype = I
    L.pa_status_string.argtypes = [I]
    L.pa_status_string.restype = ctypes.c_char_p
    L.pa_decode_workspace_size.argtypes = [I, I, I, I]
    L.pa_decode_workspace_size.restype = Z
    dec = [P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, F, F, P, Z, P, P]
    L.pa_decode.argtypes = dec
    L.pa_decode_partitions.argtypes = dec
    L.pa_decode_reduce.argtypes = [P, P, I, I, I, I, I, I, F, P, Z, P]
    L.pa_decode_multi.argtypes = [P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, I, F, F, P, Z,
                                  P, P]
    L.pa_test_decode_timeout.argtypes = dec + [I, ctypes.c_uint32]
    L.pa_test_decode_timeout.restype = I
    L.pa_decode_noalloc.argtypes = [P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, F, F, P, P]
    L.pa_decode_noalloc.restype = I
    L.pa_decode_noalloc_scratch_bytes.restype = Z
    L.pa_prefill_paged.argtypes = [P, P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, I, F, F,
                                   P, Z, P, P]
    L.pa_prefill_workspace_size.argtypes = [I, I, I, I, I]
    L.pa_prefill_workspace_size.restype = Z
    L.pa_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, F, P, P]
    L.pa_copy_blocks.argtypes = [P, P, P, I, I, I, I, I, I, P, P]
    for fn in ("pa_decode", "pa_decode_partitions", "pa_decode_reduce", "pa_prefill_paged",
               "pa_reshape_and_cache", "pa_copy_blocks", "pa_alloc_append", "pa_alloc_fork",
               "pa_alloc_prepare_write", "pa_alloc_free_seq", "pa_alloc_block_table",
               "pa_alloc_free_list"):
        getattr(L, fn).restype = I
    L.pa_alloc_create.argtypes = [I, I, P]
    L.pa_alloc_create.restype = P
    L.pa_alloc_destroy.argtypes = [P]
    L.pa_alloc_destroy.restype = None
    L.pa_alloc_append.argtypes = [P, I64, I, P]
    L.pa_alloc_fork.argtypes = [P, I64, I64]
    L.pa_alloc_prepare_write.argtypes = [P, I64, P, P]
    L.pa_alloc_free_seq.argtypes = [P, I64]
    L.pa_alloc_block_table.argtypes = [P, I64, P, I, P]
    L.pa_alloc_free_list.argtypes = [P, P, I, P]
    L.pa_alloc_num_tokens.argtypes = [P, I64]
    L.pa_alloc_refcount.argtypes = [P, ctypes.c_int32]
    L.pa_alloc_num_free.argtypes = [P]
    L.pa_alloc_num_seqs.argtypes = [P]
    L.pa_swap_blocks.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P]
    L.pa_decode_shared_prefix.argtypes = [P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, F, F,
                                          P, P, P, I, I, P, Z, P, P]
    L.pa_prefix_groups.argtypes = [P, P, I, I, I, I, I, P, P, P, P, P]
    L.pa_alloc_set_prefix_caching.argtypes = [P, I]
    L.pa_alloc_admit.argtypes = [P, I64, P, I, P, P]
    L.pa_alloc_append_tokens.argtypes = [P, I64, P, I, P]
    L.pa_alloc_cached_list.argtypes = [P, P, I, P]
    L.pa_alloc_num_cached.argtypes = [P]
    for fn in ("pa_alloc_num_tokens", "pa_alloc_refcount", "pa_alloc_num_free",
               "pa_alloc_num_seqs", "pa_alloc_num_cached"):
        getattr(L, fn).restype = I
    return L


lib = _load()

_DT = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16,
       torch.uint8: PA_FP8_E4M3, torch.float8_e4m3fn: PA_FP8_E4M3}


def status_string(s: int) -> str:
    return lib.pa_status_string(s).decode()


def dtype_code(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise PAError(PA_ERR_UNSUPPORTED, f"dtype {t.dtype}") from None


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, what: str):
    if status != PA_OK:
        raise PAError(status, what)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise PAError(PA_ERR_INVALID_ARG, "tensors must be contiguous")


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------

def pa_decode_workspace_size(num_seqs: int, n_q_heads: int, head_dim: int,
                             max_blocks_per_seq: int) -> int:
    return lib.pa_decode_workspace_size(num_seqs, n_q_heads, head_dim, max_blocks_per_seq)


def alloc_decode_workspace(q: torch.Tensor, max_blocks_per_seq: int) -> torch.Tensor:
    n = pa_decode_workspace_size(q.shape[0], q.shape[1], q.shape[2], max_blocks_per_seq)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)


def _decode_args(out, q, k_pool, v_pool, block_tables, context_lens, scale, k_scale, v_scale,
                 workspace, dev_err, stream):
    _contig(out, q, k_pool, v_pool, block_tables, context_lens)
    num_seqs, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_pool.shape
    if d2 != d or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(out.shape) != tuple(q.shape):
        raise PAError(PA_ERR_INVALID_ARG, "pa_decode shapes")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise PAError(PA_ERR_INVALID_ARG, "block_tables / context_lens must be int32")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return (_p(out), _p(q), _p(k_pool), _p(v_pool), _p(block_tables), _p(context_lens),
            float(scale), bs, n_q, n_kv, d, num_seqs, block_tables.shape[1], num_blocks,
            dtype_code(q), dtype_code(k_pool), float(k_scale), float(v_scale), _p(workspace),
            ws_bytes, _p(dev_err), _stream(stream, q.device))


def pa_decode_multi(out, q, k_pool, v_pool, block_tables, context_lens, scale, k_scale=1.0,
                    v_scale=1.0, workspace=None, dev_err=None, stream=None):
    """Multi-query decode: q / out are [num_seqs, q_len, n_q, d]; query i of a
    sequence with context c attends to keys 0 .. c - q_len + i."""
    _contig(out, q, k_pool, v_pool, block_tables, context_lens)
    num_seqs, q_len, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_pool.shape
    if d2 != d or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(out.shape) != tuple(q.shape):
        raise PAError(PA_ERR_INVALID_ARG, "pa_decode_multi shapes")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise PAError(PA_ERR_INVALID_ARG, "block_tables / context_lens must be int32")
    mb = block_tables.shape[1]
    if workspace is None:
        n = pa_decode_workspace_size(num_seqs, n_q * q_len, d, mb)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_multi(_p(out), _p(q), _p(k_pool), _p(v_pool), _p(block_tables),
                               _p(context_lens), float(scale), bs, n_q, n_kv, d, num_seqs, q_len,
                               mb, num_blocks, dtype_code(q), dtype_code(k_pool), float(k_scale),
                               float(v_scale), _p(workspace), ws_bytes, _p(dev_err),
                               _stream(stream, q.device)), "pa_decode_multi")
    return out


def prefix_groups(block_tables, context_lens, n_q_heads: int, n_kv_heads: int, kv_dtype: int):
    """Groups of sequences whose block tables start with the same blocks (from
    host copies), as pa_decode_shared_prefix takes them: a dict with
    members [n_groups, width], shared_blocks [n_groups], seq_group [num_seqs]
    (int32 CPU tensors) and width."""
    bt = block_tables.detach().cpu().contiguous().to(torch.int32)
    cl = context_lens.detach().cpu().contiguous().to(torch.int32)
    ns, mb = bt.shape
    width = 32 // (n_q_heads // n_kv_heads)
    members = torch.full((max(ns, 1), width), -1, dtype=torch.int32)
    shared = torch.zeros(max(ns, 1), dtype=torch.int32)
    seq_group = torch.full((max(ns, 1),), -1, dtype=torch.int32)
    ng, w = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.pa_prefix_groups(_p(bt), _p(cl), ns, mb, n_q_heads, n_kv_heads, kv_dtype,
                                _p(members), _p(shared), _p(seq_group), ctypes.byref(ng),
                                ctypes.byref(w)), "pa_prefix_groups")
    n, w = ng.value, w.value
    flat = members.view(-1)[:n * w]
    return {"members": flat.view(n, w).clone(), "shared_blocks": shared[:n].clone(),
            "seq_group": seq_group[:ns].clone(), "width": w}


def pa_decode_shared_prefix(out, q, k_pool, v_pool, block_tables, context_lens, scale, groups,
                            k_scale=1.0, v_scale=1.0, workspace=None, dev_err=None, stream=None):
    """pa_decode's result with each group's shared prefix read once for the
    group (groups as returned by prefix_groups, on any device)."""
    if workspace is None:
        workspace = alloc_decode_workspace(q, block_tables.shape[1])
    dev = q.device
    members = groups["members"].to(dev, torch.int32).contiguous()
    shared = groups["shared_blocks"].to(dev, torch.int32).contiguous()
    seq_group = groups["seq_group"].to(dev, torch.int32).contiguous()
    a = _decode_args(out, q, k_pool, v_pool, block_tables, context_lens, scale, k_scale,
                     v_scale, workspace, dev_err, stream)
    # pa_decode's arguments with the group arrays before the workspace
    _check(lib.pa_decode_shared_prefix(*a[:18], _p(members), _p(shared), _p(seq_group),
                                       members.shape[0], int(groups["width"]), *a[18:]),
           "pa_decode_shared_prefix")
    return out


def pa_decode(out, q, k_pool, v_pool, block_tables, context_lens, scale, k_scale=1.0,
              v_scale=1.0, workspace=None, dev_err=None, stream=None):
    """out[s][h] = softmax(scale * q[s][h] . K^T) V over the paged cache."""
    if workspace is None:
        workspace = alloc_decode_workspace(q, block_tables.shape[1])
    _check(lib.pa_decode(*_decode_args(out, q, k_pool, v_pool, block_tables, context_lens,
                                       scale, k_scale, v_scale, workspace, dev_err, stream)),
           "pa_decode")
    return out


def pa_test_decode_timeout(out, q, k_pool, v_pool, block_tables, context_lens, scale,
                           skip_tile: int, wait_limit_us: int, k_scale=1.0, v_scale=1.0,
                           workspace=None, dev_err=None, stream=None):
    """Test hook: pa_decode with short bounded waits and one tile's stage left
    unfilled in every CTA, so the waits run out (see include/pa.h)."""
    if workspace is None:
        workspace = alloc_decode_workspace(q, block_tables.shape[1])
    _check(lib.pa_test_decode_timeout(*_decode_args(out, q, k_pool, v_pool, block_tables,
                                                    context_lens, scale, k_scale, v_scale,
                                                    workspace, dev_err, stream),
                                      int(skip_tile), int(wait_limit_us)),
           "pa_test_decode_timeout")
    return out


def pa_decode_noalloc(out, q, k_pool, v_pool, block_tables, context_lens, scale, k_scale=1.0,
                      v_scale=1.0, dev_err=None, stream=None):
    """pa_decode without a caller workspace: the library's own static device
    scratch holds the partition results (see include/pa.h for its limit and
    the ordering rule between calls)."""
    a = _decode_args(out, q, k_pool, v_pool, block_tables, context_lens, scale, k_scale,
                     v_scale, None, dev_err, stream)
    st = lib.pa_decode_noalloc(*a[:18], a[20], a[21])
    if st == PA_ERR_UNSUPPORTED:
        need = pa_decode_workspace_size(q.shape[0], q.shape[1], q.shape[2],
                                        block_tables.shape[1])
        cap = lib.pa_decode_noalloc_scratch_bytes()
        if need > cap:
            raise PAError(st, f"pa_decode_noalloc needs {need} bytes of scratch; the library's "
                              f"static scratch holds {cap}")
    _check(st, "pa_decode_noalloc")
    return out


def pa_decode_partitions(out, q, k_pool, v_pool, block_tables, context_lens, scale,
                         k_scale=1.0, v_scale=1.0, workspace=None, dev_err=None, stream=None):
    _check(lib.pa_decode_partitions(*_decode_args(out, q, k_pool, v_pool, block_tables,
                                                  context_lens, scale, k_scale, v_scale,
                                                  workspace, dev_err, stream)),
           "pa_decode_partitions")


def pa_decode_reduce(out, context_lens, max_blocks_per_seq, kv_dtype, v_scale=1.0,
                     workspace=None, stream=None):
    num_seqs, n_q, d = out.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_reduce(_p(out), _p(context_lens), n_q, d, num_seqs, max_blocks_per_seq,
                                dtype_code(out), kv_dtype, float(v_scale), _p(workspace),
                                ws_bytes, _stream(stream, out.device)), "pa_decode_reduce")


# --------------------------------------------------------------------------
# prefill
# --------------------------------------------------------------------------

def pa_prefill_workspace_size(n_chunks: int, n_kv_heads: int, head_dim: int,
                              max_blocks_per_seq: int, block_size: int = 16) -> int:
    return lib.pa_prefill_workspace_size(n_chunks, n_kv_heads, head_dim, max_blocks_per_seq,
                                         block_size)


def alloc_prefill_workspace(k_pool: torch.Tensor, block_tables: torch.Tensor) -> torch.Tensor:
    """Workspace for pa_prefill_paged over these chunks' block tables."""
    num_blocks, n_kv, bs, d = k_pool.shape
    n = pa_prefill_workspace_size(block_tables.shape[0], n_kv, d, block_tables.shape[1], bs)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=k_pool.device)


def pa_prefill_paged(out, q, k_pool, v_pool, block_tables, query_start_loc, context_lens,
                     scale, max_chunk_len, k_scale=1.0, v_scale=1.0, workspace=None,
                     dev_err=None, stream=None):
    """workspace: None (the attention kernel widens K/V itself) or a device
    buffer of pa_prefill_workspace_size bytes (widened once per chunk)."""
    _contig(out, q, k_pool, v_pool, block_tables, query_start_loc, context_lens)
    total_q, n_q, d = q.shape
    num_blocks, n_kv, bs, _ = k_pool.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.pa_prefill_paged(_p(out), _p(q), _p(k_pool), _p(v_pool), _p(block_tables),
                                _p(query_start_loc), _p(context_lens), float(scale), bs, n_q,
                                n_kv, d, context_lens.shape[0], int(max_chunk_len),
                                block_tables.shape[1], num_blocks, dtype_code(q),
                                dtype_code(k_pool), float(k_scale), float(v_scale),
                                _p(workspace), ws_bytes, _p(dev_err),
                                _stream(stream, q.device)), "pa_prefill_paged")
    return out


# --------------------------------------------------------------------------
# slot write / block copy
# --------------------------------------------------------------------------

def pa_reshape_and_cache(k_pool, v_pool, key, value, slot_mapping, k_scale=1.0, v_scale=1.0,
                         dev_err=None, stream=None):
    _contig(k_pool, v_pool, key, value, slot_mapping)
    if slot_mapping.dtype != torch.int64:
        raise PAError(PA_ERR_INVALID_ARG, "slot_mapping must be int64")
    num_tokens, n_kv, d = key.shape
    num_blocks, _, bs, _ = k_pool.shape
    _check(lib.pa_reshape_and_cache(_p(k_pool), _p(v_pool), _p(key), _p(value),
                                    _p(slot_mapping), num_tokens, n_kv, d, bs, num_blocks,
                                    dtype_code(key), dtype_code(k_pool), float(k_scale),
                                    float(v_scale), _p(dev_err), _stream(stream, key.device)),
           "pa_reshape_and_cache")


def pa_copy_blocks(k_pool, v_pool, block_pairs, dev_err=None, stream=None):
    _contig(k_pool, v_pool, block_pairs)
    if block_pairs.dtype != torch.int64:
        raise PAError(PA_ERR_INVALID_ARG, "block_pairs must be int64 [n][2]")
    num_blocks, n_kv, bs, d = k_pool.shape
    n_pairs = block_pairs.numel() // 2
    _check(lib.pa_copy_blocks(_p(k_pool), _p(v_pool), _p(block_pairs), n_pairs, n_kv, d, bs,
                              num_blocks, dtype_code(k_pool), _p(dev_err),
                              _stream(stream, k_pool.device)), "pa_copy_blocks")


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, block_pairs, dev_err=None, stream=None):
    """Block dst of (dst_k, dst_v) := block src of (src_k, src_v) for every
    (src, dst) row of block_pairs.  Each pool (and block_pairs) is a tensor on
    the current CUDA device or a pinned CPU tensor."""
    _contig(dst_k, dst_v, src_k, src_v, block_pairs)
    if block_pairs.dtype != torch.int64:
        raise PAError(PA_ERR_INVALID_ARG, "block_pairs must be int64 [n][2]")
    dn, n_kv, bs, d = dst_k.shape
    sn = src_k.shape[0]
    if tuple(src_k.shape[1:]) != (n_kv, bs, d) or dst_v.shape != dst_k.shape or \
            src_v.shape != src_k.shape or dtype_code(src_k) != dtype_code(dst_k):
        raise PAError(PA_ERR_INVALID_ARG, "pa_swap_blocks pool shapes")
    dev = next((t.device for t in (dst_k, src_k, block_pairs) if t.is_cuda),
               torch.device("cuda", torch.cuda.current_device()))
    _check(lib.pa_swap_blocks(_p(dst_k), _p(dst_v), _p(src_k), _p(src_v), _p(block_pairs),
                              block_pairs.numel() // 2, n_kv, d, bs, sn, dn, dtype_code(dst_k),
                              _p(dev_err), _stream(stream, dev)), "pa_swap_blocks")


# --------------------------------------------------------------------------
# host allocator
# --------------------------------------------------------------------------

class BlockAllocator:
    """Owning wrapper of a pa_alloc handle (see include/pa.h)."""

    def __init__(self, num_blocks: int, block_size: int = 16, initial_free_order=None):
        self.num_blocks = num_blocks
        self._lib = lib  # kept so __del__ still works during interpreter shutdown
        order = None
        if initial_free_order is not None:
            arr = (ctypes.c_int32 * num_blocks)(*initial_free_order)
            order = ctypes.cast(arr, ctypes.c_void_p)
        self._h = lib.pa_alloc_create(num_blocks, block_size, order)
        if not self._h:
            raise PAError(PA_ERR_INVALID_ARG, "pa_alloc_create")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._lib.pa_alloc_destroy(h)
            self._h = None

    def append(self, seq: int, n_tokens: int):
        """Returns (status, slots list)."""
        buf = (ctypes.c_int64 * max(n_tokens, 1))()
        st = lib.pa_alloc_append(self._h, seq, n_tokens, ctypes.cast(buf, ctypes.c_void_p))
        return st, (list(buf[:n_tokens]) if st == PA_OK else [])

    def fork(self, parent: int, child: int) -> int:
        return lib.pa_alloc_fork(self._h, parent, child)

    def prepare_write(self, seq: int):
        buf = (ctypes.c_int64 * 2)()
        n = ctypes.c_int(0)
        st = lib.pa_alloc_prepare_write(self._h, seq, ctypes.cast(buf, ctypes.c_void_p),
                                        ctypes.byref(n))
        return st, ([(buf[0], buf[1])] if (st == PA_OK and n.value == 1) else [])

    def free_seq(self, seq: int) -> int:
        return lib.pa_alloc_free_seq(self._h, seq)

    def block_table(self, seq: int):
        cap = self.num_blocks
        buf = (ctypes.c_int32 * cap)()
        n = ctypes.c_int(0)
        st = lib.pa_alloc_block_table(self._h, seq, ctypes.cast(buf, ctypes.c_void_p), cap,
                                      ctypes.byref(n))
        _check(st, "pa_alloc_block_table")
        return list(buf[:n.value])

    def free_list(self):
        buf = (ctypes.c_int32 * self.num_blocks)()
        n = ctypes.c_int(0)
        _check(lib.pa_alloc_free_list(self._h, ctypes.cast(buf, ctypes.c_void_p),
                                      self.num_blocks, ctypes.byref(n)), "pa_alloc_free_list")
        return list(buf[:n.value])

    def num_tokens(self, seq: int) -> int:
        return lib.pa_alloc_num_tokens(self._h, seq)

    def refcount(self, block: int) -> int:
        return lib.pa_alloc_refcount(self._h, block)

    def num_free(self) -> int:
        return lib.pa_alloc_num_free(self._h)

    def num_seqs(self) -> int:
        return lib.pa_alloc_num_seqs(self._h)

    # -- prefix caching -------------------------------------------------------
    def set_prefix_caching(self, on: bool) -> int:
        return lib.pa_alloc_set_prefix_caching(self._h, 1 if on else 0)

    def admit(self, seq: int, tokens):
        """Returns (status, slots list, n_cached tokens)."""
        n = len(tokens)
        toks = (ctypes.c_int32 * max(n, 1))(*tokens)
        buf = (ctypes.c_int64 * max(n, 1))()
        nc = ctypes.c_int(0)
        st = lib.pa_alloc_admit(self._h, seq, ctypes.cast(toks, ctypes.c_void_p), n,
                                ctypes.cast(buf, ctypes.c_void_p), ctypes.byref(nc))
        return st, (list(buf[:n]) if st == PA_OK else []), (nc.value if st == PA_OK else 0)

    def append_tokens(self, seq: int, tokens):
        """Returns (status, slots list)."""
        n = len(tokens)
        toks = (ctypes.c_int32 * max(n, 1))(*tokens)
        buf = (ctypes.c_int64 * max(n, 1))()
        st = lib.pa_alloc_append_tokens(self._h, seq, ctypes.cast(toks, ctypes.c_void_p), n,
                                        ctypes.cast(buf, ctypes.c_void_p))
        return st, (list(buf[:n]) if st == PA_OK else [])

    def cached_list(self):
        buf = (ctypes.c_int32 * self.num_blocks)()
        n = ctypes.c_int(0)
        _check(lib.pa_alloc_cached_list(self._h, ctypes.cast(buf, ctypes.c_void_p),
                                        self.num_blocks, ctypes.byref(n)), "pa_alloc_cached_list")
        return list(buf[:n.value])

    def num_cached(self) -> int:
        return lib.pa_alloc_num_cached(self._h)
