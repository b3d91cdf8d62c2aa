"""Seeded synthetic inputs for the paged-KV decode path.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It draws random numbers and lays them out; it holds none of
the method's arithmetic (no attention, no softmax, no quantisation rule of its
own, no allocator policy).  Rounding of generated fp32 values into the storage
dtypes is done by torch's own casts (round-to-nearest-even), i.e. a library
routine, never by code that the oracle or the kernels also use.

Shapes follow the workloads the pages talk about:

* 16-token blocks ("LLM inference optimization: KV cache & PagedAttention",
  §三.1 "Logical Block Table"; "vLLM explained", "Block 的大小怎麼決定");
* Llama-2-7B layer shape (32 q / 32 kv heads, head_dim 128, fp16) from the
  block-bytes example in "vLLM explained", "Block 的大小怎麼決定";
* Llama-3-70B GQA layer shape (8 kv heads, head_dim 128) from the per-token
  KV formula example in "LLM inference optimization", §二.1.2;
* contexts up to 8K tokens (same section's 8,192-token example).

Index arrays (context lengths, block permutations) come from NumPy PCG64 so
they are identical on every machine; bulk values come from a seeded torch
generator on the requested device so full-size pools can be made in HBM.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

BLOCK_SIZE = 16

# dtype codes; the numbering is the one the C ABI uses (pa_dtype in include/pa.h)
F32, F16, BF16, FP8_E4M3 = 0, 1, 2, 3
DTYPE_NAMES = {F32: "f32", F16: "f16", BF16: "bf16", FP8_E4M3: "fp8_e4m3"}
TORCH_DTYPE = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16,
               FP8_E4M3: torch.uint8}
ELEM_BYTES = {F32: 4, F16: 2, BF16: 2, FP8_E4M3: 1}
FP8_E4M3_MAX = 448.0  # largest finite OCP E4M3FN value


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _torch_gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_as(shape, dtype_code: int, device, gen: torch.Generator,
             chunk: int = 1 << 27) -> torch.Tensor:
    """N(0,1) fp32 draws cast to a 16/32-bit storage dtype (torch RNE cast)."""
    out = torch.empty(shape, dtype=TORCH_DTYPE[dtype_code], device=device)
    flat = out.view(-1)
    for s in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - s)
        flat[s:s + n] = torch.randn(n, generator=gen, device=device,
                                    dtype=torch.float32).to(flat.dtype)
    return out


def _amax_of_draws(numels, device, gen: torch.Generator, chunk: int = 1 << 27) -> float:
    m = 0.0
    for total in numels:
        for s in range(0, total, chunk):
            n = min(chunk, total - s)
            x = torch.randn(n, generator=gen, device=device, dtype=torch.float32)
            m = max(m, float(x.abs().max()))
    return m


def randn_fp8_codes(shape, scale: float, device, gen: torch.Generator,
                    chunk: int = 1 << 27) -> torch.Tensor:
    """E4M3 codes (as uint8) of N(0,1) draws divided by a per-tensor scale.

    The cast is torch's float8_e4m3fn conversion; with scale = amax/448 of the
    same draws every quotient is inside the finite range, so no saturation rule
    is involved.
    """
    out = torch.empty(shape, dtype=torch.uint8, device=device)
    flat = out.view(-1)
    for s in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - s)
        x = torch.randn(n, generator=gen, device=device, dtype=torch.float32)
        flat[s:s + n] = (x / scale).to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def fp8_kv_pools(shape, device, gen: torch.Generator):
    """K and V pools of E4M3 codes with one per-tensor scale = amax/448 of all
    the N(0,1) draws behind both pools.  Two passes over the same generator
    state: the first finds amax, the second draws the same numbers again and
    casts them."""
    n = int(np.prod(shape))
    state = gen.get_state()
    amax = _amax_of_draws([n, n], device, gen)
    gen.set_state(state)
    scale = amax / FP8_E4M3_MAX
    k = randn_fp8_codes(shape, scale, device, gen)
    v = randn_fp8_codes(shape, scale, device, gen)
    return k, v, scale


# ----------------------------------------------------------------------------
# context-length distributions
# ----------------------------------------------------------------------------

def ctx_uniform(num_seqs: int, lo: int, hi: int, rng) -> np.ndarray:
    return rng.integers(lo, hi + 1, size=num_seqs).astype(np.int32)


def ctx_lognormal(num_seqs: int, median: float, sigma: float, lo: int, hi: int,
                  rng) -> np.ndarray:
    x = rng.lognormal(mean=math.log(median), sigma=sigma, size=num_seqs)
    return np.clip(np.rint(x), lo, hi).astype(np.int32)


def blocks_needed(ctx: np.ndarray, block_size: int = BLOCK_SIZE) -> np.ndarray:
    return (ctx.astype(np.int64) + block_size - 1) // block_size


def shuffled_block_tables(ctx: np.ndarray, num_blocks: int, max_blocks_per_seq: int,
                          rng, block_size: int = BLOCK_SIZE, fill: int = -1):
    """Give each sequence ceil(ctx/16) distinct physical blocks taken in order
    from one seeded permutation of the pool, so that neighbouring logical
    blocks land at unrelated physical places.  Unused table entries hold
    ``fill`` (-1 by default, so a read past the end is caught)."""
    need = blocks_needed(ctx, block_size)
    assert need.sum() <= num_blocks, "pool too small"
    assert need.max(initial=0) <= max_blocks_per_seq
    perm = rng.permutation(num_blocks).astype(np.int32)
    bt = np.full((len(ctx), max_blocks_per_seq), fill, dtype=np.int32)
    pos = 0
    for i, n in enumerate(need):
        bt[i, :n] = perm[pos:pos + n]
        pos += n
    return bt


# ----------------------------------------------------------------------------
# decode workloads
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class DecodeSpec:
    name: str
    num_seqs: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    q_dtype: int
    kv_dtype: int
    ctx_kind: str                 # "fixed" | "uniform" | "lognormal"
    ctx_args: tuple
    max_ctx: int                  # bound used for max_blocks_per_seq
    pool_factor: float = 1.1      # pool = ceil(factor * blocks used)
    num_blocks: Optional[int] = None  # explicit pool size (overrides factor)
    block_size: int = BLOCK_SIZE
    seed: int = 1000

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def max_blocks_per_seq(self) -> int:
        return -(-self.max_ctx // self.block_size)

    def scaled(self, **kw) -> "DecodeSpec":
        return dataclasses.replace(self, **kw)


# The five workloads.  Seeds are 1000 + the workload's index (1-based).
TINY_FP32 = DecodeSpec("tiny_fp32", 4, 4, 4, 64, F32, F32, "fixed", ((1, 17, 33, 50),),
                       max_ctx=64, num_blocks=32, seed=1001)
LLAMA2_7B_FP16 = DecodeSpec("llama2_7b_fp16", 64, 32, 32, 128, F16, F16, "uniform",
                            (128, 2048), max_ctx=2048, seed=1002)
LLAMA3_70B_GQA_BF16 = DecodeSpec("llama3_70b_gqa_bf16", 128, 64, 8, 128, BF16, BF16,
                                 "lognormal", (2048.0, 0.5, 16, 8192), max_ctx=8192,
                                 seed=1003)
# the same layer with every context at its 8192-token maximum (4.3 GB of K/V)
LLAMA3_70B_GQA_BF16_CTX8K = DecodeSpec("llama3_70b_gqa_bf16_ctx8k", 128, 64, 8, 128, BF16, BF16,
                                       "fixed", ((8192,) * 128,), max_ctx=8192, seed=1003)
# decode half of the mixed continuous-batching step (fp8 KV, per-tensor scale)
MIXED_DECODE_FP8 = DecodeSpec("mixed_step_fp8_decode", 256, 32, 8, 128, BF16, FP8_E4M3,
                              "uniform", (64, 8192), max_ctx=8192, seed=1005)

SPECS = {s.name: s for s in (TINY_FP32, LLAMA2_7B_FP16, LLAMA3_70B_GQA_BF16,
                             LLAMA3_70B_GQA_BF16_CTX8K, MIXED_DECODE_FP8)}

# Draft-token verification ("LLM inference optimization", §五: the target model
# checks K = 5 draft tokens in one forward pass): the Llama-3-70B GQA layer's
# cache and contexts, with SPEC_VERIFY_Q_LEN new queries per sequence whose
# K/V are the last SPEC_VERIFY_Q_LEN tokens of each context.
SPEC_VERIFY_BF16 = DecodeSpec("spec_verify_bf16", 128, 64, 8, 128, BF16, BF16,
                              "lognormal", (2048.0, 0.5, 16, 8192), max_ctx=8192,
                              seed=1006)
SPEC_VERIFY_Q_LEN = 5


def context_lens_for(spec: DecodeSpec, rng) -> np.ndarray:
    if spec.ctx_kind == "fixed":
        vals = np.asarray(spec.ctx_args[0], dtype=np.int32)
        assert len(vals) == spec.num_seqs
        return vals
    if spec.ctx_kind == "uniform":
        lo, hi = spec.ctx_args
        return ctx_uniform(spec.num_seqs, lo, hi, rng)
    if spec.ctx_kind == "lognormal":
        median, sigma, lo, hi = spec.ctx_args
        return ctx_lognormal(spec.num_seqs, median, sigma, lo, hi, rng)
    raise ValueError(spec.ctx_kind)


@dataclasses.dataclass
class DecodeInputs:
    spec: DecodeSpec
    q: torch.Tensor             # [num_seqs, n_q, d] in q dtype
    k_pool: torch.Tensor        # [num_blocks, n_kv, 16, d] (uint8 codes for fp8)
    v_pool: torch.Tensor
    block_tables: torch.Tensor  # int32 [num_seqs, max_blocks_per_seq]
    context_lens: torch.Tensor  # int32 [num_seqs]
    scale: float
    k_scale: float
    v_scale: float

    @property
    def num_blocks(self) -> int:
        return self.k_pool.shape[0]

    def to(self, device) -> "DecodeInputs":
        return dataclasses.replace(
            self, q=self.q.to(device), k_pool=self.k_pool.to(device),
            v_pool=self.v_pool.to(device), block_tables=self.block_tables.to(device),
            context_lens=self.context_lens.to(device))


def make_decode_inputs(spec: DecodeSpec, device="cpu", ctx: Optional[np.ndarray] = None,
                       scale: Optional[float] = None) -> DecodeInputs:
    rng = _rng(spec.seed)
    if ctx is None:
        ctx = context_lens_for(spec, rng)
    ctx = np.asarray(ctx, dtype=np.int32)
    used = int(blocks_needed(ctx, spec.block_size).sum())
    num_blocks = spec.num_blocks if spec.num_blocks is not None else \
        max(1, int(math.ceil(spec.pool_factor * used)))
    bt = shuffled_block_tables(ctx, num_blocks, spec.max_blocks_per_seq, rng,
                               spec.block_size)
    gen = _torch_gen(device, spec.seed)
    pool_shape = (num_blocks, spec.n_kv_heads, spec.block_size, spec.head_dim)
    q = randn_as((spec.num_seqs, spec.n_q_heads, spec.head_dim), spec.q_dtype, device, gen)
    if spec.kv_dtype == FP8_E4M3:
        k_pool, v_pool, kvs = fp8_kv_pools(pool_shape, device, gen)
        k_scale = v_scale = kvs
    else:
        k_pool = randn_as(pool_shape, spec.kv_dtype, device, gen)
        v_pool = randn_as(pool_shape, spec.kv_dtype, device, gen)
        k_scale = v_scale = 1.0
    if scale is None:
        scale = 1.0 / math.sqrt(spec.head_dim)
    return DecodeInputs(spec, q, k_pool, v_pool,
                        torch.from_numpy(bt).to(device),
                        torch.from_numpy(ctx).to(device), scale, k_scale, v_scale)


# Shared-prefix parallel sampling ("LLM inference optimization", §三.2: the
# samples of a prompt share its blocks): 16 prompts x 4 samples, 32 q / 8 kv
# heads, bf16; prompt 2048 + U{1..15} tokens (its full blocks shared by the 4
# samples), then 0-512 divergent tokens per sample in private blocks.
SHARED_PREFIX_BF16 = DecodeSpec("shared_prefix_bf16", 64, 32, 8, 128, BF16, BF16, "fixed",
                                ((),), max_ctx=2048 + 15 + 512 + 16, seed=1004)


def make_shared_prefix_inputs(device="cpu", n_prompts: int = 16, n_samples: int = 4,
                              seed: int = 1004):
    """Decode inputs whose sequences 4p .. 4p+3 share prompt p's full blocks.
    Returns (DecodeInputs, groups) with groups[p] = the prompt's sample
    indices and its number of shared full blocks."""
    rng = _rng(seed)
    plen = 2048 + rng.integers(1, 16, size=n_prompts)
    div = rng.integers(0, 513, size=(n_prompts, n_samples))
    B = BLOCK_SIZE
    shared = [int(l) // B for l in plen]
    ctx = np.array([int(plen[p] + div[p, s]) for p in range(n_prompts)
                    for s in range(n_samples)], np.int32)
    private = [-(-int(ctx[p * n_samples + s]) // B) - shared[p] for p in range(n_prompts)
               for s in range(n_samples)]
    num_blocks = sum(shared) + sum(private)
    perm = rng.permutation(num_blocks).astype(np.int32)
    spec = SHARED_PREFIX_BF16.scaled(num_seqs=n_prompts * n_samples)
    mb = spec.max_blocks_per_seq
    bt = np.full((n_prompts * n_samples, mb), -1, np.int32)
    nxt = 0
    groups = []
    for p in range(n_prompts):
        pref = perm[nxt:nxt + shared[p]]
        nxt += shared[p]
        members = []
        for s in range(n_samples):
            i = p * n_samples + s
            bt[i, :shared[p]] = pref
            k = private[i]
            bt[i, shared[p]:shared[p] + k] = perm[nxt:nxt + k]
            nxt += k
            members.append(i)
        groups.append((members, shared[p]))
    gen = _torch_gen(device, seed)
    pool_shape = (num_blocks, spec.n_kv_heads, B, spec.head_dim)
    q = randn_as((spec.num_seqs, spec.n_q_heads, spec.head_dim), spec.q_dtype, device, gen)
    k_pool = randn_as(pool_shape, spec.kv_dtype, device, gen)
    v_pool = randn_as(pool_shape, spec.kv_dtype, device, gen)
    inp = DecodeInputs(spec, q, k_pool, v_pool, torch.from_numpy(bt).to(device),
                       torch.from_numpy(ctx).to(device), 1.0 / math.sqrt(spec.head_dim), 1.0, 1.0)
    return inp, groups


def make_multi_queries(inp: DecodeInputs, q_len: int, seed: int) -> torch.Tensor:
    """Queries [num_seqs, q_len, n_q, d] for multi-query decode over inp's cache
    (N(0,1) draws rounded to the query dtype)."""
    spec = inp.spec
    gen = _torch_gen(inp.k_pool.device, seed)
    return randn_as((spec.num_seqs, q_len, spec.n_q_heads, spec.head_dim), spec.q_dtype,
                    inp.k_pool.device, gen)


# ----------------------------------------------------------------------------
# new-token K/V for the slot scatter
# ----------------------------------------------------------------------------

def make_new_kv(num_tokens: int, n_kv: int, head_dim: int, dtype_code: int, device,
                seed: int):
    gen = _torch_gen(device, seed)
    k = randn_as((num_tokens, n_kv, head_dim), dtype_code, device, gen)
    v = randn_as((num_tokens, n_kv, head_dim), dtype_code, device, gen)
    return k, v


def slots_from_positions(block_tables: np.ndarray, seq_ids: np.ndarray,
                         positions: np.ndarray, block_size: int = BLOCK_SIZE) -> np.ndarray:
    """slot_mapping entries for (sequence, logical position) pairs.

    This is the encoding the C ABI defines for a slot: the physical block id
    the sequence's table holds for the position's logical block, times the
    block size, plus the offset inside the block."""
    blk = block_tables[seq_ids, positions // block_size].astype(np.int64)
    return blk * block_size + (positions % block_size)


# ----------------------------------------------------------------------------
# chunked-prefill workload (the prefill half of the mixed step)
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class PrefillSpec:
    name: str
    n_chunks: int
    chunk_len: int
    history: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    q_dtype: int
    kv_dtype: int
    extra_blocks: int = 0
    block_size: int = BLOCK_SIZE
    seed: int = 1005


MIXED_PREFILL_FP8 = PrefillSpec("mixed_step_fp8_prefill", 2, 512, 4096, 32, 8, 128,
                                BF16, FP8_E4M3, seed=2005)


@dataclasses.dataclass
class PrefillInputs:
    spec: PrefillSpec
    q: torch.Tensor                # [total_q, n_q, d]
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    block_tables: torch.Tensor     # int32 [n_chunks, max_blocks]
    query_start_loc: torch.Tensor  # int32 [n_chunks + 1]
    context_lens: torch.Tensor     # int32 [n_chunks] = history + chunk length
    scale: float
    k_scale: float
    v_scale: float


def make_prefill_inputs(spec: PrefillSpec, device="cpu",
                        chunk_lens: Optional[list] = None,
                        histories: Optional[list] = None) -> PrefillInputs:
    rng = _rng(spec.seed)
    chunk_lens = list(chunk_lens or [spec.chunk_len] * spec.n_chunks)
    histories = list(histories or [spec.history] * spec.n_chunks)
    ctx = np.asarray([h + c for h, c in zip(histories, chunk_lens)], dtype=np.int32)
    used = int(blocks_needed(ctx, spec.block_size).sum())
    num_blocks = used + spec.extra_blocks + 1
    max_blocks = int(blocks_needed(ctx, spec.block_size).max())
    bt = shuffled_block_tables(ctx, num_blocks, max_blocks, rng, spec.block_size)
    qsl = np.zeros(len(chunk_lens) + 1, dtype=np.int32)
    qsl[1:] = np.cumsum(chunk_lens)
    gen = _torch_gen(device, spec.seed)
    q = randn_as((int(qsl[-1]), spec.n_q_heads, spec.head_dim), spec.q_dtype, device, gen)
    pool_shape = (num_blocks, spec.n_kv_heads, spec.block_size, spec.head_dim)
    if spec.kv_dtype == FP8_E4M3:
        k_pool, v_pool, kvs = fp8_kv_pools(pool_shape, device, gen)
        k_scale = v_scale = kvs
    else:
        k_pool = randn_as(pool_shape, spec.kv_dtype, device, gen)
        v_pool = randn_as(pool_shape, spec.kv_dtype, device, gen)
        k_scale = v_scale = 1.0
    return PrefillInputs(spec, q, k_pool, v_pool, torch.from_numpy(bt).to(device),
                         torch.from_numpy(qsl).to(device), torch.from_numpy(ctx).to(device),
                         1.0 / math.sqrt(spec.head_dim), k_scale, v_scale)


# ----------------------------------------------------------------------------
# byte model (for reporting throughput; not part of the computation)
# ----------------------------------------------------------------------------

def kv_bytes_per_token(n_layers: int, n_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """K and V bytes one token occupies across all layers: 2 * L * H_kv * d * b
    ("LLM inference optimization", §二.1.2 per-token formula, read with the
    KV head count as its worked example uses)."""
    return 2 * n_layers * n_kv_heads * head_dim * elem_bytes


def block_bytes(block_size: int, n_layers: int, n_kv_heads: int, head_dim: int,
                elem_bytes: int) -> int:
    """Bytes of one block across all layers: 2 * B * L * H_kv * d * b
    ("vLLM explained", "Block 的大小怎麼決定")."""
    return 2 * block_size * n_layers * n_kv_heads * head_dim * elem_bytes


def decode_algorithmic_bytes(context_lens: np.ndarray, n_q: int, n_kv: int, head_dim: int,
                             q_elem: int, kv_elem: int, out_elem: Optional[int] = None) -> int:
    """K and V of every valid context token (not whole blocks) + q + out."""
    out_elem = q_elem if out_elem is None else out_elem
    toks = int(np.asarray(context_lens, dtype=np.int64).sum())
    kv = toks * 2 * n_kv * head_dim * kv_elem
    qo = len(context_lens) * n_q * head_dim * (q_elem + out_elem)
    return kv + qo
