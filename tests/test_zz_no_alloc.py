"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin whose host program owns all device memory, a loop that
cannot pay for cudaMalloc's implicit synchronisation) have no workspace to
hand to pa_decode, so this entry point keeps its partition results in a
scratch array that is part of the library.  It runs pa_decode's own kernels,
so the tests call it through the C ABI twice in a row, on different inputs,
and require each result to equal pa_decode's (with a workspace of its own)
bit for bit; they check that a warmed-up call changes the device's free
memory by nothing, that a request whose scratch need is within a few KB of
the built-in size works, and that one beyond it is refused before any launch.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from pagedattention_paged_kv_pa_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _call_noalloc(B, out, inp, err):
    v = lambda t: ctypes.c_void_p(t.data_ptr())
    s = inp.spec
    return B.lib.pa_decode_noalloc(
        v(out), v(inp.q), v(inp.k_pool), v(inp.v_pool), v(inp.block_tables),
        v(inp.context_lens), inp.scale, 16, s.n_q_heads, s.n_kv_heads, s.head_dim,
        s.num_seqs, inp.block_tables.shape[1], inp.num_blocks, s.q_dtype,
        B.dtype_code(inp.k_pool), inp.k_scale, inp.v_scale, v(err),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _reference(B, inp):
    ref = torch.empty_like(inp.q)
    B.pa_decode(ref, inp.q, inp.k_pool, inp.v_pool, inp.block_tables, inp.context_lens,
                inp.scale, inp.k_scale, inp.v_scale)
    return ref


def _noalloc(B, inp, dev):
    out = torch.full_like(inp.q, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    assert _call_noalloc(B, out, inp, err) == B.PA_OK
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out


def test_noalloc_equals_pa_decode_on_two_calls(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding as B
    cases = [
        (W.LLAMA3_70B_GQA_BF16.scaled(num_seqs=8),
         np.array([16, 700, 2048, 5000, 8192, 1, 513, 3333], np.int32)),
        (W.MIXED_DECODE_FP8.scaled(num_seqs=6),
         np.array([64, 900, 4097, 8000, 512, 2500], np.int32)),
    ]
    for k, (spec, ctx) in enumerate(cases):
        inp = W.make_decode_inputs(spec, device=cuda_device, ctx=ctx)
        need = B.pa_decode_workspace_size(spec.num_seqs, spec.n_q_heads, spec.head_dim,
                                          inp.block_tables.shape[1])
        assert 0 < need <= B.lib.pa_decode_noalloc_scratch_bytes()
        ref = _reference(B, inp)
        out = _noalloc(B, inp, cuda_device)
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {k + 1}"


def test_noalloc_allocates_nothing(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding as B
    spec = W.LLAMA3_70B_GQA_BF16.scaled(num_seqs=4)
    inp = W.make_decode_inputs(spec, device=cuda_device,
                               ctx=np.array([3000, 17, 8192, 1025], np.int32))
    _noalloc(B, inp, cuda_device)  # the first call may load the library's module
    free0 = torch.cuda.mem_get_info(cuda_device)[0]
    for _ in range(3):
        _noalloc(B, inp, cuda_device)
    assert torch.cuda.mem_get_info(cuda_device)[0] == free0


def test_noalloc_at_the_scratch_limit(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding as B
    cap = B.lib.pa_decode_noalloc_scratch_bytes()
    # 63 sequences x 64 q heads x 8 partitions of an 8K table: 32,256 rows of
    # 128 fp32 outputs plus a (max, sum) pair, 4 KiB short of the 16 MiB
    spec = W.LLAMA3_70B_GQA_BF16.scaled(num_seqs=63)
    need = B.pa_decode_workspace_size(63, 64, 128, spec.max_blocks_per_seq)
    assert need <= cap and cap - need <= 8192
    ctx = np.random.default_rng(17).integers(1, 8193, size=63).astype(np.int32)
    ctx[:3] = (8192, 8191, 7169)  # every partition of the table in use
    inp = W.make_decode_inputs(spec, device=cuda_device, ctx=ctx)
    ref = _reference(B, inp)
    for _ in range(2):
        out = _noalloc(B, inp, cuda_device)
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_noalloc_refuses_requests_beyond_its_scratch(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding as B
    cap = B.lib.pa_decode_noalloc_scratch_bytes()
    # one sequence more than the case at the limit
    assert B.pa_decode_workspace_size(64, 64, 128, 512) > cap
    v = ctypes.c_void_p(16)
    st = B.lib.pa_decode_noalloc(v, v, v, v, v, v, 0.1, 16, 64, 8, 128, 64, 512, 1000,
                                 B.PA_BF16, B.PA_BF16, 1.0, 1.0, None, None)
    assert st == B.PA_ERR_UNSUPPORTED
