"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin whose host program owns all device memory, a loop that
cannot pay for cudaMalloc's implicit synchronisation) have no workspace to
hand to pa_decode, so this entry point keeps its partition results in a
scratch array that is part of the library.  The test calls it through the C
ABI twice in a row, on different inputs, and checks each result against
pa_decode with a workspace of its own, within the parity tolerances.  It also
checks that a request too big for the built-in scratch is refused before any
launch.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from pagedattention_paged_kv_pa_b200 import workloads as W
from tests import parity as P

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


def test_noalloc_matches_pa_decode_on_two_calls(cuda_device):
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
        ref = torch.empty_like(inp.q)
        B.pa_decode(ref, inp.q, inp.k_pool, inp.v_pool, inp.block_tables, inp.context_lens,
                    inp.scale, inp.k_scale, inp.v_scale)
        out = torch.full_like(inp.q, float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        assert _call_noalloc(B, out, inp, err) == B.PA_OK
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        P.assert_close(out.float().cpu().numpy(), ref.float().cpu().numpy(), spec.q_dtype,
                       spec.kv_dtype, f"no-alloc call {k + 1}")


def test_noalloc_refuses_requests_beyond_its_scratch(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding as B
    cap = B.lib.pa_decode_noalloc_scratch_bytes()
    # 128 sequences x 64 q heads at 8K context need ~68 MB of partition results
    assert B.pa_decode_workspace_size(128, 64, 128, 512) > cap
    v = ctypes.c_void_p(16)
    st = B.lib.pa_decode_noalloc(v, v, v, v, v, v, 0.1, 16, 64, 8, 128, 128, 512, 1000,
                                 B.PA_BF16, B.PA_BF16, 1.0, 1.0, None, None)
    assert st == B.PA_ERR_UNSUPPORTED
