"""The error path of the kernels' bounded waits, exercised without a GPU
fault.  pa_test_decode_timeout runs pa_decode with every wait of the
partition kernel limited to a couple of milliseconds and with each CTA's
producer leaving one tile's shared-memory stage unfilled, as if its load had
never arrived (a flag that nothing sets).  The waits on that stage run out:
the kernel must flag PA_DEVERR_TIMEOUT, let the loads it did issue land and
return, and the next ordinary call on the same context must match the oracle.
"""
import time

import numpy as np
import pytest
import torch

from pagedattention_paged_kv_pa_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

PA_DEVERR_TIMEOUT = 4


@pytest.fixture(scope="module")
def B(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding
    return binding


@pytest.mark.parametrize("kv_dt", [W.BF16, W.FP8_E4M3])
def test_a_wait_that_runs_out_is_flagged_and_the_context_stays_usable(B, cuda_device, kv_dt):
    # partitions of 64-128 blocks, one of 13 blocks and one of 5 (which never
    # reaches the skipped tile 5 and completes normally)
    ctx = np.array([3000, 200, 1100], np.int32)
    spec = W.DecodeSpec("timeout", 3, 16, 2, 128, W.BF16, kv_dt, "fixed", (ctx,), max_ctx=3072,
                        seed=501)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    d = inp.to(cuda_device)
    out = torch.empty_like(d.q)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    t0 = time.monotonic()
    B.pa_test_decode_timeout(out, d.q, d.k_pool, d.v_pool, d.block_tables, d.context_lens,
                             d.scale, skip_tile=5, wait_limit_us=2000, k_scale=d.k_scale,
                             v_scale=d.v_scale, dev_err=err)
    torch.cuda.synchronize()
    assert time.monotonic() - t0 < 30
    assert int(err.item()) & PA_DEVERR_TIMEOUT
    gpu, e2 = P.run_decode(inp, cuda_device)
    assert e2 == 0
    P.assert_close(gpu, P.oracle_decode(inp), W.BF16, kv_dt, "decode after a timed-out call")


def test_the_hook_refuses_bad_arguments(B, cuda_device):
    spec = W.DecodeSpec("timeout_args", 1, 8, 2, 128, W.BF16, W.BF16, "fixed",
                        (np.array([40], np.int32),), max_ctx=64)
    d = W.make_decode_inputs(spec).to(cuda_device)
    out = torch.empty_like(d.q)
    for skip, limit in ((-1, 2000), (0, 0), (0, 2_000_000)):
        with pytest.raises(B.PAError):
            B.pa_test_decode_timeout(out, d.q, d.k_pool, d.v_pool, d.block_tables,
                                     d.context_lens, d.scale, skip_tile=skip,
                                     wait_limit_us=limit)
