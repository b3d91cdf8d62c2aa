"""GPU parity of pa_decode_shared_prefix: decode in which each group of
sequences whose tables start with the same blocks (the samples of one prompt,
"LLM inference optimization", §三.2) reads those blocks once for the group.
The result is pa_decode's: checked against the fp64 oracle, against pa_decode,
and bit for bit against pa_decode when no group is given."""
import numpy as np
import pytest
import torch

from pagedattention_paged_kv_pa_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda_device):
    from pagedattention_paged_kv_pa_b200 import binding
    return binding


def _run(B, inp, dev, groups=None, dev_err=None):
    d = inp.to(dev)
    out = torch.empty_like(d.q)
    err = torch.zeros(1, dtype=torch.int32, device=dev) if dev_err is None else dev_err
    if groups is None:
        B.pa_decode(out, d.q, d.k_pool, d.v_pool, d.block_tables, d.context_lens, d.scale,
                    d.k_scale, d.v_scale, dev_err=err)
    else:
        B.pa_decode_shared_prefix(out, d.q, d.k_pool, d.v_pool, d.block_tables, d.context_lens,
                                  d.scale, groups, d.k_scale, d.v_scale, dev_err=err)
    torch.cuda.synchronize(dev)
    return out.float().cpu().numpy().astype(np.float64), int(err.item())


def _grouped_inputs(n_prompts, n_samples, prefix_lens, extra, G, d, kv_dt, seed):
    """Prompts whose samples share the prompt's full blocks, then private
    blocks; contexts = prefix + extra[p][s] tokens."""
    rng = np.random.default_rng(seed)
    n_kv = 2
    ctx = np.array([prefix_lens[p] + extra[p][s] for p in range(n_prompts)
                    for s in range(n_samples)], np.int32)
    shared = [l // 16 for l in prefix_lens]
    own = [-(-int(ctx[p * n_samples + s]) // 16) - shared[p] for p in range(n_prompts)
           for s in range(n_samples)]
    nb = sum(shared) + sum(own) + 8
    perm = rng.permutation(nb).astype(np.int32)
    mb = int(-(-ctx.max() // 16)) + 1
    bt = np.full((len(ctx), mb), -1, np.int32)
    nxt = 0
    for p in range(n_prompts):
        pre = perm[nxt:nxt + shared[p]]
        nxt += shared[p]
        for s in range(n_samples):
            i = p * n_samples + s
            bt[i, :shared[p]] = pre
            bt[i, shared[p]:shared[p] + own[i]] = perm[nxt:nxt + own[i]]
            nxt += own[i]
    # the generator's own pool (sized for unshared tables) is large enough for
    # ids 0 .. nb-1; its tables are replaced by the shared ones below
    spec = W.DecodeSpec("grp", len(ctx), n_kv * G, n_kv, d, W.BF16, kv_dt, "fixed", (ctx,),
                        max_ctx=mb * 16, seed=seed)
    inp = W.make_decode_inputs(spec, ctx=ctx)
    assert inp.num_blocks >= nb
    return W.DecodeInputs(spec, inp.q, inp.k_pool, inp.v_pool, torch.from_numpy(bt),
                          torch.from_numpy(ctx), inp.scale, inp.k_scale, inp.v_scale)


def test_shared_prefix_workload_matches_oracle_and_decode(B, cuda_device):
    inp, _ = W.make_shared_prefix_inputs("cpu")
    groups = B.prefix_groups(inp.block_tables, inp.context_lens, 32, 8, W.BF16)
    assert len(groups["members"]) == 16 and groups["width"] == 4
    gpu, err = _run(B, inp, cuda_device, groups)
    assert err == 0
    ref = P.oracle_decode(inp)
    P.assert_close(gpu, ref, W.BF16, W.BF16, "shared-prefix decode vs oracle")
    plain, _ = _run(B, inp, cuda_device)
    P.assert_close(gpu, plain, W.BF16, W.BF16, "shared-prefix decode vs pa_decode")


@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("kv_dt", [W.BF16, W.FP8_E4M3])
def test_groups_grid(B, cuda_device, G, d, kv_dt):
    part = 2048 if kv_dt == W.FP8_E4M3 else 1024
    n_samples = 3
    # prompt 0: exactly two partitions shared, one sample ending there (its whole
    # context is shared: written straight to out when it is one partition, here
    # two); prompt 1: one partition + 37 tokens shared, contexts beyond
    prefix = [2 * part, part + 37]
    extra = [[0, 5, 300], [1, 700, 16]]
    inp = _grouped_inputs(2, n_samples, prefix, extra, G, d, kv_dt, seed=40 + G + d)
    groups = B.prefix_groups(inp.block_tables, inp.context_lens, inp.spec.n_q_heads,
                             inp.spec.n_kv_heads, kv_dt)
    assert len(groups["members"]) == 2
    gpu, err = _run(B, inp, cuda_device, groups)
    assert err == 0
    ref = P.oracle_decode(inp)
    P.assert_close(gpu, ref, W.BF16, kv_dt, f"groups G={G} d={d} kv={kv_dt}")


def test_single_partition_members_are_written_directly(B, cuda_device):
    # every member's context is exactly the one shared partition
    inp = _grouped_inputs(1, 4, [1024], [[0, 0, 0, 0]], 4, 128, W.BF16, seed=9)
    groups = B.prefix_groups(inp.block_tables, inp.context_lens, 8, 2, W.BF16)
    gpu, err = _run(B, inp, cuda_device, groups)
    assert err == 0
    P.assert_close(gpu, P.oracle_decode(inp), W.BF16, W.BF16, "one shared partition")


def test_no_groups_is_decode_bit_for_bit(B, cuda_device):
    inp, _ = W.make_shared_prefix_inputs("cpu")
    none = {"members": torch.zeros((0, 4), dtype=torch.int32),
            "shared_blocks": torch.zeros(0, dtype=torch.int32),
            "seq_group": torch.full((inp.spec.num_seqs,), -1, dtype=torch.int32), "width": 4}
    a, _ = _run(B, inp, cuda_device, none)
    b, _ = _run(B, inp, cuda_device)
    assert np.array_equal(a, b)


def test_member_index_out_of_range_is_flagged(B, cuda_device):
    inp = _grouped_inputs(1, 2, [1024], [[10, 20]], 4, 128, W.BF16, seed=3)
    groups = B.prefix_groups(inp.block_tables, inp.context_lens, 8, 2, W.BF16)
    groups["members"] = groups["members"].clone()
    groups["members"][0, 0] = 1 << 20   # not a sequence
    _, err = _run(B, inp, cuda_device, groups)
    assert err & 1  # PA_DEVERR_BLOCK_ID
