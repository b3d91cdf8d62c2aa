"""The C ABI library loads without a GPU, exports every symbol include/pa.h
declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def B():
    from pagedattention_paged_kv_pa_b200 import build
    build.build()
    from pagedattention_paged_kv_pa_b200 import binding
    return binding


def test_header_declares_the_hot_path_calls():
    names = _declared()
    for n in ("pa_decode", "pa_reshape_and_cache", "pa_copy_blocks", "pa_prefill_paged",
              "pa_alloc_create", "pa_alloc_prepare_write"):
        assert n in names


def test_library_exports_every_declared_symbol(B):
    names = _declared()
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(l.split()[-1] for l in out.splitlines() if " T " in l)
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(B.EXPORTS) == set(names)


def test_library_needs_no_cuda_driver_to_load(B):
    out = subprocess.run(["ldd", B.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out  # driver entry points are fetched at run time
    assert B.lib.pa_abi_version() == 2


def test_status_strings(B):
    assert B.status_string(0) == "ok"
    assert "unsupported" in B.status_string(2)


def _dec(B, **kw):
    a = dict(out=16, q=16, k=16, v=16, bt=16, cl=16, scale=0.1, bs=16, nq=8, nkv=2, d=128,
             ns=4, mb=4, nb=10, qdt=B.PA_BF16, kvdt=B.PA_BF16, ks=1.0, vs=1.0, ws=None,
             wsb=0, err=None, st=None)
    a.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return B.lib.pa_decode(v(a["out"]), v(a["q"]), v(a["k"]), v(a["v"]), v(a["bt"]), v(a["cl"]),
                           a["scale"], a["bs"], a["nq"], a["nkv"], a["d"], a["ns"], a["mb"],
                           a["nb"], a["qdt"], a["kvdt"], a["ks"], a["vs"], v(a["ws"]), a["wsb"],
                           v(a["err"]), v(a["st"]))


def test_decode_argument_errors_are_synchronous(B):
    # none of these reach a launch, so they are safe without a GPU
    assert _dec(B, bs=32) == B.PA_ERR_UNSUPPORTED
    assert _dec(B, d=96) == B.PA_ERR_UNSUPPORTED
    assert _dec(B, nq=6, nkv=4) == B.PA_ERR_INVALID_ARG
    assert _dec(B, nq=32, nkv=2) == B.PA_ERR_UNSUPPORTED          # group 16 > 8
    assert _dec(B, qdt=B.PA_F32, kvdt=B.PA_BF16) == B.PA_ERR_UNSUPPORTED
    assert _dec(B, qdt=B.PA_FP8_E4M3, kvdt=B.PA_FP8_E4M3) == B.PA_ERR_UNSUPPORTED
    assert _dec(B, q=None) == B.PA_ERR_INVALID_ARG
    assert _dec(B, q=24) == B.PA_ERR_INVALID_ARG                  # misaligned pointer
    assert _dec(B, mb=0) == B.PA_ERR_INVALID_ARG
    assert _dec(B, ns=0) == B.PA_OK                               # nothing to do
    assert _dec(B, ns=65536) == B.PA_ERR_UNSUPPORTED              # beyond the grid's z
    # more than one partition needs a workspace of the advertised size
    ws = B.pa_decode_workspace_size(4, 8, 128, 512)
    assert ws > 0
    assert _dec(B, mb=512) == B.PA_ERR_INVALID_ARG
    assert _dec(B, mb=512, ws=16, wsb=ws - 1) == B.PA_ERR_INVALID_ARG
    assert _dec(B, kvdt=B.PA_FP8_E4M3, ks=0.0) == B.PA_ERR_INVALID_ARG
    assert B.pa_decode_workspace_size(4, 8, 128, 32) == 0          # a single partition


def _multi(B, q_len, **kw):
    a = dict(out=16, q=16, k=16, v=16, bt=16, cl=16, scale=0.1, bs=16, nq=8, nkv=2, d=128,
             ns=4, mb=4, nb=10, qdt=B.PA_BF16, kvdt=B.PA_BF16, ks=1.0, vs=1.0, ws=None,
             wsb=0, err=None, st=None)
    a.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return B.lib.pa_decode_multi(v(a["out"]), v(a["q"]), v(a["k"]), v(a["v"]), v(a["bt"]),
                                 v(a["cl"]), a["scale"], a["bs"], a["nq"], a["nkv"], a["d"],
                                 a["ns"], q_len, a["mb"], a["nb"], a["qdt"], a["kvdt"], a["ks"],
                                 a["vs"], v(a["ws"]), a["wsb"], v(a["err"]), v(a["st"]))


def test_multi_query_decode_argument_errors_are_synchronous(B):
    assert _multi(B, 0) == B.PA_ERR_INVALID_ARG
    assert _multi(B, 9) == B.PA_ERR_INVALID_ARG
    assert _multi(B, 2, qdt=B.PA_F32, kvdt=B.PA_F32) == B.PA_ERR_UNSUPPORTED
    assert _multi(B, 2, bs=32) == B.PA_ERR_UNSUPPORTED
    assert _multi(B, 2, q=None) == B.PA_ERR_INVALID_ARG
    assert _multi(B, 2, ns=0) == B.PA_OK
    # the workspace holds every (query, q head) row of a sequence
    ws = B.pa_decode_workspace_size(4, 8 * 3, 128, 512)
    assert ws > 2 * B.pa_decode_workspace_size(4, 8, 128, 512)
    assert _multi(B, 3, mb=512, ws=16, wsb=ws - 1) == B.PA_ERR_INVALID_ARG


def test_swap_argument_errors_are_synchronous(B):
    v = ctypes.c_void_p
    L = B.lib
    args = lambda **k: dict(dk=16, dv=16, sk=16, sv=16, pr=16, n=2, nkv=8, d=128, bs=16, sn=10,
                            dn=10, dt=B.PA_BF16, **k)

    def call(a):
        return L.pa_swap_blocks(v(a["dk"]) if a["dk"] else None, v(a["dv"]), v(a["sk"]),
                                v(a["sv"]), v(a["pr"]) if a["pr"] else None, a["n"], a["nkv"],
                                a["d"], a["bs"], a["sn"], a["dn"], a["dt"], None, None)
    assert call({**args(), "bs": 32}) == B.PA_ERR_UNSUPPORTED
    assert call({**args(), "n": -1}) == B.PA_ERR_INVALID_ARG
    assert call({**args(), "sn": 0}) == B.PA_ERR_INVALID_ARG
    assert call({**args(), "n": 0}) == B.PA_OK
    assert call({**args(), "dk": 0}) == B.PA_ERR_INVALID_ARG
    assert call({**args(), "pr": 0}) == B.PA_ERR_INVALID_ARG
    assert call({**args(), "sk": 24}) == B.PA_ERR_INVALID_ARG        # misaligned pool


def test_cache_op_argument_errors_are_synchronous(B):
    v = ctypes.c_void_p
    L = B.lib
    assert L.pa_reshape_and_cache(v(16), v(16), v(16), v(16), v(16), 4, 2, 128, 8, 10,
                                  B.PA_BF16, B.PA_BF16, 1.0, 1.0, None, None) == B.PA_ERR_UNSUPPORTED
    assert L.pa_reshape_and_cache(v(16), v(16), v(16), v(16), v(16), 4, 2, 128, 16, 10,
                                  B.PA_BF16, B.PA_F16, 1.0, 1.0, None, None) == B.PA_ERR_UNSUPPORTED
    assert L.pa_reshape_and_cache(v(16), v(16), v(16), v(16), v(16), 4, 2, 128, 16, 10,
                                  B.PA_BF16, B.PA_FP8_E4M3, 0.0, 1.0, None, None) == B.PA_ERR_INVALID_ARG
    assert L.pa_reshape_and_cache(None, None, None, None, None, 0, 2, 128, 16, 10,
                                  B.PA_BF16, B.PA_BF16, 1.0, 1.0, None, None) == B.PA_OK
    assert L.pa_copy_blocks(v(16), v(16), None, 3, 8, 128, 16, 10, B.PA_BF16, None,
                            None) == B.PA_ERR_INVALID_ARG
    assert L.pa_copy_blocks(None, None, None, 0, 8, 128, 16, 10, B.PA_BF16, None,
                            None) == B.PA_OK


def test_prefix_groups_from_host_tables(B):
    # bf16 caches: 1024-token partitions = 64 blocks.  Sequences 0-3 start with
    # block 7; 0-2 share 70 blocks, 3 leaves them after 64; 4 is alone; 5 starts
    # with block 7 too but holds less than one partition; 6, 7 share 100 blocks.
    mb = 110
    bt = np.full((8, mb), -1, np.int32)
    pre = np.arange(1000, 1000 + 100, dtype=np.int32)
    pre[0] = 7
    for s in (0, 1, 2, 3):
        bt[s, :70] = pre[:70]
    bt[3, 64:70] = np.arange(5000, 5006)
    bt[4, :70] = np.arange(6000, 6070)
    bt[5, :10] = pre[:10]
    other = np.arange(8000, 8105, dtype=np.int32)
    bt[6, :105] = other
    bt[7, :100] = other[:100]
    bt[7, 100:103] = [9000, 9001, 9002]
    ctx = np.array([70 * 16, 70 * 16 - 5, 70 * 16, 70 * 16, 70 * 16, 150, 105 * 16, 103 * 16],
                   np.int32)
    g = B.prefix_groups(torch.from_numpy(bt), torch.from_numpy(ctx), 32, 8, B.PA_BF16)
    assert g["width"] == 4
    assert g["members"].tolist() == [[0, 1, 2, 3], [6, 7, -1, -1]]
    # 1's context ends 5 tokens into its 70th block: 69 full blocks; 3 diverges at 64
    assert g["shared_blocks"].tolist() == [64, 100]
    assert g["seq_group"].tolist() == [0, 0, 0, 0, -1, -1, 1, 1]
    # groups are at most 32 / G wide: with G = 8, 4 members
    bt2 = np.tile(bt[6], (6, 1))
    g2 = B.prefix_groups(torch.from_numpy(bt2), torch.full((6,), 1600, dtype=torch.int32),
                         64, 8, B.PA_BF16)
    assert g2["members"].tolist() == [[0, 1, 2, 3], [4, 5, -1, -1]]


def _pre(B, **kw):
    a = dict(out=16, q=16, k=16, v=16, bt=16, qsl=16, cl=16, scale=0.1, bs=16, nq=8, nkv=2,
             d=128, nc=3, mcl=64, mb=5, nb=10, qdt=B.PA_BF16, kvdt=B.PA_FP8_E4M3, ks=1.0,
             vs=1.0, ws=None, wsb=0, err=None, st=None)
    a.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return B.lib.pa_prefill_paged(v(a["out"]), v(a["q"]), v(a["k"]), v(a["v"]), v(a["bt"]),
                                  v(a["qsl"]), v(a["cl"]), a["scale"], a["bs"], a["nq"],
                                  a["nkv"], a["d"], a["nc"], a["mcl"], a["mb"], a["nb"],
                                  a["qdt"], a["kvdt"], a["ks"], a["vs"], v(a["ws"]), a["wsb"],
                                  v(a["err"]), v(a["st"]))


def test_prefill_workspace_size_and_refusals(B):
    # K and V, f16, per (chunk, kv head): max_blocks * 16 keys rounded up to 128 rows
    assert B.pa_prefill_workspace_size(3, 2, 128, 5) == 2 * 3 * 2 * 128 * 128 * 2
    assert B.pa_prefill_workspace_size(3, 2, 128, 8) == 2 * 3 * 2 * 128 * 128 * 2
    assert B.pa_prefill_workspace_size(3, 2, 128, 9) == 2 * 3 * 2 * 256 * 128 * 2
    assert B.pa_prefill_workspace_size(0, 2, 128, 9) == 0
    assert B.pa_prefill_workspace_size(3, 2, 64, 9) == 0     # head_dim 128 only
    assert B.pa_prefill_workspace_size(3, 2, 128, 9, 32) == 0
    need = B.pa_prefill_workspace_size(3, 2, 128, 5)
    # none of these reach a launch, so they are safe without a GPU
    assert _pre(B, ws=4096, wsb=need - 16) == B.PA_ERR_INVALID_ARG   # too small
    assert _pre(B, ws=4104, wsb=need) == B.PA_ERR_INVALID_ARG        # misaligned
    assert _pre(B, d=64) == B.PA_ERR_UNSUPPORTED
    assert _pre(B, nq=6, nkv=4) == B.PA_ERR_INVALID_ARG
    assert _pre(B, nb=1 << 27, nkv=2) == B.PA_ERR_UNSUPPORTED        # pool rows >= 2^31
    assert _pre(B, nc=0) == B.PA_OK                                   # nothing to do
    # workspace rows (chunks x kv heads x max_blocks*16 rounded up to 128) >= 2^31
    big = dict(nc=65535, nq=16, nkv=16, mb=2048)
    need_big = B.pa_prefill_workspace_size(65535, 16, 128, 2048)
    assert need_big == 2 * 65535 * 16 * 32768 * 128 * 2
    assert _pre(B, ws=4096, wsb=need_big, **big) == B.PA_ERR_UNSUPPORTED
