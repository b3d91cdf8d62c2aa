"""Pins for the oracle's paged attention (CPU only).

Each test checks the oracle against something other than itself:
closed forms, NumPy's textbook softmax(q K^T * scale) V on contiguous
tensors, invariants the pages state (paging changes nothing; blocks need not
be contiguous; shared blocks read like private copies) and the pages' worked
block-table example.
"""
import os

import numpy as np
import pytest
import torch

import oracle as orc
from pagedattention_paged_kv_pa_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
B = 16


# ---------------------------------------------------------------------------
# helpers written independently of the oracle
# ---------------------------------------------------------------------------

def numpy_attention(q, K, V, scale):
    """softmax(q K^T * scale) V for one query vector (textbook, NumPy)."""
    s = (K @ q) * scale
    w = np.exp(s - s.max())
    return (w[:, None] * V).sum(0) / w.sum()


def place_in_pool(seqs_K, seqs_V, n_kv, d, num_blocks, rng, dtype=np.float32):
    """Build a paged pool from contiguous per-sequence K/V [n_kv, ctx, d].

    Padding each sequence to whole blocks and reshaping to
    [n_kv, blocks, 16, d] gives one 16-token tile per logical block; the tiles
    are then dropped at physical ids drawn from a permutation of the pool.
    """
    kp = rng.standard_normal((num_blocks, n_kv, B, d)).astype(dtype)
    vp = rng.standard_normal((num_blocks, n_kv, B, d)).astype(dtype)
    perm = rng.permutation(num_blocks)
    nblk = [-(-K.shape[1] // B) for K in seqs_K]
    bt = np.full((len(seqs_K), max(max(nblk), 1)), -1, dtype=np.int32)
    pos = 0
    for i, (K, V) in enumerate(zip(seqs_K, seqs_V)):
        n = nblk[i]
        ids = perm[pos:pos + n]
        pos += n
        bt[i, :n] = ids
        pad = n * B - K.shape[1]
        Kt = np.pad(K, ((0, 0), (0, pad), (0, 0))).reshape(n_kv, n, B, d).transpose(1, 0, 2, 3)
        Vt = np.pad(V, ((0, 0), (0, pad), (0, 0))).reshape(n_kv, n, B, d).transpose(1, 0, 2, 3)
        # the tail of a partial last block keeps whatever the pool held
        keep_k, keep_v = kp[ids].copy(), vp[ids].copy()
        kp[ids] = Kt
        vp[ids] = Vt
        if pad:
            kp[ids[-1], :, B - pad:] = keep_k[-1][:, B - pad:]
            vp[ids[-1], :, B - pad:] = keep_v[-1][:, B - pad:]
    return kp, vp, bt


def random_case(ctxs, n_q, n_kv, d, seed, extra_blocks=5):
    rng = np.random.default_rng(seed)
    Ks = [rng.standard_normal((n_kv, c, d)) for c in ctxs]
    Vs = [rng.standard_normal((n_kv, c, d)) for c in ctxs]
    # store as float32 so the pool holds exactly the values we attend with
    Ks = [k.astype(np.float32) for k in Ks]
    Vs = [v.astype(np.float32) for v in Vs]
    nb = sum(-(-c // B) for c in ctxs) + extra_blocks
    kp, vp, bt = place_in_pool(Ks, Vs, n_kv, d, nb, rng)
    q = rng.standard_normal((len(ctxs), n_q, d)).astype(np.float32)
    return q, Ks, Vs, kp, vp, bt, np.asarray(ctxs, dtype=np.int32)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def test_ctx1_returns_v0_exactly():
    q, Ks, Vs, kp, vp, bt, cl = random_case([1, 1, 1], 4, 2, 64, seed=10)
    out = orc.paged_decode(q, kp, vp, bt, cl, 0.125, orc.F32, orc.F32)
    for s in range(3):
        for h in range(4):
            assert np.array_equal(out[s, h], Vs[s][h // 2, 0].astype(np.float64))


def test_zero_query_gives_mean_of_v():
    q, Ks, Vs, kp, vp, bt, cl = random_case([37, 100], 2, 2, 64, seed=11)
    q[:] = 0
    out = orc.paged_decode(q, kp, vp, bt, cl, 0.125, orc.F32, orc.F32)
    for s in range(2):
        for h in range(2):
            np.testing.assert_allclose(out[s, h], Vs[s][h].astype(np.float64).mean(0),
                                       rtol=0, atol=1e-14)


def test_equal_values_give_that_value():
    q, Ks, Vs, kp, vp, bt, cl = random_case([50], 1, 1, 64, seed=12)
    row = np.random.default_rng(5).standard_normal(64).astype(np.float32)
    Vs[0][0][:] = row
    kp, vp, bt = place_in_pool(Ks, Vs, 1, 64, 10, np.random.default_rng(6))
    out = orc.paged_decode(q, kp, vp, bt, cl, 0.125, orc.F32, orc.F32)
    np.testing.assert_allclose(out[0, 0], row.astype(np.float64), rtol=1e-14, atol=1e-15)


def test_dominant_key_selects_its_value():
    q, Ks, Vs, kp, vp, bt, cl = random_case([40], 1, 1, 64, seed=13)
    Ks[0][0, 23] = (q[0, 0] * 8).astype(np.float32)  # s_23 = 8 |q|^2 / 8 >> others
    kp, vp, bt = place_in_pool(Ks, Vs, 1, 64, 10, np.random.default_rng(7))
    out = orc.paged_decode(q, kp, vp, bt, cl, 1.0, orc.F32, orc.F32)
    np.testing.assert_allclose(out[0, 0], Vs[0][0, 23].astype(np.float64), atol=1e-12)


def test_empty_context_gives_zero_row():
    q, Ks, Vs, kp, vp, bt, cl = random_case([0, 5], 2, 2, 64, seed=14)
    out = orc.paged_decode(q, kp, vp, bt, cl, 0.125, orc.F32, orc.F32)
    assert np.array_equal(out[0], np.zeros((2, 64)))


# ---------------------------------------------------------------------------
# paging leaves the math unchanged ("vLLM explained", "兩層實作")
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("ctxs,n_q,n_kv,d", [
    ([1, 17, 33, 50], 4, 4, 64),          # the tiny fp32 workload's lengths
    ([128, 700, 2048], 8, 2, 128),        # GQA group 4
    ([16, 31, 32, 33, 255], 8, 1, 64),    # MQA, block edges
])
def test_paged_equals_contiguous_numpy(ctxs, n_q, n_kv, d):
    q, Ks, Vs, kp, vp, bt, cl = random_case(ctxs, n_q, n_kv, d, seed=sum(ctxs))
    scale = 1 / np.sqrt(d)
    out = orc.paged_decode(q, kp, vp, bt, cl, scale, orc.F32, orc.F32)
    G = n_q // n_kv
    for s in range(len(ctxs)):
        for h in range(n_q):
            ref = numpy_attention(q[s, h].astype(np.float64), Ks[s][h // G].astype(np.float64),
                                  Vs[s][h // G].astype(np.float64), scale)
            np.testing.assert_allclose(out[s, h], ref, rtol=1e-12, atol=1e-14)


def test_permuting_physical_blocks_is_bit_identical():
    # blocks need not be contiguous and other requests' blocks may sit between
    # them ("vLLM explained", "PagedAttention" figure caption)
    q, Ks, Vs, kp, vp, bt, cl = random_case([5, 48, 300, 129], 8, 2, 128, seed=20, extra_blocks=9)
    out = orc.paged_decode(q, kp, vp, bt, cl, 0.09, orc.F32, orc.F32)
    rng = np.random.default_rng(21)
    for _ in range(3):
        pi = rng.permutation(kp.shape[0])
        kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
        kp2[pi] = kp
        vp2[pi] = vp
        bt2 = np.where(bt >= 0, pi[np.maximum(bt, 0)], -1).astype(np.int32)
        out2 = orc.paged_decode(q, kp2, vp2, bt2, cl, 0.09, orc.F32, orc.F32)
        assert np.array_equal(out, out2)


def test_shared_block_reads_like_private_copy():
    # copy-on-write sharing: two sequences point at the same physical prefix
    # blocks ("LLM inference optimization", §三.2)
    rng = np.random.default_rng(30)
    d, n_kv = 64, 2
    kp = rng.standard_normal((12, n_kv, B, d)).astype(np.float32)
    vp = rng.standard_normal((12, n_kv, B, d)).astype(np.float32)
    q = rng.standard_normal((2, 4, d)).astype(np.float32)
    shared = np.array([[3, 8, 1, -1], [3, 8, 6, -1]], dtype=np.int32)
    cl = np.array([40, 45], dtype=np.int32)
    out_shared = orc.paged_decode(q, kp, vp, shared, cl, 0.125, orc.F32, orc.F32)
    kp2, vp2 = kp.copy(), vp.copy()
    kp2[[10, 11]] = kp[[3, 8]]
    vp2[[10, 11]] = vp[[3, 8]]
    private = np.array([[3, 8, 1, -1], [10, 11, 6, -1]], dtype=np.int32)
    out_private = orc.paged_decode(q, kp2, vp2, private, cl, 0.125, orc.F32, orc.F32)
    assert np.array_equal(out_shared, out_private)


def _read_golden_table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "worked_block_table.txt"))
            if l.strip() and not l.startswith("#")]
    tables = {}
    for req, lb, pb in rows:
        tables.setdefault(req, {})[int(lb)] = int(pb)
    return {k: [v[i] for i in range(len(v))] for k, v in tables.items()}


def test_worked_block_table_example():
    t = _read_golden_table()
    assert t == {"req1": [7, 2, 9], "req2": [7, 5]}
    rng = np.random.default_rng(40)
    d, n_kv, n_q = 64, 1, 2
    kp = rng.standard_normal((10, n_kv, B, d)).astype(np.float32)
    vp = rng.standard_normal((10, n_kv, B, d)).astype(np.float32)
    q = rng.standard_normal((2, n_q, d)).astype(np.float32)
    bt = np.array([t["req1"], t["req2"] + [-1]], dtype=np.int32)
    cl = np.array([45, 29], dtype=np.int32)  # req1: 33..48 tokens, req2: 17..32 tokens
    out = orc.paged_decode(q, kp, vp, bt, cl, 0.125, orc.F32, orc.F32)
    # contiguous reading: logical block j is tokens 16j..16j+15
    for s, ids in enumerate([t["req1"], t["req2"]]):
        K = np.concatenate([kp[i, 0] for i in ids])[:cl[s]].astype(np.float64)
        V = np.concatenate([vp[i, 0] for i in ids])[:cl[s]].astype(np.float64)
        for h in range(n_q):
            np.testing.assert_allclose(out[s, h], numpy_attention(q[s, h].astype(np.float64),
                                                                  K, V, 0.125),
                                       rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# dtypes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("code,tdtype", [(orc.F16, torch.float16), (orc.BF16, torch.bfloat16)])
def test_half_precision_storage_is_decoded_exactly(code, tdtype):
    q, Ks, Vs, kp, vp, bt, cl = random_case([77, 16], 4, 2, 128, seed=50)
    q16 = torch.from_numpy(q).to(tdtype)
    kp16 = torch.from_numpy(kp).to(tdtype)
    vp16 = torch.from_numpy(vp).to(tdtype)
    out = orc.paged_decode(q16, kp16, vp16, bt, cl, 0.088, code, code)
    out32 = orc.paged_decode(q16.float().numpy(), kp16.float().numpy(), vp16.float().numpy(),
                             bt, cl, 0.088, orc.F32, orc.F32)
    assert np.array_equal(out, out32)


def test_fp8_cache_values_times_scale():
    rng = np.random.default_rng(60)
    d, n_kv, n_q = 128, 2, 8
    ctx = [200, 33]
    codes_k = rng.integers(0, 256, size=(30, n_kv, B, d), dtype=np.uint8)
    codes_v = rng.integers(0, 256, size=(30, n_kv, B, d), dtype=np.uint8)
    codes_k[(codes_k & 0x7F) == 0x7F] = 0x11  # no NaN codes
    codes_v[(codes_v & 0x7F) == 0x7F] = 0x22
    bt = np.full((2, 13), -1, dtype=np.int32)
    bt[0, :13] = rng.permutation(30)[:13]
    bt[1, :3] = [29, 28, 27] if 29 not in bt[0] else [0, 1, 2]
    q = torch.randn(2, n_q, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    ks, vs = 0.0123, 0.0456
    out = orc.paged_decode(q, codes_k, codes_v, bt, np.array(ctx, np.int32), 0.088,
                           orc.BF16, orc.FP8_E4M3, ks, vs)
    kf = torch.from_numpy(codes_k).view(torch.float8_e4m3fn).double().numpy() * ks
    vf = torch.from_numpy(codes_v).view(torch.float8_e4m3fn).double().numpy() * vs
    qd = q.double().numpy()
    for s in range(2):
        ids = bt[s][bt[s] >= 0]
        for h in range(n_q):
            K = np.concatenate([kf[i, h // 4] for i in ids])[:ctx[s]]
            V = np.concatenate([vf[i, h // 4] for i in ids])[:ctx[s]]
            np.testing.assert_allclose(out[s, h], numpy_attention(qd[s, h], K, V, 0.088),
                                       rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# chunked prefill (causal)
# ---------------------------------------------------------------------------

def numpy_causal(Q, K, V, H, scale):
    """Textbook masked attention: row i sees keys j <= H + i."""
    S = (Q @ K.T) * scale
    L, T = S.shape
    mask = np.arange(T)[None, :] <= (H + np.arange(L))[:, None]
    S = np.where(mask, S, -np.inf)
    S = S - S.max(1, keepdims=True)
    P = np.exp(S)
    return (P @ V) / P.sum(1, keepdims=True)


@pytest.mark.parametrize("H,L", [(0, 37), (50, 20), (64, 16)])
def test_prefill_is_causal_attention(H, L):
    rng = np.random.default_rng(70 + H)
    d, n_kv, n_q = 64, 2, 4
    T = H + L
    K = rng.standard_normal((n_kv, T, d)).astype(np.float32)
    V = rng.standard_normal((n_kv, T, d)).astype(np.float32)
    kp, vp, bt = place_in_pool([K], [V], n_kv, d, -(-T // B) + 3, rng)
    q = rng.standard_normal((L, n_q, d)).astype(np.float32)
    qsl = np.array([0, L], np.int32)
    out = orc.paged_prefill(q, kp, vp, bt, qsl, np.array([T], np.int32), 0.125,
                            orc.F32, orc.F32)
    for h in range(n_q):
        ref = numpy_causal(q[:, h].astype(np.float64), K[h // 2].astype(np.float64),
                           V[h // 2].astype(np.float64), H, 0.125)
        np.testing.assert_allclose(out[:, h], ref, rtol=1e-12, atol=1e-14)


def test_prefill_two_chunks_are_independent_sequences():
    rng = np.random.default_rng(80)
    d, n_kv, n_q = 64, 1, 2
    Ks = [rng.standard_normal((n_kv, T, d)).astype(np.float32) for T in (40, 70)]
    Vs = [rng.standard_normal((n_kv, T, d)).astype(np.float32) for T in (40, 70)]
    kp, vp, bt = place_in_pool(Ks, Vs, n_kv, d, 12, rng)
    Ls = [8, 30]
    q = rng.standard_normal((sum(Ls), n_q, d)).astype(np.float32)
    qsl = np.array([0, 8, 38], np.int32)
    out = orc.paged_prefill(q, kp, vp, bt, qsl, np.array([40, 70], np.int32), 0.1,
                            orc.F32, orc.F32)
    for c, (T, L) in enumerate(zip((40, 70), Ls)):
        for h in range(n_q):
            ref = numpy_causal(q[qsl[c]:qsl[c + 1], h].astype(np.float64),
                               Ks[c][0].astype(np.float64), Vs[c][0].astype(np.float64),
                               T - L, 0.1)
            np.testing.assert_allclose(out[qsl[c]:qsl[c + 1], h], ref, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# byte model
# ---------------------------------------------------------------------------

def test_byte_formulas_match_pages():
    vals = dict(l.split() for l in open(os.path.join(GOLDEN, "kv_byte_formulas.txt"))
                if l.strip() and not l.startswith("#"))
    per_tok = W.kv_bytes_per_token(80, 8, 128, 2)
    assert per_tok == int(vals["llama3_70b_kv_bytes_per_token"])
    # the page's "2.56 GB" for 8K tokens is 2.5 GiB read with 1 KB = 1024 B
    assert per_tok * int(vals["llama3_70b_ctx_tokens"]) == int(2.5 * 2 ** 30)
    blk = W.block_bytes(16, 32, 32, 128, 2)
    assert blk == int(vals["llama2_7b_block_bytes"]) == 8 * 2 ** 20
    assert blk // 16 == int(vals["llama2_7b_kv_bytes_per_token"])
    # one layer's share, used by the decode byte model
    assert W.kv_bytes_per_token(1, 8, 128, 2) == 4096
    assert W.kv_bytes_per_token(1, 32, 128, 2) == 16384
