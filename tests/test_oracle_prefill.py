"""Pins of the oracle's chunked-prefill attention (the causal multi-token form
of paged attention): a whole prompt as one chunk equals PyTorch's causal
scaled-dot-product attention in float64; any chunking of a prompt gives the
rows of the whole-prompt pass; a one-token chunk is a decode step; brute force
in plain Python floats on a tiny case; physical placement is invisible."""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle.fp import decode


def paged_setup(lens, Hkv, D, B, dtype, seed, shuffle=True):
    """Contiguous K/V bits per sequence and the same rows laid out in a pool
    through block tables (written by plain indexing here)."""
    rng = np.random.default_rng(seed)
    nb = [-(-L // B) for L in lens]
    nblocks = sum(nb) + 3
    perm = rng.permutation(nblocks) if shuffle else np.arange(nblocks)
    g = torch.Generator().manual_seed(seed)
    dt = W.TORCH_DTYPES[dtype]
    kpool = W.bits(torch.randn(nblocks, Hkv, B, D, generator=g).to(dt))
    vpool = W.bits(torch.randn(nblocks, Hkv, B, D, generator=g).to(dt))
    tables = np.full((len(lens), max(nb)), -1, dtype=np.int64)
    rows, at = [], 0
    for s, L in enumerate(lens):
        k = W.bits(torch.randn(L, Hkv, D, generator=g).to(dt))
        v = W.bits(torch.randn(L, Hkv, D, generator=g).to(dt))
        tables[s, :nb[s]] = perm[at:at + nb[s]]
        at += nb[s]
        for t in range(L):
            kpool[tables[s, t // B], :, t % B] = k[t]
            vpool[tables[s, t // B], :, t % B] = v[t]
        rows.append((k, v))
    return kpool, vpool, tables, rows


def chunk_queries(chunks, Hq, D, dtype, seed):
    g = torch.Generator().manual_seed(seed + 99)
    T = int(sum(chunks))
    q = W.bits(torch.randn(T, Hq, D, generator=g).to(W.TORCH_DTYPES[dtype]))
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int64)
    return q, qs


@pytest.mark.parametrize("Hq,Hkv,dtype", [(4, 4, "f16"), (8, 2, "bf16")])
def test_whole_prompt_is_causal_sdpa(Hq, Hkv, dtype):
    D, B = 32, 8
    lens = [1, 7, 8, 9, 40]
    kp, vp, tables, rows = paged_setup(lens, Hkv, D, B, dtype, seed=1)
    q, qs = chunk_queries(lens, Hq, D, dtype, seed=1)
    scale = 1 / math.sqrt(D)
    got = OA.paged_prefill_attention(q, kp, vp, tables, np.array(lens), qs, scale, Hkv, B, dtype)
    for s, L in enumerate(lens):
        qq = torch.from_numpy(decode(q[qs[s]:qs[s + 1]], dtype)).permute(1, 0, 2)   # [Hq, L, D]
        kk = torch.from_numpy(decode(rows[s][0], dtype)).permute(1, 0, 2)
        vv = torch.from_numpy(decode(rows[s][1], dtype)).permute(1, 0, 2)
        G = Hq // Hkv
        kk, vv = kk.repeat_interleave(G, 0), vv.repeat_interleave(G, 0)
        want = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True,
                                                                scale=scale)
        np.testing.assert_allclose(got[qs[s]:qs[s + 1]], want.permute(1, 0, 2).numpy(),
                                   rtol=0, atol=1e-12)


def test_chunking_is_invisible():
    """Rows of a prompt computed chunk by chunk (each chunk with the context
    length reached after it) equal the rows of the whole-prompt pass."""
    Hq, Hkv, D, B, dtype = 8, 4, 16, 4, "bf16"
    L = 37
    kp, vp, tables, _ = paged_setup([L], Hkv, D, B, dtype, seed=2)
    q, qs = chunk_queries([L], Hq, D, dtype, seed=2)
    scale = 0.3
    whole = OA.paged_prefill_attention(q, kp, vp, tables, np.array([L]), qs, scale, Hkv, B, dtype)
    for cuts in ([5, 20, 37], [1, 2, 3, 36, 37], [16, 37]):
        start = 0
        for end in cuts:
            part = OA.paged_prefill_attention(q[start:end], kp, vp, tables, np.array([end]),
                                              np.array([0, end - start]), scale, Hkv, B, dtype)
            assert np.array_equal(part, whole[start:end])
            start = end


def test_one_token_chunks_are_decode():
    Hq, Hkv, D, B, dtype = 8, 2, 32, 16, "f16"
    lens = [1, 15, 16, 17, 100]
    kp, vp, tables, _ = paged_setup(lens, Hkv, D, B, dtype, seed=3)
    q, qs = chunk_queries([1] * len(lens), Hq, D, dtype, seed=3)
    got = OA.paged_prefill_attention(q, kp, vp, tables, np.array(lens), qs, 0.2, Hkv, B, dtype)
    want = OA.paged_decode_attention(q, kp, vp, tables, np.array(lens), 0.2, Hkv, B, dtype)
    assert np.array_equal(got, want)


def test_brute_force_tiny():
    """Three tokens of a five-token sequence, one head, written out with
    Python floats: row i sees positions 0 .. 2 + i."""
    Hq = Hkv = 1
    D, B, dtype = 4, 2, "f16"
    kp, vp, tables, rows = paged_setup([5], Hkv, D, B, dtype, seed=4)
    q, qs = chunk_queries([3], Hq, D, dtype, seed=4)
    scale = 0.7
    got = OA.paged_prefill_attention(q, kp, vp, tables, np.array([5]), qs, scale, Hkv, B, dtype)
    K = decode(rows[0][0], dtype)[:, 0].tolist()
    V = decode(rows[0][1], dtype)[:, 0].tolist()
    Q = decode(q, dtype)[:, 0].tolist()
    for i in range(3):
        p = 2 + i
        z = [scale * sum(Q[i][d] * K[t][d] for d in range(D)) for t in range(p + 1)]
        mz = max(z)
        w = [math.exp(x - mz) for x in z]
        den = sum(w)
        for d in range(D):
            want = sum(w[t] * V[t][d] for t in range(p + 1)) / den
            assert abs(got[i, 0, d] - want) < 1e-12


def test_placement_invisible_and_empty_chunks():
    Hq, Hkv, D, B, dtype = 4, 2, 16, 4, "bf16"
    lens = [9, 30, 3]
    chunks = [4, 0, 3]
    a = paged_setup(lens, Hkv, D, B, dtype, seed=5, shuffle=True)
    b = paged_setup(lens, Hkv, D, B, dtype, seed=5, shuffle=False)
    q, qs = chunk_queries(chunks, Hq, D, dtype, seed=5)
    ra = OA.paged_prefill_attention(q, a[0], a[1], a[2], np.array(lens), qs, 0.25, Hkv, B, dtype)
    rb = OA.paged_prefill_attention(q, b[0], b[1], b[2], np.array(lens), qs, 0.25, Hkv, B, dtype)
    assert ra.shape == (7, Hq, D) and np.array_equal(ra, rb)
