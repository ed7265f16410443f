"""Prefix caching and chunked prefill together, as a serving step uses them:
each arriving request takes its cached full blocks from the native manager
(allocate_prefix), only its uncached tokens are written to the pool, and those
tokens run as one prefill chunk over the request's whole context -- cached
blocks included, most of them written by other requests.  Checked against the
oracle (pool bit for bit, attention within 2e-3) and against ordinary causal
attention over the request's own contiguous K/V rows."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle import cache_ops as OC
from oracle.block_manager import BlockManager as OracleBM
from oracle.fp import decode
from parity import TOL, max_abs_err

pytestmark = pytest.mark.gpu


def test_prefix_hits_then_chunked_prefill(pa, cuda_device):
    dev = cuda_device
    sh = W.Shape(32, 8, 128, 16, "bf16")
    B, Hq, Hkv, D = sh.block_size, sh.num_q_heads, sh.num_kv_heads, sh.head_dim
    G = Hq // Hkv
    wl = W.prefix_workload(shape=sh, num_requests=30, live=10, seed=9)
    nat = pa.BlockManager(wl.num_blocks, B, wl.free_order)
    ora = OracleBM(wl.num_blocks, B, wl.free_order)
    k_pool, v_pool = W.empty_pool(sh, wl.num_blocks, seed=6, device=dev)
    kb, vb = W.bits(k_pool), W.bits(v_pool)
    g = torch.Generator(device=dev); g.manual_seed(23)
    scale = 1.0 / np.sqrt(D)
    hits = 0
    for kind, i in wl.events:
        if kind == "free":
            nat.free_seq(i); ora.free_seq(i)
            continue
        toks = wl.requests[i]
        n = len(toks)
        k, v = W.prefix_kv_rows(toks, sh, seed=3, device=dev)
        slots, cached = nat.allocate_prefix(i, toks)
        oslots, ocached = ora.allocate_prefix(i, toks)
        assert slots.tolist() == oslots and cached == ocached
        hits += cached
        # only the uncached tokens are written
        new = slice(cached, n)
        pa.pa_reshape_and_cache(k[new].contiguous(), v[new].contiguous(), k_pool, v_pool,
                                torch.as_tensor(slots[new], device=dev))
        OC.reshape_and_cache(W.bits(k)[new], W.bits(v)[new], kb, vb, np.array(oslots[new]), B)
        # the chunk: the uncached tokens (the last token when the whole prompt was cached)
        c0 = min(cached, n - 1)
        C = n - c0
        q = torch.randn(C, Hq, D, generator=g, device=dev).to(torch.bfloat16)
        table = np.array([nat.block_table(i)], dtype=np.int32)
        assert table[0].tolist() == ora.block_table(i)
        out = torch.empty(C, Hq, D, device=dev)
        pa.pa_paged_prefill_attention(out, q, k_pool, v_pool, torch.as_tensor(table, device=dev),
                                      torch.tensor([n], dtype=torch.int32, device=dev),
                                      torch.tensor([0, C], dtype=torch.int32, device=dev),
                                      scale, Hkv, C)
        got = out.cpu().numpy()
        qb = W.bits(q)
        want = OA.paged_prefill_attention(qb, kb, vb, table.astype(np.int64), np.array([n]),
                                          np.array([0, C]), scale, Hkv, B, "bf16")
        assert max_abs_err(got, want) <= TOL, i
        # sharing is invisible: causal attention over the request's own rows
        kr, vr = decode(W.bits(k), "bf16"), decode(W.bits(v), "bf16")
        for row in (0, C - 1):
            p = c0 + row
            for h in (0, Hq - 1):
                ref = OA.softmax_attention(decode(qb[row, h], "bf16"), kr[:p + 1, h // G],
                                           vr[:p + 1, h // G], scale)
                assert np.abs(got[row, h] - ref).max() <= TOL
    torch.cuda.synchronize()
    assert hits > 0
    assert np.array_equal(W.bits(k_pool), kb) and np.array_equal(W.bits(v_pool), vb)
    assert pa.pa_device_error() == 0
    nat.close()
