"""GPU parity with prefix caching across requests: chat-like requests that
share system prompts get their cached full blocks from the native manager,
their prompt K/V are written through the slots it returns (cached tokens
skipped), and fused decode steps run over the shared pool.  Checked against
the oracle (pool bit for bit, attention within 2e-3) and against ordinary
attention over each request's own contiguous K/V rows."""
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


def test_prefix_cached_requests_decode(pa, cuda_device):
    dev = cuda_device
    sh = W.Shape(32, 8, 128, 16, "bf16")
    B, Hkv, D = sh.block_size, sh.num_kv_heads, sh.head_dim
    wl = W.prefix_workload(shape=sh, num_requests=36, live=10, seed=8)
    nat = pa.BlockManager(wl.num_blocks, B, wl.free_order)
    ora = OracleBM(wl.num_blocks, B, wl.free_order)
    k_pool, v_pool = W.empty_pool(sh, wl.num_blocks, seed=5, device=dev)
    kb, vb = W.bits(k_pool), W.bits(v_pool)
    rows = {}                      # request -> (K bits, V bits) of all its tokens so far
    alive, hits = [], 0
    g = torch.Generator(device=dev); g.manual_seed(17)
    maxb = 40                      # longest request here: 25 blocks
    ws = pa.alloc_workspace(16, sh.num_q_heads, Hkv, D, B, maxb * B, dev)
    scale = 1.0 / np.sqrt(D)
    for e, (kind, i) in enumerate(wl.events):
        if kind == "free":
            nat.free_seq(i); ora.free_seq(i); alive.remove(i); del rows[i]
            continue
        toks = wl.requests[i]
        k, v = W.prefix_kv_rows(toks, sh, seed=3, device=dev)
        slots, cached = nat.allocate_prefix(i, toks)
        oslots, ocached = ora.allocate_prefix(i, toks)
        assert slots.tolist() == oslots and cached == ocached
        hits += cached
        pa.pa_reshape_and_cache(k, v, k_pool, v_pool, torch.as_tensor(slots, device=dev))
        OC.reshape_and_cache(W.bits(k), W.bits(v), kb, vb, np.array(oslots), B)
        rows[i] = (W.bits(k), W.bits(v))
        alive.append(i)
        if e % 3:
            continue
        # one fused decode step over every live request
        seqs = sorted(alive)
        S = len(seqs)
        q = torch.randn(S, sh.num_q_heads, D, generator=g, device=dev).to(torch.bfloat16)
        kn = torch.randn(S, Hkv, D, generator=g, device=dev).to(torch.bfloat16)
        vn = torch.randn(S, Hkv, D, generator=g, device=dev).to(torch.bfloat16)
        slots, pairs = nat.append_slots(seqs)
        owant = [ora.append_slot(s) for s in seqs]
        assert slots.tolist() == [w[0] for w in owant] and len(pairs) == 0
        tables, lens = nat.block_tables(seqs, maxb)
        out = torch.empty(S, sh.num_q_heads, D, device=dev)
        pa.pa_decode_step(out, q, kn, vn, k_pool, v_pool, torch.as_tensor(tables, device=dev),
                          torch.as_tensor(lens, device=dev), scale, Hkv,
                          max_context_len=maxb * B, workspace=ws)
        OC.reshape_and_cache(W.bits(kn), W.bits(vn), kb, vb, np.array([w[0] for w in owant]), B)
        otab = np.full((S, maxb), -1, dtype=np.int64)
        for r, s in enumerate(seqs):
            t = ora.block_table(s)
            otab[r, :len(t)] = t
            rows[s] = (np.concatenate([rows[s][0], W.bits(kn)[r:r + 1]]),
                       np.concatenate([rows[s][1], W.bits(vn)[r:r + 1]]))
        assert np.array_equal(tables, otab)
        qb = W.bits(q)
        want = OA.paged_decode_attention(qb, kb, vb, otab, lens, scale, Hkv, B, "bf16")
        got = out.cpu().numpy()
        assert max_abs_err(got, want) <= TOL
        # sharing is invisible: ordinary attention over the request's own rows
        G = sh.num_q_heads // Hkv
        for r, s in enumerate(seqs[:3]):
            kr, vr = decode(rows[s][0], "bf16"), decode(rows[s][1], "bf16")
            for h in (0, sh.num_q_heads - 1):
                ref = OA.softmax_attention(decode(qb[r, h], "bf16"), kr[:, h // G], vr[:, h // G],
                                           scale)
                assert np.abs(got[r, h] - ref).max() <= TOL
    torch.cuda.synchronize()
    assert hits > 0
    assert np.array_equal(W.bits(k_pool), kb) and np.array_equal(W.bits(v_pool), vb)
    assert pa.pa_device_error() == 0
    nat.close()
