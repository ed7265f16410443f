"""Randomized GPU parity sweep: seeded random configurations across the whole
supported space -- head_dim 64/128, block size 16/32, fp16/bf16, query-head
groups 1..16, ragged and empty sequences, NaN poison in every unused slot --
for the two-call decode step (a third of the cases under random launch
tunings), the fused decode step and chunked prefill, each against the oracle
(2e-3 max-abs, the pool bit for bit)."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle import cache_ops as OC
from parity import TOL, Expected, library_fused_step, library_step, max_abs_err

pytestmark = pytest.mark.gpu

GROUPS = [1, 2, 3, 4, 6, 8, 16]


def random_shape(rng):
    G = int(rng.choice(GROUPS))
    Hkv = int(rng.choice([1, 2, 4, 8] if G <= 8 else [1, 2, 4]))
    return W.Shape(G * Hkv, Hkv, int(rng.choice([64, 128])), int(rng.choice([16, 32])),
                   str(rng.choice(["f16", "bf16"])))


def random_lens(rng, n, top):
    lens = rng.integers(1, top, size=n)
    lens[rng.random(n) < 0.1] = 0                       # some empty sequences
    edge = rng.random(n) < 0.2                          # some on block edges
    lens[edge] = (rng.integers(1, max(2, top // 32), size=int(edge.sum())) * 16
                  + rng.integers(-1, 2, size=int(edge.sum())))
    return np.clip(lens, 0, None)


@pytest.mark.parametrize("case", range(24))
def test_decode_random(pa, cuda_device, case):
    rng = np.random.default_rng(1000 + case)
    sh = random_shape(rng)
    lens = random_lens(rng, int(rng.integers(1, 40)), 3000)
    b = W.make_decode_batch(sh, lens, seed=2000 + case, device=cuda_device, poison="nan")
    exp = Expected(b)
    tuning = None
    if case % 3 == 1:
        tuning = (int(rng.integers(0, 4)), int(rng.integers(0, 4)), int(rng.integers(0, 200)))
    slots, tables, out = library_step(pa, b, tuning)
    assert np.array_equal(slots, exp.slots)
    idx = torch.as_tensor(exp.blocks, device=cuda_device)
    if len(exp.blocks):
        assert np.array_equal(W.bits(b.k_cache.index_select(0, idx)), exp.k_after)
        assert np.array_equal(W.bits(b.v_cache.index_select(0, idx)), exp.v_after)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert max_abs_err(got, exp.out) <= TOL, (case, sh, lens.tolist())
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("case", range(16))
def test_fused_decode_random(pa, cuda_device, case):
    rng = np.random.default_rng(3000 + case)
    sh = random_shape(rng)
    lens = random_lens(rng, int(rng.integers(1, 30)), 2500)
    b = W.make_decode_batch(sh, lens, seed=4000 + case, device=cuda_device, poison="nan")
    exp = Expected(b)
    tables, out = library_fused_step(pa, b)
    idx = torch.as_tensor(exp.blocks, device=cuda_device)
    if len(exp.blocks):
        assert np.array_equal(W.bits(b.k_cache.index_select(0, idx)), exp.k_after)
        assert np.array_equal(W.bits(b.v_cache.index_select(0, idx)), exp.v_after)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert max_abs_err(got, exp.out) <= TOL, (case, sh, lens.tolist())
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("case", range(20))
def test_prefill_random(pa, cuda_device, case):
    rng = np.random.default_rng(5000 + case)
    sh = random_shape(rng)
    S = int(rng.integers(1, 6))
    chunks = rng.integers(0, 260, size=S)
    chunks[rng.random(S) < 0.15] = 1                    # decode-like chunks
    lens = chunks + rng.integers(0, 1500, size=S)
    b = W.make_prefill_batch(sh, lens, chunks, seed=6000 + case, device=cuda_device,
                             poison="nan")
    B, dev = sh.block_size, cuda_device
    kb, vb = W.bits(b.k_cache), W.bits(b.v_cache)
    nat = pa.BlockManager(b.num_blocks, B, b.free_order)
    slots = []
    for s in range(S):
        nat.allocate(s, int(lens[s] - chunks[s]))
        slots.append(nat.append_slots([s] * int(chunks[s]))[0])
    tables, _ = nat.block_tables(np.arange(S), b.block_tables.shape[1])
    nat.close()
    assert np.array_equal(tables, b.block_tables)
    slots = np.concatenate(slots).astype(np.int64)
    pa.pa_reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache,
                            torch.as_tensor(slots, device=dev))
    OC.reshape_and_cache(W.bits(b.k_new), W.bits(b.v_new), kb, vb, slots, B)
    out = torch.full((b.num_tokens, sh.num_q_heads, sh.head_dim), float("nan"), device=dev)
    pa.pa_paged_prefill_attention(out, b.q, b.k_cache, b.v_cache,
                                  torch.as_tensor(b.block_tables, device=dev),
                                  torch.as_tensor(b.context_lens, device=dev),
                                  torch.as_tensor(b.query_start, device=dev), b.scale,
                                  sh.num_kv_heads, int(chunks.max(initial=0)))
    torch.cuda.synchronize()
    assert np.array_equal(W.bits(b.k_cache), kb) and np.array_equal(W.bits(b.v_cache), vb)
    want = OA.paged_prefill_attention(W.bits(b.q), kb, vb, b.block_tables, b.context_lens,
                                      b.query_start, b.scale, sh.num_kv_heads, B, sh.dtype)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert max_abs_err(got, want) <= TOL, (case, sh, lens.tolist(), chunks.tolist())
    assert pa.pa_device_error() == 0
