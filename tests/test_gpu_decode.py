"""GPU parity: one decode step (block manager -> reshape_and_cache -> paged
decode attention) through the C ABI against the oracle.

Bars: slots, block tables and the cache write bit-exact; attention within
2e-3 max-abs of the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import workloads as W
from parity import TOL, Expected, library_step, max_abs_err

pytestmark = pytest.mark.gpu


def check_step(pa, batch, seqs=None, tuning=None, tol=TOL):
    exp = Expected(batch, seqs)        # before any kernel touches the pool
    slots, tables, out = library_step(pa, batch, tuning)
    assert np.array_equal(slots, exp.slots)
    for s in exp.seqs:
        t = exp.tables[s]
        assert tables[s, :len(t)].tolist() == t
    # cache write: the sampled part of the pool, bit for bit
    idx = torch.as_tensor(exp.blocks, device=batch.k_cache.device)
    if len(exp.blocks):
        assert np.array_equal(W.bits(batch.k_cache.index_select(0, idx)), exp.k_after)
        assert np.array_equal(W.bits(batch.v_cache.index_select(0, idx)), exp.v_after)
    got = out.cpu().numpy()[exp.seqs]
    err = max_abs_err(got, exp.out)
    assert np.isfinite(got).all()
    assert err <= tol, err
    assert pa.pa_device_error() == 0
    return err, got, exp


def test_tiny_workload(pa, cuda_device):
    b = W.standard_batch("tiny", device=cuda_device)
    err, got, exp = check_step(pa, b)
    # the length-1 sequence returns its own (just written) V exactly
    v_new = b.v_new[0].float().cpu().numpy()           # [Hkv, D]
    assert np.array_equal(got[0], v_new)


SHAPES = [
    # dtype, D, B, Hq, Hkv
    ("f16", 64, 16, 4, 4), ("bf16", 128, 16, 8, 8), ("f16", 128, 32, 4, 4),
    ("bf16", 64, 32, 2, 2), ("bf16", 128, 16, 8, 2), ("f16", 128, 16, 8, 4),
    ("bf16", 128, 16, 16, 2), ("bf16", 64, 16, 12, 2), ("f16", 128, 32, 32, 4),
    ("bf16", 128, 32, 32, 2), ("bf16", 128, 16, 3, 1), ("f16", 64, 32, 10, 1),
]
LENS = [1, 15, 16, 17, 31, 33, 100, 257, 1000, 2048, 3001, 7]


@pytest.mark.parametrize("dtype,D,B,Hq,Hkv", SHAPES)
def test_shapes_ragged_lengths(pa, cuda_device, dtype, D, B, Hq, Hkv):
    sh = W.Shape(Hq, Hkv, D, B, dtype)
    b = W.make_decode_batch(sh, LENS, seed=D * 7 + B + Hq, device=cuda_device, poison="nan")
    check_step(pa, b)


@pytest.mark.parametrize("tuning", [(1, 1, 1), (2, 2, 1), (3, 0, 2), (0, 4, 64), (4, 1, 1000)])
def test_split_points_do_not_matter(pa, cuda_device, tuning):
    """Every way of cutting the work across warps (few tiles per warp: many
    split segments merged; many per warp: few) gives the oracle's result."""
    sh = W.Shape(16, 4, 128, 16, "bf16")
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 1500, size=24)
    b = W.make_decode_batch(sh, lens, seed=5, device=cuda_device, poison="nan")
    check_step(pa, b, tuning=tuning)


def test_empty_sequences_give_zero_rows(pa, cuda_device):
    sh = W.Shape(8, 2, 128, 16, "bf16")
    b = W.make_decode_batch(sh, [0, 5, 0, 40, 0], seed=9, device=cuda_device)
    _, got, _ = check_step(pa, b)
    assert (got[[0, 2, 4]] == 0).all()


def test_physical_placement_is_invisible(pa, cuda_device):
    """Permuting the pool and the tables together leaves the GPU output
    bit-identical (split points depend on lengths only)."""
    sh = W.Shape(32, 8, 128, 16, "bf16")
    rng = np.random.default_rng(1)
    lens = rng.integers(1, 600, size=40)
    b = W.make_decode_batch(sh, lens, seed=4, device=cuda_device)
    dev = cuda_device
    tables = torch.as_tensor(b.block_tables, device=dev)
    lens_d = torch.as_tensor(b.context_lens, device=dev)
    out1 = torch.empty(len(lens), 32, 128, device=dev)
    pa.pa_paged_decode_attention(out1, b.q, b.k_cache, b.v_cache, tables, lens_d, b.scale, 8)
    perm = torch.as_tensor(rng.permutation(b.num_blocks), device=dev)
    k2 = torch.empty_like(b.k_cache); v2 = torch.empty_like(b.v_cache)
    k2[perm] = b.k_cache; v2[perm] = b.v_cache
    t2 = torch.where(tables >= 0, perm[tables.clamp_min(0).long()].int(), tables)
    out2 = torch.empty_like(out1)
    pa.pa_paged_decode_attention(out2, b.q, k2, v2, t2, lens_d, b.scale, 8)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


def test_reshape_and_cache_bit_exact(pa, cuda_device):
    from oracle.cache_ops import reshape_and_cache
    for dtype, D, B in (("bf16", 128, 16), ("f16", 64, 32)):
        sh = W.Shape(4, 4, D, B, dtype)
        k, v = W.empty_pool(sh, 50, seed=2, device=cuda_device)
        rng = np.random.default_rng(0)
        T = 300
        slots = rng.choice(50 * B, size=T, replace=False).astype(np.int64)
        slots[::7] = -1
        g = torch.Generator(device=cuda_device); g.manual_seed(1)
        kn = torch.randn(T, 4, D, generator=g, device=cuda_device).to(k.dtype)
        vn = torch.randn(T, 4, D, generator=g, device=cuda_device).to(k.dtype)
        kb, vb = W.bits(k), W.bits(v)
        reshape_and_cache(W.bits(kn), W.bits(vn), kb, vb, slots, B)
        pa.pa_reshape_and_cache(kn, vn, k, v, torch.as_tensor(slots, device=cuda_device))
        torch.cuda.synchronize()
        assert np.array_equal(W.bits(k), kb) and np.array_equal(W.bits(v), vb)


def test_copy_blocks_bit_exact(pa, cuda_device):
    from oracle.cache_ops import copy_blocks
    sh = W.Shape(32, 8, 128, 16, "bf16")
    k, v = W.empty_pool(sh, 64, seed=3, device=cuda_device)
    pairs = np.array([[3, 10], [3, 11], [7, 0], [63, 62], [20, 21]], dtype=np.int64)
    kb, vb = W.bits(k), W.bits(v)
    copy_blocks(kb, vb, pairs)
    pa.pa_copy_blocks(k, v, torch.as_tensor(pairs, device=cuda_device))
    torch.cuda.synchronize()
    assert np.array_equal(W.bits(k), kb) and np.array_equal(W.bits(v), vb)


def test_device_checks_report_instead_of_faulting(pa, cuda_device):
    """Out-of-pool indices are skipped and reported in the error word."""
    pa.pa_device_error(clear=True)
    sh = W.Shape(4, 2, 64, 16, "f16")
    b = W.make_decode_batch(sh, [20, 40], seed=1, device=cuda_device)
    dev = cuda_device
    tables = torch.as_tensor(b.block_tables, device=dev).clone()
    tables[1, 1] = b.num_blocks + 5
    lens = torch.as_tensor(b.context_lens, device=dev)
    out = torch.empty(2, 4, 64, device=dev)
    pa.pa_paged_decode_attention(out, b.q, b.k_cache, b.v_cache, tables, lens, b.scale, 2)
    assert pa.pa_device_error() & pa.DEVERR["block_id"]
    lens2 = torch.as_tensor(np.array([10_000, 40], dtype=np.int32), device=dev)
    pa.pa_paged_decode_attention(out, b.q, b.k_cache, b.v_cache,
                                 torch.as_tensor(b.block_tables, device=dev), lens2, b.scale, 2,
                                 max_context_len=b.max_blocks_per_seq * 16)
    assert pa.pa_device_error() & pa.DEVERR["context_len"]
    kn = torch.zeros(1, 2, 64, dtype=torch.float16, device=dev)
    pa.pa_reshape_and_cache(kn, kn.clone(), b.k_cache, b.v_cache,
                            torch.tensor([b.num_blocks * 16 + 3], device=dev))
    assert pa.pa_device_error() & pa.DEVERR["slot"]
    pa.pa_copy_blocks(b.k_cache, b.v_cache, torch.tensor([[0, b.num_blocks]], device=dev))
    assert pa.pa_device_error() & pa.DEVERR["copy_pair"]
    assert pa.pa_device_error() == 0


def test_many_sequences(pa, cuda_device):
    """More sequences than one pass of a CTA's threads covers (the chunked
    scan of the launch plan), short and ragged, some empty."""
    sh = W.Shape(8, 2, 64, 16, "bf16")
    rng = np.random.default_rng(17)
    lens = rng.integers(0, 40, size=1500)
    b = W.make_decode_batch(sh, lens, seed=21, device=cuda_device, poison="nan")
    seqs = list(range(0, 1500, 7)) + [1499]
    check_step(pa, b, seqs=seqs)


FUSED_SHAPES = [("bf16", 128, 16, 32, 8), ("f16", 128, 16, 8, 8), ("bf16", 64, 32, 16, 2),
                ("f16", 64, 16, 4, 4), ("bf16", 128, 32, 64, 8)]


@pytest.mark.parametrize("dtype,D,B,Hq,Hkv", FUSED_SHAPES)
def test_fused_decode_step(pa, cuda_device, dtype, D, B, Hq, Hkv):
    """pa_decode_step (newest token's cache write + attention in one launch)
    against the oracle: the pool bit for bit, the output within tolerance."""
    from parity import library_fused_step
    sh = W.Shape(Hq, Hkv, D, B, dtype)
    lens = [1, 0, 15, 16, 17, 33, 100, 257, 1000, 2048, 3001, 7]
    b = W.make_decode_batch(sh, lens, seed=D + B + Hq + 1, device=cuda_device, poison="nan")
    exp = Expected(b)
    tables, out = library_fused_step(pa, b)
    idx = torch.as_tensor(exp.blocks, device=cuda_device)
    assert np.array_equal(W.bits(b.k_cache.index_select(0, idx)), exp.k_after)
    assert np.array_equal(W.bits(b.v_cache.index_select(0, idx)), exp.v_after)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert max_abs_err(got, exp.out) <= TOL
    assert (got[1] == 0).all()
    assert pa.pa_device_error() == 0


def test_fused_step_equals_two_calls(pa, cuda_device):
    """The fused step gives bit for bit the result of reshape_and_cache
    followed by decode attention."""
    from parity import library_fused_step
    sh = W.Shape(32, 8, 128, 16, "bf16")
    rng = np.random.default_rng(8)
    lens = rng.integers(1, 2500, size=64)
    b1 = W.make_decode_batch(sh, lens, seed=6, device=cuda_device)
    b2 = W.make_decode_batch(sh, lens, seed=6, device=cuda_device)
    _, _, out1 = library_step(pa, b1)
    _, out2 = library_fused_step(pa, b2)
    assert torch.equal(out1, out2)
    assert torch.equal(b1.k_cache, b2.k_cache) and torch.equal(b1.v_cache, b2.v_cache)
