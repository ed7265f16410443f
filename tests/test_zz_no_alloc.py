"""The allocation-free decode entry point, for callers that cannot allocate
device memory (a plugin handed only its input and output buffers by a host
framework that owns all device memory, or a latency-critical caller where
cudaMalloc is not allowed).  Its split-context scratch is the library's own
fixed device array instead of a caller workspace; it runs the same kernels
with the same launch plan, so its result must be bit-identical to the
workspace entry point's, and within the attention tolerance of the oracle.
Collected last on purpose (file name)."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from parity import TOL, max_abs_err

pytestmark = pytest.mark.gpu


def _both(pa, b, device):
    tables = torch.as_tensor(b.block_tables, device=device)
    lens = torch.as_tensor(b.context_lens, device=device)
    S, Hq, D = b.q.shape
    ref = torch.empty(S, Hq, D, device=device)
    pa.pa_paged_decode_attention(ref, b.q, b.k_cache, b.v_cache, tables, lens, b.scale,
                                 b.shape.num_kv_heads)
    got = torch.full((S, Hq, D), float("nan"), device=device)
    pa.pa_paged_decode_attention_no_alloc(got, b.q, b.k_cache, b.v_cache, tables, lens,
                                          b.scale, b.shape.num_kv_heads)
    torch.cuda.synchronize()
    return ref, got


def _check(pa, b, device):
    # the oracle on the pool as drawn (neither call writes the cache)
    sh = b.shape
    want = OA.paged_decode_attention(W.bits(b.q), W.bits(b.k_cache), W.bits(b.v_cache),
                                     b.block_tables, b.context_lens, b.scale, sh.num_kv_heads,
                                     sh.block_size, sh.dtype)
    ref, got = _both(pa, b, device)
    assert torch.equal(got, ref)
    err = max_abs_err(got.cpu().numpy(), want)
    assert err <= TOL, err


def test_no_alloc_matches_workspace_entry_point_twice(pa, cuda_device):
    # two calls in a row, on different inputs: the shared scratch keeps the
    # first call's contents and the second must not depend on them
    sh = W.Shape(32, 8, 128, 16, "bf16")
    for seed in (11, 12):
        lens = np.random.default_rng(seed).integers(1, 3000, size=48)
        b = W.make_decode_batch(sh, lens, seed=seed, device=cuda_device, poison="nan")
        _check(pa, b, cuda_device)
    assert pa.pa_device_error() == 0


def test_no_alloc_largest_group_that_fits_at_default_tuning(pa, cuda_device):
    """head_dim 128, block 16: group size 13 is the largest whose default
    launch fits the fixed scratch; it runs and matches."""
    sh = W.Shape(26, 2, 128, 16, "bf16")           # 13 heads per group
    lens = np.random.default_rng(5).integers(1, 5000, size=12)
    b = W.make_decode_batch(sh, lens, seed=5, device=cuda_device, poison="nan")
    _check(pa, b, cuda_device)
    assert pa.pa_device_error() == 0


def test_no_alloc_refuses_launches_beyond_its_scratch(pa, cuda_device):
    """head_dim 128, block 16, 16 heads per group: the default launch needs
    more than the fixed scratch, so the call is refused with
    PA_ERR_WORKSPACE and nothing is launched."""
    sh = W.Shape(64, 4, 128, 16, "bf16")           # 16 heads per group
    b = W.make_decode_batch(sh, [100, 200], seed=3, device=cuda_device)
    tables = torch.as_tensor(b.block_tables, device=cuda_device)
    lens = torch.as_tensor(b.context_lens, device=cuda_device)
    out = torch.zeros(2, 64, 128, device=cuda_device)
    with pytest.raises(pa.PAError) as e:
        pa.pa_paged_decode_attention_no_alloc(out, b.q, b.k_cache, b.v_cache, tables, lens,
                                              b.scale, 4)
    assert e.value.status == -7
    torch.cuda.synchronize()
    assert (out == 0).all()
