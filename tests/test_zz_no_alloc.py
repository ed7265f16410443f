"""The allocation-free decode entry point, for callers that cannot allocate
device memory (a plugin handed only its input and output buffers by a host
framework that owns all device memory, or a latency-critical caller where
cudaMalloc is not allowed).  Its split-context scratch is the library's own
fixed device array instead of a caller workspace; the result must be that of
the workspace entry point.  Collected last on purpose (file name)."""
import numpy as np
import pytest
import torch

import workloads as W
from parity import TOL

pytestmark = pytest.mark.gpu


def _batch(seed, device):
    sh = W.Shape(32, 8, 128, 16, "bf16")
    lens = np.random.default_rng(seed).integers(1, 3000, size=48)
    return W.make_decode_batch(sh, lens, seed=seed, device=device, poison="nan")


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


def test_no_alloc_matches_workspace_entry_point_twice(pa, cuda_device):
    # two calls in a row, on different inputs: the shared scratch keeps the
    # first call's contents and the second must not depend on them
    for seed in (11, 12):
        b = _batch(seed, cuda_device)
        ref, got = _both(pa, b, cuda_device)
        assert torch.isfinite(got).all()
        err = float((got - ref).abs().max())
        assert err <= TOL, (seed, err)
    assert pa.pa_device_error() == 0


def test_no_alloc_refuses_launches_beyond_its_scratch(pa, cuda_device):
    """A launch layout needing more than the fixed scratch is refused with
    PA_ERR_WORKSPACE, and nothing is launched."""
    sh = W.Shape(64, 4, 128, 16, "bf16")           # 16 heads per group
    b = W.make_decode_batch(sh, [100, 200], seed=3, device=cuda_device)
    tables = torch.as_tensor(b.block_tables, device=cuda_device)
    lens = torch.as_tensor(b.context_lens, device=cuda_device)
    out = torch.zeros(2, 64, 128, device=cuda_device)
    pa.pa_decode_tuning(0, 4, 0)                   # 4 CTAs per SM: a larger grid
    try:
        with pytest.raises(pa.PAError) as e:
            pa.pa_paged_decode_attention_no_alloc(out, b.q, b.k_cache, b.v_cache, tables, lens,
                                                  b.scale, 4)
        assert e.value.status == -7
    finally:
        pa.pa_decode_tuning(0, 0, 0)
    torch.cuda.synchronize()
    assert (out == 0).all()
