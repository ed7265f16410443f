"""Failure detection on the GPU without a fault or a hang: every wait inside
the kernels (on a TMA copy, on the tensor cores, between the prefill
kernel's warp roles) is bounded by the library's wait limit.  A tiny limit
makes those waits run out while valid copies are in flight, so the kernels'
give-up path really executes: the time-out bit is set, the copies and MMAs
already issued are drained, the prefill kernel frees its tensor memory, and
the call returns.  The context stays usable: with the default limit restored,
the next calls (the prefill one allocates tensor memory again) match the
oracle."""
import numpy as np
import pytest
import torch

import workloads as W
from parity import TOL, Expected, library_fused_step, library_step, max_abs_err
from test_gpu_prefill import run_prefill

pytestmark = pytest.mark.gpu

TIMEOUT = 0x10


def _with_tiny_limit(pa, fn):
    assert pa.pa_device_error() == 0          # clean start
    pa.pa_set_wait_limit(1)                   # 1 ns: the first wait that is not yet satisfied gives up
    try:
        fn()
        torch.cuda.synchronize()
    finally:
        pa.pa_set_wait_limit(0)               # back to the default 2 s
    return pa.pa_device_error()               # read and clear


def _decode_batch(device, seed):
    sh = W.Shape(32, 8, 128, 16, "bf16")
    lens = np.random.default_rng(seed).integers(1, 3000, size=64)
    return W.make_decode_batch(sh, lens, seed=seed, device=device)


@pytest.mark.parametrize("entry", ["attention", "decode_step"])
def test_decode_wait_runs_out_then_recovers(pa, cuda_device, entry):
    b = _decode_batch(cuda_device, 21)
    if entry == "attention":
        flags = _with_tiny_limit(pa, lambda: library_step(pa, b))
    else:
        flags = _with_tiny_limit(pa, lambda: library_fused_step(pa, b))
    assert flags & TIMEOUT, flags
    assert flags == TIMEOUT                   # nothing else went wrong
    # the same process, default limit: a fresh batch matches the oracle
    b = _decode_batch(cuda_device, 22)
    exp = Expected(b)
    if entry == "attention":
        _, _, out = library_step(pa, b)
    else:
        _, out = library_fused_step(pa, b)
    assert max_abs_err(out.cpu().numpy(), exp.out) <= TOL
    assert pa.pa_device_error() == 0


def test_prefill_wait_runs_out_then_recovers(pa, cuda_device):
    sh = W.Shape(32, 8, 128, 16, "bf16")
    ctx, chunks = [700, 1000, 300, 129], [300, 200, 300, 128]
    b = W.make_prefill_batch(sh, ctx, chunks, seed=31, device=cuda_device)
    flags = _with_tiny_limit(pa, lambda: run_prefill(pa, b))
    assert flags == TIMEOUT, flags
    # tensor memory was freed by every CTA that gave up: the next launch
    # allocates it again on the same SMs and completes
    b = W.make_prefill_batch(sh, ctx, chunks, seed=32, device=cuda_device, poison="nan")
    got, want = run_prefill(pa, b)
    assert np.isfinite(got).all()
    assert max_abs_err(got, want) <= TOL
    assert pa.pa_device_error() == 0
