"""Split-context partials and their merge across calls: one workspace serves
any sequence of calls -- different head sizes, groups, block sizes and
launch shapes (CTAs per SM, stages, fewest tiles per warp) in turn -- with no
clearing between them, and a sequence cut into thousands of parts (one tile
per warp) merges exactly; each result checked against the oracle (2e-3
max-abs)."""
import numpy as np
import pytest
import torch

import workloads as W
from parity import TOL, Expected, max_abs_err

pytestmark = pytest.mark.gpu

# (shape, context lengths, launch tuning (stages, CTAs per SM, fewest tiles per warp))
CASES = [
    (W.Shape(32, 8, 128, 16, "bf16"), [4000, 1, 700, 0, 2500, 33], (0, 0, 0)),
    (W.Shape(8, 8, 64, 32, "f16"), [3000, 17, 0, 1200, 64], (1, 3, 2)),
    (W.Shape(64, 4, 128, 32, "bf16"), [5000, 900, 31, 2048], (2, 1, 1)),
    (W.Shape(24, 4, 64, 16, "f16"), [1, 4096, 1500, 15, 16, 17], (0, 2, 3)),
    (W.Shape(32, 8, 128, 16, "bf16"), [4000, 1, 700, 0, 2500, 33], (0, 0, 0)),
]


def test_one_workspace_across_shapes_and_launch_shapes(pa, cuda_device):
    dev = cuda_device
    need = max(pa.pa_paged_decode_workspace_bytes(len(lens), sh.num_q_heads, sh.num_kv_heads,
                                                  sh.head_dim, sh.block_size, max(lens))
               for sh, lens, _ in CASES)
    ws = torch.full((need,), 0xff, dtype=torch.uint8, device=dev)   # no clearing needed
    for rep in range(2):
        for i, (sh, lens, tuning) in enumerate(CASES):
            b = W.make_decode_batch(sh, np.array(lens), seed=70 + 10 * i + rep, device=dev,
                                    poison="nan")
            exp = Expected(b)
            bm = pa.BlockManager(b.num_blocks, sh.block_size, b.free_order)
            for s, L in enumerate(lens):
                bm.allocate(s, int(L))
            tables, d_lens = bm.block_tables(np.arange(len(lens)), b.max_blocks_per_seq)
            bm.close()
            slots = torch.as_tensor(exp.slots, device=dev)
            pa.pa_reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache, slots)
            out = torch.full((len(lens), sh.num_q_heads, sh.head_dim), float("nan"), device=dev)
            pa.pa_decode_tuning(*tuning)
            try:
                pa.pa_paged_decode_attention(out, b.q, b.k_cache, b.v_cache,
                                             torch.as_tensor(tables, device=dev),
                                             torch.as_tensor(d_lens, device=dev), b.scale,
                                             sh.num_kv_heads, max_context_len=max(lens),
                                             workspace=ws)
            finally:
                pa.pa_decode_tuning(0, 0, 0)
            got = out.cpu().numpy()
            assert np.isfinite(got).all(), (rep, i)
            assert max_abs_err(got, exp.out) <= TOL, (rep, i, sh, lens, tuning)
    assert pa.pa_device_error() == 0


def test_many_parts_per_sequence(pa, cuda_device):
    # at most one tile per warp where the tiles allow: a 64 K-token sequence is
    # cut into hundreds of parts, all merged into one output row per head
    dev = cuda_device
    sh = W.Shape(16, 2, 128, 16, "bf16")
    lens = np.array([65536, 3, 40000])
    b = W.make_decode_batch(sh, lens, seed=91, device=dev, poison="nan")
    exp = Expected(b)
    pa.pa_reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache,
                            torch.as_tensor(exp.slots, device=dev))
    out = torch.empty(len(lens), sh.num_q_heads, sh.head_dim, device=dev)
    bm = pa.BlockManager(b.num_blocks, sh.block_size, b.free_order)
    for s, L in enumerate(lens):
        bm.allocate(s, int(L))
    tables, d_lens = bm.block_tables(np.arange(len(lens)), b.max_blocks_per_seq)
    bm.close()
    ws = pa.alloc_workspace(len(lens), sh.num_q_heads, sh.num_kv_heads, sh.head_dim,
                            sh.block_size, int(lens.max()), dev)
    pa.pa_decode_tuning(0, 0, 1)
    try:
        for _ in range(3):   # repeated calls on the same workspace
            out.fill_(float("nan"))
            pa.pa_paged_decode_attention(out, b.q, b.k_cache, b.v_cache,
                                         torch.as_tensor(tables, device=dev),
                                         torch.as_tensor(d_lens, device=dev), b.scale,
                                         sh.num_kv_heads, max_context_len=int(lens.max()),
                                         workspace=ws)
            assert max_abs_err(out.cpu().numpy(), exp.out) <= TOL
    finally:
        pa.pa_decode_tuning(0, 0, 0)
    assert pa.pa_device_error() == 0
