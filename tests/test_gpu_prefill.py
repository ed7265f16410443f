"""GPU parity of chunked prefill (the tensor-core kernel behind
pa_paged_prefill_attention) against the oracle.

Each sequence's earlier context is allocated by the native block manager,
its chunk appended token by token (append_slots with the sequence repeated),
the chunk's K/V written by pa_reshape_and_cache, then every chunk token
attends causally over the paged cache.  Bars: slots and tables bit-exact
against the oracle's manager, the pool bit-exact, attention within 2e-3."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle import cache_ops as OC
from oracle.block_manager import BlockManager as OracleBM
from parity import TOL, max_abs_err

pytestmark = pytest.mark.gpu


def run_prefill(pa, b, seqs=None, max_query_len=None):
    """Manager -> cache write -> prefill attention through the library, and
    the oracle's result for ``seqs`` (all by default).  Returns (out, want)."""
    sh = b.shape
    B, dev = sh.block_size, b.q.device
    S = b.num_seqs
    kb, vb = W.bits(b.k_cache), W.bits(b.v_cache)          # before any kernel runs
    nat = pa.BlockManager(b.num_blocks, B, b.free_order)
    ora = OracleBM(b.num_blocks, B, b.free_order)
    slots, oslots = [], []
    for s in range(S):
        L, C = int(b.context_lens[s]), int(b.chunk_lens[s])
        nat.allocate(s, L - C)
        ora.allocate(s, L - C)
        sl, pairs = nat.append_slots([s] * C)
        osl = [ora.append_slot(s)[0] for _ in range(C)]
        assert sl.tolist() == osl and len(pairs) == 0
        slots += osl
    tables, lens = nat.block_tables(np.arange(S), b.block_tables.shape[1])
    assert np.array_equal(tables, b.block_tables) and np.array_equal(lens, b.context_lens)
    slot_map = torch.as_tensor(np.array(slots, dtype=np.int64), device=dev)
    pa.pa_reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache, slot_map)
    OC.reshape_and_cache(W.bits(b.k_new), W.bits(b.v_new), kb, vb, np.array(slots), B)
    T = b.num_tokens
    out = torch.full((T, sh.num_q_heads, sh.head_dim), float("nan"), device=dev)
    mq = int(b.chunk_lens.max(initial=0)) if max_query_len is None else max_query_len
    pa.pa_paged_prefill_attention(out, b.q, b.k_cache, b.v_cache,
                                  torch.as_tensor(b.block_tables, device=dev),
                                  torch.as_tensor(b.context_lens, device=dev),
                                  torch.as_tensor(b.query_start, device=dev), b.scale,
                                  sh.num_kv_heads, mq)
    torch.cuda.synchronize()
    assert np.array_equal(W.bits(b.k_cache), kb) and np.array_equal(W.bits(b.v_cache), vb)
    want = OA.paged_prefill_attention(W.bits(b.q), kb, vb, b.block_tables, b.context_lens,
                                      b.query_start, b.scale, sh.num_kv_heads, B, sh.dtype,
                                      seqs=seqs)
    nat.close()
    return out.cpu().numpy(), want


SHAPES = [
    # dtype, D, B, Hq, Hkv
    ("bf16", 128, 16, 32, 8), ("f16", 128, 16, 8, 8), ("bf16", 64, 32, 16, 2),
    ("f16", 64, 16, 4, 4), ("bf16", 128, 32, 64, 8), ("bf16", 128, 16, 12, 4),
    ("f16", 128, 16, 16, 1), ("bf16", 64, 16, 6, 1),
]
CONTEXT = [1, 40, 130, 1000, 7, 64, 700, 129]
CHUNKS = [1, 5, 130, 300, 0, 64, 200, 128]


@pytest.mark.parametrize("dtype,D,B,Hq,Hkv", SHAPES)
def test_prefill_shapes_ragged(pa, cuda_device, dtype, D, B, Hq, Hkv):
    sh = W.Shape(Hq, Hkv, D, B, dtype)
    b = W.make_prefill_batch(sh, CONTEXT, CHUNKS, seed=D + B + Hq, device=cuda_device,
                             poison="nan")
    got, want = run_prefill(pa, b)
    assert np.isfinite(got).all()
    assert max_abs_err(got, want) <= TOL
    assert pa.pa_device_error() == 0


def test_one_token_chunks_match_decode(pa, cuda_device):
    """Chunks of one token are decode steps: the prefill kernel and the decode
    kernel agree (within the tolerance; different kernels, different
    rounding) and both match the oracle."""
    sh = W.Shape(32, 8, 128, 16, "bf16")
    lens = [1, 15, 16, 17, 300, 2048, 3001]
    b = W.make_prefill_batch(sh, lens, [1] * len(lens), seed=12, device=cuda_device,
                             poison="nan")
    got, want = run_prefill(pa, b)
    assert max_abs_err(got, want) <= TOL
    dev = cuda_device
    out_d = torch.empty(len(lens), 32, 128, device=dev)
    pa.pa_paged_decode_attention(out_d, b.q, b.k_cache, b.v_cache,
                                 torch.as_tensor(b.block_tables, device=dev),
                                 torch.as_tensor(b.context_lens, device=dev), b.scale, 8)
    assert max_abs_err(out_d.cpu().numpy(), got) <= TOL


def test_chunking_is_invisible(pa, cuda_device):
    """One prompt processed as three chunks gives the rows of the one-chunk pass."""
    sh = W.Shape(16, 4, 128, 16, "bf16")
    L = 505
    whole = W.make_prefill_batch(sh, [L], [L], seed=3, device=cuda_device)
    got_whole, want = run_prefill(pa, whole)
    assert max_abs_err(got_whole, want) <= TOL
    dev = cuda_device
    start = 0
    for end in (128, 428, 505):
        out = torch.empty(end - start, 16, 128, device=dev)
        pa.pa_paged_prefill_attention(out, whole.q[start:end].contiguous(), whole.k_cache,
                                      whole.v_cache, torch.as_tensor(whole.block_tables, device=dev),
                                      torch.tensor([end], dtype=torch.int32, device=dev),
                                      torch.tensor([0, end - start], dtype=torch.int32, device=dev),
                                      whole.scale, 4, end - start)
        assert max_abs_err(out.cpu().numpy(), got_whole[start:end]) <= TOL
        start = end
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("seed", [W.SEEDS["gqa8b"] + 100, W.SEEDS["gqa8b"] + 1])
def test_benchmark_workload_every_sequence(pa, cuda_device, seed):
    """The chunked-prefill benchmark mix at full size (16 sequences, 512-token
    chunks on 0..3584 cached tokens, GQA 32/8 heads, bf16; the first seed
    draws the batch the benchmark times, in the launch configuration it
    times, the second another draw of the mix): every row of every sequence
    against the oracle, and the pool bit for bit."""
    sh = W.SHAPES["gqa8b"]
    lens, chunks = W.prefill_lens(np.random.default_rng(seed))
    b = W.make_prefill_batch(sh, lens, chunks, seed=seed, device=cuda_device, poison="nan")
    got, want = run_prefill(pa, b)
    assert np.isfinite(got).all()
    assert max_abs_err(got, want) <= TOL
    assert pa.pa_device_error() == 0


def test_bad_chunk_reports_instead_of_faulting(pa, cuda_device):
    """A chunk longer than its context is refused on the device (error word)
    and its rows are left unwritten; the other sequence is computed."""
    pa.pa_device_error(clear=True)
    sh = W.Shape(8, 2, 64, 16, "f16")
    b = W.make_prefill_batch(sh, [20, 40], [4, 8], seed=1, device=cuda_device)
    dev = cuda_device
    out = torch.full((12, 8, 64), 7.0, device=dev)
    lens_bad = torch.tensor([2, 40], dtype=torch.int32, device=dev)       # chunk 4 > 2
    pa.pa_paged_prefill_attention(out, b.q, b.k_cache, b.v_cache,
                                  torch.as_tensor(b.block_tables, device=dev), lens_bad,
                                  torch.as_tensor(b.query_start, device=dev), b.scale, 2, 8)
    assert pa.pa_device_error() & pa.DEVERR["context_len"]
    o = out.cpu().numpy()
    assert (o[:4] == 7.0).all() and np.isfinite(o[4:]).all() and not (o[4:] == 7.0).all()
    # max_query_len so small that the grid (two 32-token query tiles per CTA at
    # G = 4) misses the end of a 100-token chunk: reported, the covered rows
    # computed, the rest left alone
    b2 = W.make_prefill_batch(sh, [150], [100], seed=2, device=dev)
    out2 = torch.full((100, 8, 64), 7.0, device=dev)
    pa.pa_paged_prefill_attention(out2, b2.q, b2.k_cache, b2.v_cache,
                                  torch.as_tensor(b2.block_tables, device=dev),
                                  torch.as_tensor(b2.context_lens, device=dev),
                                  torch.as_tensor(b2.query_start, device=dev), b2.scale, 2, 10)
    assert pa.pa_device_error() & pa.DEVERR["context_len"]
    o2 = out2.cpu().numpy()
    assert np.isfinite(o2[:64]).all() and not (o2[:64] == 7.0).all() and (o2[64:] == 7.0).all()


@pytest.mark.parametrize("scale", [0.0, -0.06, 0.9])
def test_any_scale(pa, cuda_device, scale):
    """The softmax scale is any float: zero (uniform weights), negative, and
    large enough that the lazy rescaling of O triggers often."""
    sh = W.Shape(16, 4, 128, 16, "bf16")
    b = W.make_prefill_batch(sh, [300, 77, 1000], [300, 20, 129], seed=31, device=cuda_device,
                             poison="nan")
    b.scale = scale
    got, want = run_prefill(pa, b)
    assert np.isfinite(got).all()
    assert max_abs_err(got, want) <= TOL
    assert pa.pa_device_error() == 0


def test_bad_block_id_reports_instead_of_faulting(pa, cuda_device):
    """A block-table entry outside the pool is skipped by the copy engine and
    reported in the error word; the other sequence's rows still match the
    oracle."""
    pa.pa_device_error(clear=True)
    sh = W.Shape(8, 2, 128, 16, "bf16")
    b = W.make_prefill_batch(sh, [300, 200], [40, 64], seed=8, device=cuda_device)
    dev = cuda_device
    tables = b.block_tables.copy()
    tables[0, 3] = b.num_blocks + 11                      # sequence 0 only
    out = torch.empty(b.num_tokens, 8, 128, device=dev)
    pa.pa_paged_prefill_attention(out, b.q, b.k_cache, b.v_cache,
                                  torch.as_tensor(tables, device=dev),
                                  torch.as_tensor(b.context_lens, device=dev),
                                  torch.as_tensor(b.query_start, device=dev), b.scale, 2, 64)
    assert pa.pa_device_error() & pa.DEVERR["block_id"]
    want = OA.paged_prefill_attention(W.bits(b.q), W.bits(b.k_cache), W.bits(b.v_cache),
                                      b.block_tables, b.context_lens, b.query_start, b.scale, 2,
                                      16, "bf16", seqs=[1])
    rows = np.arange(b.query_start[1], b.query_start[2])
    assert max_abs_err(out.cpu().numpy()[rows], want[rows]) <= TOL
    assert pa.pa_device_error() == 0


def test_bf16_values_beyond_fp16_range_are_reported(pa, cuda_device):
    """P.V runs in fp16, with a bf16 V tile converted exactly within fp16's
    range; a bf16 V value beyond it becomes infinite, the rows that read it
    come out not finite, and that is reported (PA_DEVERR_RANGE), never
    silent.  Sequences that never read the value still match the oracle."""
    sh = W.Shape(8, 2, 128, 16, "bf16")
    b = W.make_prefill_batch(sh, [300, 500], [100, 200], seed=9, device=cuda_device)
    blk = int(b.block_tables[1, 0])                  # a prefix block of sequence 1
    b.v_cache[blk, 0, 3, 5] = 1.0e6
    got, want = run_prefill(pa, b)
    assert pa.pa_device_error() == pa.DEVERR["range"]
    rows0 = slice(int(b.query_start[0]), int(b.query_start[1]))
    assert max_abs_err(got[rows0], want[rows0]) <= TOL
    rows1 = slice(int(b.query_start[1]), int(b.query_start[2]))
    assert not np.isfinite(got[rows1, 0:4]).all()     # kv head 0's query heads


def test_finite_bf16_inputs_raise_no_range_flag(pa, cuda_device):
    """The range check looks at the outputs: large finite V values inside
    fp16's range (65280, bf16's largest below 65504) convert exactly and are
    not reported."""
    sh = W.Shape(8, 2, 128, 16, "bf16")
    b = W.make_prefill_batch(sh, [300, 500], [100, 200], seed=19, device=cuda_device)
    blk = int(b.block_tables[1, 0])
    b.v_cache[blk, 0, 3, 5] = 65280.0
    b.v_cache[blk, 1, 7, 9] = -65280.0
    got, want = run_prefill(pa, b)
    assert pa.pa_device_error() == 0
    assert max_abs_err(got, want) <= TOL * 65280.0


@pytest.mark.parametrize("S", [32, 40])
def test_many_sequences_every_unit_runs(pa, cuda_device, S):
    """Up to 32 sequences the launch order ranks them by context length (ties
    by index), beyond that it keeps the plain order; either way every
    (sequence, query-tile pair, kv head) unit runs: the output starts as NaN
    and every row must match the oracle."""
    rng = np.random.default_rng(100 + S)
    sh = W.Shape(8, 2, 64, 16, "bf16")
    lens = rng.integers(1, 600, size=S)
    lens[::5] = 300                                   # tied context lengths
    chunks = np.minimum(lens, rng.integers(1, 100, size=S))
    b = W.make_prefill_batch(sh, lens, chunks, seed=S, device=cuda_device, poison="nan")
    got, want = run_prefill(pa, b)
    assert np.isfinite(got).all()
    assert max_abs_err(got, want) <= TOL
    assert pa.pa_device_error() == 0
