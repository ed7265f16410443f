"""GPU parity at full workload sizes, in the launch configuration the
benchmark times: 13B-class, GQA 8B-class and long-context decode, every
sequence compared with the oracle and the whole pool compared bit for bit
after the step's cache write, through both the fused entry point the
benchmark times (pa_decode_step) and the two-call path (reshape_and_cache +
paged decode attention); and the 64-step parallel sampling run with
copy-on-write (every step checked)."""
import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import cache_ops as OC
from oracle.block_manager import BlockManager as OracleBM
import workloads as W
from parity import TOL, Expected, library_fused_step, library_step, max_abs_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["13b", "gqa8b", "long", "long32"])
@pytest.mark.parametrize("path", ["fused", "two_call"])
def test_full_size_workload(pa, cuda_device, name, path):
    b = W.standard_batch(name, device=cuda_device)
    exp = Expected(b, whole_pool=True)          # every sequence, from the pool as drawn
    if path == "fused":
        # the benchmark's launch: pa_decode_step with a workspace sized for
        # every tuning and the table's capacity as the context bound
        tables, out = library_fused_step(pa, b, max_context_len=b.max_blocks_per_seq *
                                         b.shape.block_size)
    else:
        slots, tables, out = library_step(pa, b)
        assert np.array_equal(slots, exp.slots)
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        assert tables[s, :-(-L // b.shape.block_size)].tolist() == exp.tables[s]
    got = out.cpu().numpy()
    err = max_abs_err(got, exp.out)
    assert err <= TOL, err
    assert np.array_equal(W.bits(b.k_cache), exp.k_pool)
    assert np.array_equal(W.bits(b.v_cache), exp.v_pool)
    assert pa.pa_device_error() == 0


def test_peaked_long_context_follows_the_hot_tokens(pa, cuda_device):
    """In the long-context workload the softmax is peaked on the planted
    positions: their weight dominates, and the oracle agrees with the GPU."""
    b = W.standard_batch("long", device=cuda_device)
    exp = Expected(b, [0])
    _, _, out = library_step(pa, b)
    err = max_abs_err(out.cpu().numpy()[[0]], exp.out)
    assert err <= TOL


@pytest.mark.parametrize("fused", [False, True])
def test_parallel_sampling_copy_on_write(pa, cuda_device, fused):
    wl = W.cow_workload(device=cuda_device)
    sh = wl.shape
    B = sh.block_size
    S = wl.num_seqs
    dev = cuda_device
    k, v = W.empty_pool(sh, wl.num_blocks, wl.seed, device=dev)
    kb, vb = W.bits(k), W.bits(v)                 # oracle's copy, as drawn
    pk, pv = W.bits(wl.prompt_k), W.bits(wl.prompt_v)
    obm = OracleBM(wl.num_blocks, B, wl.free_order)
    nbm = pa.BlockManager(wl.num_blocks, B, wl.free_order)
    off = 0
    for p, P in enumerate(wl.prompt_lens):
        P = int(P)
        s0 = wl.seq_id(p, 0)
        oslots = obm.allocate(s0, P)
        nslots = nbm.allocate(s0, P)
        assert nslots.tolist() == oslots
        OC.reshape_and_cache(pk[off:off + P], pv[off:off + P], kb, vb, np.array(oslots), B)
        pa.pa_reshape_and_cache(wl.prompt_k[off:off + P].contiguous(),
                                wl.prompt_v[off:off + P].contiguous(), k, v,
                                torch.as_tensor(nslots, device=dev))
        for br in range(1, wl.branches):
            obm.fork(s0, wl.seq_id(p, br))
            nbm.fork(s0, wl.seq_id(p, br))
        off += P
    ws = pa.alloc_workspace(S, sh.num_q_heads, sh.num_kv_heads, sh.head_dim, B, 4096, dev)
    seqs = np.arange(S)
    rng = np.random.default_rng(0)
    cap = 64
    total_cow = 0
    for step in range(wl.steps):
        q, kn, vn = wl.step_inputs(step)
        qb, knb, vnb = W.bits(q), W.bits(kn), W.bits(vn)
        # block manager: slots and copy pairs, bit for bit
        nslots, npairs = nbm.append_slots(seqs)
        oslots, opairs = [], []
        for s in range(S):
            sl, cow = obm.append_slot(s)
            oslots.append(sl)
            if cow is not None:
                opairs.append(cow)
        assert nslots.tolist() == oslots
        assert [tuple(x) for x in npairs.tolist()] == opairs
        total_cow += len(opairs)
        # device: copy-on-write copies before the step's cache write
        if len(npairs):
            pa.pa_copy_blocks(k, v, torch.as_tensor(npairs, device=dev))
        tables, lens = nbm.block_tables(seqs, cap)
        out = torch.empty(S, sh.num_q_heads, sh.head_dim, device=dev)
        scale = 1.0 / np.sqrt(sh.head_dim)
        if fused:
            pa.pa_decode_step(out, q, kn, vn, k, v, torch.as_tensor(tables, device=dev),
                              torch.as_tensor(lens, device=dev), scale, sh.num_kv_heads,
                              max_context_len=cap * B, workspace=ws)
        else:
            pa.pa_reshape_and_cache(kn, vn, k, v, torch.as_tensor(nslots, device=dev))
            pa.pa_paged_decode_attention(out, q, k, v, torch.as_tensor(tables, device=dev),
                                         torch.as_tensor(lens, device=dev), scale,
                                         sh.num_kv_heads, max_context_len=cap * B, workspace=ws)
        if opairs:
            OC.copy_blocks(kb, vb, np.array(opairs))
        OC.reshape_and_cache(knb, vnb, kb, vb, np.array(oslots), B)
        if step in (0, 1, wl.steps - 1):
            torch.cuda.synchronize()
            assert np.array_equal(W.bits(k), kb) and np.array_equal(W.bits(v), vb)
        check = seqs if step in (0, wl.steps - 1) else rng.choice(S, size=16, replace=False)
        otables = np.full((S, cap), -1, dtype=np.int64)
        olens = np.zeros(S, dtype=np.int64)
        for s in check:
            t = obm.block_table(int(s))
            otables[s, :len(t)] = t
            olens[s] = obm.seq_len(int(s))
        want = OA.paged_decode_attention(qb, kb, vb, otables, olens, 1.0 / np.sqrt(sh.head_dim),
                                         sh.num_kv_heads, B, sh.dtype, seqs=[int(s) for s in check])
        got = out.cpu().numpy()
        err = max_abs_err(got[check], want[check])
        assert err <= TOL, (step, err)
    assert total_cow == 7 * int(np.sum(wl.prompt_lens % B != 0))
    assert pa.pa_device_error() == 0
