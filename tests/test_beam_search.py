"""Beam search over paged KV blocks ("Why OS Virtual Memory Paging Saved LLM
Inference: The vLLM Breakthrough", section 3: beam-search branches share the
same physical prompt blocks; a branch that writes gets a private block).

Each step every live beam appends its token (copy-on-write where its last
block is shared), then the k survivors are drawn among the beams: a beam drawn
c > 1 times is forked c-1 times, a beam not drawn is freed, returning its
blocks.  The native manager must match the oracle's bit for bit under this
churn, hold no block twice or leak any, and -- on the GPU -- the decode
outputs of every beam must match the oracle's."""
import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import cache_ops as OC
from oracle.block_manager import BlockManager as OracleBM
import workloads as W
from parity import TOL, max_abs_err


def survivor_plan(k, steps, seed):
    """For every step, the parent index (into the live beams) of each survivor."""
    rng = np.random.default_rng(seed)
    plan = []
    for _ in range(steps):
        # skewed draws: good beams get picked several times, others die
        w = rng.dirichlet(np.full(k, 0.5))
        plan.append(np.sort(rng.choice(k, size=k, p=w)))
    return plan


def select(bm, live, parents, next_id):
    """Apply one selection to a manager: forks first, then frees.  Returns the
    new live list and the next free sequence id."""
    counts = np.bincount(parents, minlength=len(live))
    new_live = []
    for i, s in enumerate(live):
        if counts[i] >= 1:
            new_live.append(s)
            for _ in range(counts[i] - 1):
                bm.fork(s, next_id)
                new_live.append(next_id)
                next_id += 1
    for i, s in enumerate(live):
        if counts[i] == 0:
            bm.free_seq(s)
    return sorted(new_live), next_id


def test_beam_churn_native_matches_oracle(pa):
    k, steps, B = 6, 60, 8
    order = np.random.default_rng(4).permutation(400)
    nat = pa.BlockManager(400, B, order)
    ora = OracleBM(400, B, order)
    for bm in (nat, ora):
        bm.allocate(0, 13)
        for c in range(1, k):
            bm.fork(0, c)
    live_n = list(range(k)); live_o = list(range(k)); nid_n = nid_o = k
    for step, parents in enumerate(survivor_plan(k, steps, 9)):
        slots, pairs = nat.append_slots(live_n)
        want = [ora.append_slot(s) for s in live_o]
        assert slots.tolist() == [w[0] for w in want]
        assert [tuple(x) for x in pairs.tolist()] == [w[1] for w in want if w[1] is not None]
        live_n, nid_n = select(nat, live_n, parents, nid_n)
        live_o, nid_o = select(ora, live_o, parents, nid_o)
        assert live_n == live_o
        held = {}
        for s in live_n:
            t = nat.block_table(s)
            assert t == ora.block_table(s)
            assert len(t) == -(-nat.seq_len(s) // B)
            for b in t:
                held[b] = held.get(b, 0) + 1
        for b in range(400):
            assert nat.ref_count(b) == ora.ref_count(b) == held.get(b, 0)
        assert nat.num_free() == ora.num_free() == 400 - len(held)
    for s in live_n:
        nat.free_seq(s)
    assert nat.num_free() == 400


@pytest.mark.gpu
def test_beam_decode_matches_oracle(pa, cuda_device):
    k, steps = 8, 24
    sh = W.Shape(32, 8, 128, 16, "bf16")
    B, dev = sh.block_size, cuda_device
    num_blocks = 512
    order = np.random.default_rng(2).permutation(num_blocks).astype(np.int32)
    k_pool, v_pool = W.empty_pool(sh, num_blocks, 31, device=dev)
    kb, vb = W.bits(k_pool), W.bits(v_pool)
    nat = pa.BlockManager(num_blocks, B, order)
    ora = OracleBM(num_blocks, B, order)
    P = 37
    g = torch.Generator(device=dev); g.manual_seed(5)
    pk = torch.randn(P, sh.num_kv_heads, sh.head_dim, generator=g, device=dev).to(torch.bfloat16)
    pv = torch.randn(P, sh.num_kv_heads, sh.head_dim, generator=g, device=dev).to(torch.bfloat16)
    slots = nat.allocate(0, P)
    oslots = ora.allocate(0, P)
    assert slots.tolist() == oslots
    pa.pa_reshape_and_cache(pk, pv, k_pool, v_pool, torch.as_tensor(slots, device=dev))
    OC.reshape_and_cache(W.bits(pk), W.bits(pv), kb, vb, np.array(oslots), B)
    for c in range(1, k):
        nat.fork(0, c); ora.fork(0, c)
    live, nid = list(range(k)), k
    ws = pa.alloc_workspace(k, sh.num_q_heads, sh.num_kv_heads, sh.head_dim, B, 256, dev)
    scale = 1.0 / np.sqrt(sh.head_dim)
    for step, parents in enumerate(survivor_plan(k, steps, 3)):
        q = torch.randn(k, sh.num_q_heads, sh.head_dim, generator=g, device=dev).to(torch.bfloat16)
        kn = torch.randn(k, sh.num_kv_heads, sh.head_dim, generator=g, device=dev).to(torch.bfloat16)
        vn = torch.randn(k, sh.num_kv_heads, sh.head_dim, generator=g, device=dev).to(torch.bfloat16)
        slots, pairs = nat.append_slots(live)
        oapp = [ora.append_slot(s) for s in live]
        oslots = [a[0] for a in oapp]
        opairs = [a[1] for a in oapp if a[1] is not None]
        assert slots.tolist() == oslots
        assert [tuple(x) for x in pairs.tolist()] == opairs
        if len(pairs):
            pa.pa_copy_blocks(k_pool, v_pool, torch.as_tensor(pairs, device=dev))
            OC.copy_blocks(kb, vb, np.array(opairs))
        tables, lens = nat.block_tables(live, 16)
        out = torch.empty(k, sh.num_q_heads, sh.head_dim, device=dev)
        pa.pa_decode_step(out, q, kn, vn, k_pool, v_pool, torch.as_tensor(tables, device=dev),
                          torch.as_tensor(lens, device=dev), scale, sh.num_kv_heads,
                          max_context_len=16 * B, workspace=ws)
        OC.reshape_and_cache(W.bits(kn), W.bits(vn), kb, vb, np.array(oslots), B)
        otab = np.full((k, 16), -1, dtype=np.int64)
        olens = np.zeros(k, dtype=np.int64)
        for i, s in enumerate(live):
            t = ora.block_table(s)
            otab[i, :len(t)] = t
            olens[i] = ora.seq_len(s)
        want = OA.paged_decode_attention(W.bits(q), kb, vb, otab, olens, scale, sh.num_kv_heads,
                                         B, "bf16")
        assert max_abs_err(out.cpu().numpy(), want) <= TOL, step
        live_n, nid_n = select(nat, live, parents, nid)
        live_o, _ = select(ora, live, parents, nid)
        assert live_n == live_o
        live, nid = live_n, nid_n
    torch.cuda.synchronize()
    assert np.array_equal(W.bits(k_pool), kb) and np.array_equal(W.bits(v_pool), vb)
    assert pa.pa_device_error() == 0
