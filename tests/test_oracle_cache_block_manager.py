"""Pins for oracle/cache_ops.py, oracle/block_manager.py and oracle/utilisation.py:
invariants the pages state, closed forms and brute force on tiny inputs."""
import itertools

import numpy as np
import pytest

from oracle import attention as A
from oracle import cache_ops as C
from oracle import utilisation as U
from oracle.block_manager import BlockManager, NoBlocks, SeqExists, UnknownSeq
import workloads as W


def ceil_div(a, b):
    return -(-a // b)


# ---------------------------------------------------------------- cache ops

def test_reshape_and_cache_places_each_token_in_its_slot():
    """Read every written token back element by element through (slot // B,
    slot % B); every other element keeps its old bits."""
    rng = np.random.default_rng(0)
    NB, H, B, D, T = 6, 3, 4, 5, 9
    k = rng.integers(0, 1 << 16, size=(NB, H, B, D), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(NB, H, B, D), dtype=np.uint16)
    k0, v0 = k.copy(), v.copy()
    kn = rng.integers(0, 1 << 16, size=(T, H, D), dtype=np.uint16)
    vn = rng.integers(0, 1 << 16, size=(T, H, D), dtype=np.uint16)
    slots = rng.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[2] = -1
    C.reshape_and_cache(kn, vn, k, v, slots, B)
    written = {}
    for t in range(T):
        if slots[t] >= 0:
            written[(int(slots[t]) // B, int(slots[t]) % B)] = t
    for blk, h, off, d in itertools.product(range(NB), range(H), range(B), range(D)):
        t = written.get((blk, off))
        wk = k0[blk, h, off, d] if t is None else kn[t, h, d]
        wv = v0[blk, h, off, d] if t is None else vn[t, h, d]
        assert k[blk, h, off, d] == wk and v[blk, h, off, d] == wv


def test_copy_blocks_copies_whole_blocks_only():
    rng = np.random.default_rng(1)
    k = rng.integers(0, 1 << 16, size=(8, 2, 4, 3), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(8, 2, 4, 3), dtype=np.uint16)
    k0, v0 = k.copy(), v.copy()
    pairs = np.array([[1, 5], [1, 6], [3, 0]], dtype=np.int64)
    C.copy_blocks(k, v, pairs)
    for blk in range(8):
        src = {5: 1, 6: 1, 0: 3}.get(blk, blk)
        assert np.array_equal(k[blk], k0[src]) and np.array_equal(v[blk], v0[src])


# ---------------------------------------------------------------- block manager

def check_invariants(bm: BlockManager):
    B = bm.block_size
    held = {}
    for s in bm.seqs():
        t = bm.block_table(s)
        # [P1] section 2: blocks only as tokens need them
        assert len(t) == ceil_div(bm.seq_len(s), B)
        # idle slots of a sequence lie in its last block only: fewer than B
        assert len(t) * B - bm.seq_len(s) < B or bm.seq_len(s) == 0
        for b in t:
            held[b] = held.get(b, 0) + 1
    for b in range(bm.num_blocks):
        assert bm.ref_count(b) == held.get(b, 0)
    assert bm.num_free() + len(held) == bm.num_blocks
    assert set(bm.free).isdisjoint(held)


def test_allocate_takes_ceil_blocks_from_the_front():
    order = [5, 2, 7, 0, 1, 3, 4, 6]
    bm = BlockManager(8, 4, order)
    slots = bm.allocate(10, 9)
    assert bm.block_table(10) == [5, 2, 7]
    assert slots == [5 * 4 + i for i in range(4)] + [2 * 4 + i for i in range(4)] + [7 * 4]
    assert bm.num_free() == 5
    check_invariants(bm)


def test_append_takes_a_block_exactly_at_block_boundaries():
    bm = BlockManager(20, 4)
    bm.allocate(0, 0)
    for n in range(1, 30):
        before = len(bm.block_table(0))
        slot, cow = bm.append_slot(0)
        after = len(bm.block_table(0))
        assert cow is None
        assert after - before == (1 if (n - 1) % 4 == 0 else 0)
        assert slot == bm.block_table(0)[(n - 1) // 4] * 4 + (n - 1) % 4
        check_invariants(bm)


def test_freed_blocks_return_to_the_back():
    bm = BlockManager(6, 2, [3, 1, 4, 0, 5, 2])
    bm.allocate(0, 3)            # takes 3, 1
    bm.allocate(1, 1)            # takes 4
    bm.free_seq(0)
    assert list(bm.free) == [0, 5, 2, 3, 1]
    check_invariants(bm)


def test_fork_shares_every_block():
    """[P1] section 3: branches share the exact same physical prompt blocks."""
    bm = BlockManager(32, 16)
    bm.allocate(0, 50)
    for c in range(1, 8):
        bm.fork(0, c)
    for c in range(8):
        assert bm.block_table(c) == bm.block_table(0)
    for b in bm.block_table(0):
        assert bm.ref_count(b) == 8
    check_invariants(bm)


def test_first_write_to_a_shared_partial_block_copies():
    """[P1] section 3: a branch that writes gets a private block.  With 8
    sharers of a partial last block, branches 0-6 copy and branch 7, by then
    the only holder, writes in place."""
    bm = BlockManager(64, 16)
    bm.allocate(0, 50)
    for c in range(1, 8):
        bm.fork(0, c)
    last = bm.block_table(0)[-1]
    cows = []
    for c in range(8):
        slot, cow = bm.append_slot(c)
        cows.append(cow)
        assert slot == bm.block_table(c)[-1] * 16 + 50 % 16
    assert all(cw is not None and cw[0] == last for cw in cows[:7])
    assert cows[7] is None and bm.block_table(7)[-1] == last
    lasts = [bm.block_table(c)[-1] for c in range(8)]
    assert len(set(lasts)) == 8
    # the full prompt blocks stay shared
    for b in bm.block_table(0)[:-1]:
        assert bm.ref_count(b) == 8
    check_invariants(bm)


def test_block_aligned_prompt_needs_no_copy():
    bm = BlockManager(64, 16)
    bm.allocate(0, 48)
    for c in range(1, 4):
        bm.fork(0, c)
    for c in range(4):
        _, cow = bm.append_slot(c)
        assert cow is None
    check_invariants(bm)


def test_cow_count_on_the_parallel_sampling_workload():
    """32 prompts x 8 branches: 7 copies per prompt whose length is not a
    multiple of B, none otherwise, all on the first step."""
    wl = W.cow_workload(steps=3)
    B = wl.shape.block_size
    bm = BlockManager(wl.num_blocks, B, wl.free_order)
    for p, P in enumerate(wl.prompt_lens):
        bm.allocate(wl.seq_id(p, 0), int(P))
        for b in range(1, wl.branches):
            bm.fork(wl.seq_id(p, 0), wl.seq_id(p, b))
    per_step = []
    for step in range(wl.steps):
        n = 0
        for s in range(wl.num_seqs):
            _, cow = bm.append_slot(s)
            n += cow is not None
        per_step.append(n)
        check_invariants(bm)
    assert per_step[0] == 7 * int(np.sum(wl.prompt_lens % B != 0))
    assert per_step[1:] == [0] * (wl.steps - 1)


def test_failures_leave_state_unchanged():
    bm = BlockManager(4, 4)
    bm.allocate(0, 10)                      # 3 blocks
    snap = (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()}, dict(bm.lens))
    with pytest.raises(NoBlocks):
        bm.allocate(1, 9)
    with pytest.raises(SeqExists):
        bm.allocate(0, 1)
    with pytest.raises(UnknownSeq):
        bm.append_slot(7)
    with pytest.raises(UnknownSeq):
        bm.fork(9, 10)
    with pytest.raises(UnknownSeq):
        bm.free_seq(3)
    assert snap == (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()}, dict(bm.lens))
    bm.allocate(1, 4)                       # last block
    bm.append_slot(0)
    bm.append_slot(0)                       # len 12 -> block 3 full
    snap = (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()}, dict(bm.lens))
    with pytest.raises(NoBlocks):
        bm.append_slot(0)                   # needs a 4th block
    assert snap == (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()}, dict(bm.lens))


def test_random_churn_keeps_invariants():
    rng = np.random.default_rng(3)
    bm = BlockManager(200, 8, rng.permutation(200))
    live, nxt = [], 0
    for _ in range(3000):
        op = rng.integers(4)
        try:
            if op == 0 or not live:
                bm.allocate(nxt, int(rng.integers(0, 40))); live.append(nxt); nxt += 1
            elif op == 1:
                bm.fork(live[rng.integers(len(live))], nxt); live.append(nxt); nxt += 1
            elif op == 2:
                bm.append_slot(live[rng.integers(len(live))])
            else:
                s = live.pop(rng.integers(len(live))); bm.free_seq(s)
        except NoBlocks:
            pass
        check_invariants(bm)
    for s in live:
        bm.free_seq(s)
    assert bm.num_free() == 200


# ---------------------------------------------------------------- sharing is invisible

def _run_branches(shared: bool, seed=4, steps=6):
    """Two prompts x three branches: forked (shared blocks + copy-on-write)
    or each branch holding its own copy of the prompt from the start."""
    sh = W.Shape(4, 2, 16, 4, "bf16")
    wl = W.cow_workload(num_prompts=2, branches=3, steps=steps, prompt_range=(5, 11), shape=sh, seed=seed)
    B = sh.block_size
    bm = BlockManager(wl.num_blocks, B, wl.free_order)
    k, v = W.empty_pool(sh, wl.num_blocks, seed)
    kb, vb = W.bits(k), W.bits(v)
    pk, pv = W.bits(wl.prompt_k), W.bits(wl.prompt_v)
    off = 0
    for p, P in enumerate(wl.prompt_lens):
        P = int(P)
        for b in range(wl.branches):
            s = wl.seq_id(p, b)
            if shared and b > 0:
                bm.fork(wl.seq_id(p, 0), s)
                continue
            slots = bm.allocate(s, P)
            C.reshape_and_cache(pk[off:off + P], pv[off:off + P], kb, vb, np.array(slots), B)
        off += P
    outs = []
    for step in range(wl.steps):
        q, kn, vn = (W.bits(x) for x in wl.step_inputs(step))
        slots, pairs = [], []
        for s in range(wl.num_seqs):
            slot, cow = bm.append_slot(s)
            slots.append(slot)
            if cow is not None:
                pairs.append(cow)
        if pairs:
            C.copy_blocks(kb, vb, np.array(pairs))
        C.reshape_and_cache(kn, vn, kb, vb, np.array(slots), B)
        maxb = max(len(bm.block_table(s)) for s in range(wl.num_seqs))
        tables = np.full((wl.num_seqs, maxb), -1, dtype=np.int32)
        lens = np.zeros(wl.num_seqs, dtype=np.int32)
        for s in range(wl.num_seqs):
            t = bm.block_table(s)
            tables[s, :len(t)] = t
            lens[s] = bm.seq_len(s)
        outs.append(A.paged_decode_attention(q, kb, vb, tables, lens, 0.25, sh.num_kv_heads, B, "bf16"))
    return outs, bm


def test_shared_prompt_blocks_give_the_unshared_result():
    """[P1] section 3: sharing is a memory saving only -- forked branches with
    copy-on-write produce bit-identical outputs to branches that each own a
    copy of the prompt."""
    a, bm_a = _run_branches(True)
    b, bm_b = _run_branches(False)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    # and the shared run holds fewer blocks
    assert bm_a.num_free() > bm_b.num_free()


# ---------------------------------------------------------------- utilisation

def test_paged_idle_bound():
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 5000, size=500)
    for B in (1, 16, 32):
        idle = U.paged_idle(lens, B)
        assert idle == sum((-L) % B for L in lens)
        assert all(ceil_div(L, B) * B - L < B for L in lens)
    assert U.paged_idle(lens, 1) == 0


def test_shared_report_counts_shared_blocks_once():
    tables = {0: [3, 4, 5], 1: [3, 4, 6]}
    lens = {0: 10, 1: 9}
    r = U.shared_report(tables, lens, 4)
    assert r["physical_blocks"] == 4 and r["filled_slots"] == 4 + 4 + 2 + 1
    assert r["logical_tokens"] == 19
