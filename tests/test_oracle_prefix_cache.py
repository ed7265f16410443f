"""Pins of the oracle's prefix caching across requests ("Can OS paging
techniques reduce LLM serving memory waste?", second paragraph: blocks shared
across the requests of a batch; "vLLM & PagedAttention: Operating Systems
Ideas for LLM Serving", introduction: block tables make KV memory reusable
and shareable).

Each pin is checked against something other than the oracle's own map:
pairwise comparison of the requests' token prefixes, a closed-form count of
blocks in use, the plain allocator, and, for attention, ordinary attention
over the request's contiguous K/V rows."""
import numpy as np
import pytest

import workloads as W
from oracle import attention as OA
from oracle import cache_ops as OC
from oracle.block_manager import BlockManager, NoBlocks


def _state(bm):
    return (list(bm.free), list(bm.ref), {s: list(t) for s, t in bm.tables.items()},
            dict(bm.lens), dict(bm.cache), dict(bm.key_of))


def test_no_shared_prefix_is_plain_allocate():
    """Prompts whose first tokens all differ never hit: allocate_prefix then
    hands out exactly what allocate does, slot for slot."""
    rng = np.random.default_rng(0)
    B, n = 8, 300
    order = rng.permutation(n)
    a, b = BlockManager(n, B, order), BlockManager(n, B, order)
    for s in range(20):
        toks = np.concatenate([[100_000 + s], rng.integers(0, 50, size=int(rng.integers(0, 60)))])
        slots, cached = a.allocate_prefix(s, toks)
        assert cached == 0
        assert slots == b.allocate(s, len(toks))
        if s % 3 == 2:
            a.free_seq(s - 1); b.free_seq(s - 1)
    for s in sorted(a.tables):
        assert a.block_table(s) == b.block_table(s)
    assert list(a.free) == list(b.free) and a.ref == b.ref


def _common_blocks(x, y, B):
    """Number of leading full blocks on which two token lists agree (brute force)."""
    k = 0
    while (k + 1) * B <= min(len(x), len(y)) and list(x[:(k + 1) * B]) == list(y[:(k + 1) * B]):
        k += 1
    return k


def test_sharing_follows_token_prefixes():
    """All requests alive, no eviction: two requests share their j-th block
    exactly when their tokens agree up to the end of that block; the blocks
    in use are the distinct full-block prefixes plus one per partial block;
    every reference count is the number of tables holding the block."""
    wl = W.prefix_workload(num_requests=40, live=1000, num_blocks=4000, seed=3)
    B = wl.shape.block_size
    bm = BlockManager(wl.num_blocks, B, wl.free_order)
    for i, toks in enumerate(wl.requests):
        slots, cached = bm.allocate_prefix(i, toks)
        # the cached tokens are the longest run of full blocks an earlier request shares
        best = max([_common_blocks(toks, wl.requests[j], B) for j in range(i)] + [0])
        assert cached == best * B
        assert slots[:cached] == [-1] * cached and min(slots[cached:], default=0) >= 0
    reqs = wl.requests
    for i in range(len(reqs)):
        ti = bm.block_table(i)
        assert len(ti) == -(-len(reqs[i]) // B)
        for j in range(i):
            tj = bm.block_table(j)
            c = _common_blocks(reqs[i], reqs[j], B)
            for blk in range(min(len(ti), len(tj))):
                assert (ti[blk] == tj[blk]) == (blk < c), (i, j, blk)
    prefixes = {tuple(r[:(k + 1) * B]) for r in reqs for k in range(len(r) // B)}
    partial = sum(1 for r in reqs if len(r) % B)
    used = {b for s in bm.tables for b in bm.tables[s]}
    assert len(used) == len(prefixes) + partial
    assert bm.num_free() == wl.num_blocks - len(used)
    assert bm.num_cached() == len(prefixes)
    for b in range(wl.num_blocks):
        assert bm.ref_count(b) == sum(bm.tables[s].count(b) for s in bm.tables)


def test_freed_blocks_are_retained_and_revived():
    B = 4
    bm = BlockManager(12, B)
    toks = list(range(10))                          # blocks: [0..3] [4..7] and a partial
    s0, c0 = bm.allocate_prefix(0, toks)
    assert c0 == 0 and bm.block_table(0) == [0, 1, 2]
    bm.free_seq(0)                                  # 0, 1, 2 to the back of the free list
    assert list(bm.free) == list(range(3, 12)) + [0, 1, 2]
    assert bm.num_cached() == 2
    s1, c1 = bm.allocate_prefix(1, toks)
    # the two full blocks come back from the free list; the partial one is new (block 3)
    assert c1 == 8 and bm.block_table(1) == [0, 1, 3]
    assert s1 == [-1] * 8 + [12, 13]
    assert list(bm.free) == list(range(4, 12)) + [2]
    assert bm.ref_count(0) == bm.ref_count(1) == 1
    # a second live holder adds a reference and takes nothing from the free list
    s2, c2 = bm.allocate_prefix(2, toks[:8])
    assert c2 == 8 and s2 == [-1] * 8 and bm.block_table(2) == [0, 1]
    assert bm.ref_count(0) == bm.ref_count(1) == 2 and bm.num_free() == 9


def test_reuse_of_a_block_drops_its_entry_and_lookups_stop_at_the_first_miss():
    B = 4
    bm = BlockManager(6, B)
    toks = list(range(12))                          # three full blocks
    bm.allocate_prefix(0, toks)                     # blocks 0, 1, 2
    bm.free_seq(0)                                  # free list 3 4 5 0 1 2
    bm.allocate(1, 16)                              # takes 3 4 5 0: block 0's entry goes
    assert bm.num_cached() == 2
    bm.free_seq(1)                                  # free list 1 2 3 4 5 0
    slots, cached = bm.allocate_prefix(2, toks)
    # the first block misses, so blocks 1 and 2, although still entered, are
    # not looked up: fresh blocks 1, 2, 3 come from the front of the free list
    assert cached == 0 and bm.block_table(2) == [1, 2, 3]
    assert slots == list(range(4, 16))
    # the prefixes now point at the new blocks; the replaced entries are gone
    assert bm.num_cached() == 3
    assert sorted(bm.cache.values()) == [1, 2, 3]


def test_failure_leaves_state_unchanged():
    B = 4
    bm = BlockManager(5, B)
    bm.allocate_prefix(0, list(range(8)))           # blocks 0, 1
    bm.free_seq(0)
    bm.allocate(1, 4)                               # block 2
    before = _state(bm)
    # needs 2 hits (both free, so they leave the free list) + 3 new = 3 free left: too few
    with pytest.raises(NoBlocks):
        bm.allocate_prefix(2, list(range(8)) + list(range(100, 111)))
    assert _state(bm) == before
    slots, cached = bm.allocate_prefix(3, list(range(8)) + [7, 7])
    assert cached == 8 and bm.num_free() == 1       # 4 free - 2 revived - 1 new


def test_cached_blocks_are_never_written_or_copied():
    """Forks of a prefix-cached request copy only their partial last block;
    appends never land in a cached (full) block."""
    wl = W.prefix_workload(num_requests=16, live=1000, num_blocks=2000, seed=5)
    B = wl.shape.block_size
    bm = BlockManager(wl.num_blocks, B, wl.free_order)
    nxt = 1000
    for i, toks in enumerate(wl.requests):
        bm.allocate_prefix(i, toks)
        for _ in range(2):
            bm.fork(i, nxt); nxt += 1
    for _ in range(3 * B):
        for s in sorted(bm.tables):
            slot, cow = bm.append_slot(s)
            assert slot // B not in bm.key_of
            if cow is not None:
                assert cow[0] not in bm.key_of


def test_attention_over_shared_blocks_equals_contiguous():
    """Requests whose prompts share prefixes, their caches written through
    the slots allocate_prefix returns (cached tokens skipped): the paged
    oracle over the shared pool equals ordinary attention over each request's
    own contiguous K/V rows."""
    sh = W.Shape(4, 2, 16, 4, "bf16")
    wl = W.prefix_workload(shape=sh, num_requests=10, system_range=(5, 30),
                           suffix_range=(1, 9), live=1000, num_blocks=400, seed=11)
    B = sh.block_size
    bm = BlockManager(wl.num_blocks, B, wl.free_order)
    kp, vp = W.empty_pool(sh, wl.num_blocks, seed=1)
    kb, vb = W.bits(kp), W.bits(vp)
    rows = []
    for i, toks in enumerate(wl.requests):
        k, v = W.prefix_kv_rows(toks, sh, seed=2)
        slots, _ = bm.allocate_prefix(i, toks)
        OC.reshape_and_cache(W.bits(k), W.bits(v), kb, vb, np.array(slots), B)
        rows.append((W.bits(k), W.bits(v)))
    S = len(wl.requests)
    import torch
    qf = torch.randn(S, sh.num_q_heads, sh.head_dim, generator=torch.Generator().manual_seed(3))
    qb = W.bits(qf.to(torch.bfloat16))
    maxb = max(len(bm.block_table(s)) for s in range(S))
    tables = np.full((S, maxb), -1, dtype=np.int64)
    lens = np.zeros(S, dtype=np.int64)
    for s in range(S):
        t = bm.block_table(s)
        tables[s, :len(t)] = t
        lens[s] = bm.seq_len(s)
    scale = 1.0 / np.sqrt(sh.head_dim)
    got = OA.paged_decode_attention(qb, kb, vb, tables, lens, scale, sh.num_kv_heads, B, "bf16")
    from oracle.fp import decode
    G = sh.num_q_heads // sh.num_kv_heads
    for s in range(S):
        kr, vr = (decode(x, "bf16") for x in rows[s])
        for h in range(sh.num_q_heads):
            want = OA.softmax_attention(decode(qb[s, h], "bf16"), kr[:, h // G], vr[:, h // G],
                                        scale)
            assert np.array_equal(got[s, h], want)
    assert bm.num_cached() > 0 and any(bm.ref_count(b) > 1 for b in range(wl.num_blocks))
