"""The native block manager's prefix caching against the oracle, bit for bit:
chat-like requests sharing system prompts arrive and finish in a pool small
enough that freed prefixes are revived and later handed out again, with
decode appends (copy-on-write included) and forks in between."""
import numpy as np
import pytest

import workloads as W
from oracle.block_manager import BlockManager as OracleBM
from oracle.block_manager import NoBlocks


def compare(nat, ora, num_blocks):
    live = ora.seqs()
    assert nat.num_seqs() == len(live)
    for s in live:
        assert nat.block_table(s) == ora.block_table(s)
        assert nat.seq_len(s) == ora.seq_len(s)
    for b in range(num_blocks):
        assert nat.ref_count(b) == ora.ref_count(b)
    assert nat.num_free() == ora.num_free()
    assert nat.num_cached() == ora.num_cached()


@pytest.mark.parametrize("seed,live", [(7, 12), (8, 6), (9, 20)])
def test_prefix_workload_matches_oracle(pa, seed, live):
    wl = W.prefix_workload(num_requests=60, live=live, seed=seed)
    B = wl.shape.block_size
    nat = pa.BlockManager(wl.num_blocks, B, wl.free_order)
    ora = OracleBM(wl.num_blocks, B, wl.free_order)
    rng = np.random.default_rng(seed)
    alive, hits = [], 0
    for kind, i in wl.events:
        if kind == "free":
            for s in (i, 10_000 + i):                    # the request and its branch, if any
                if s in alive:
                    nat.free_seq(s); ora.free_seq(s); alive.remove(s)
        else:
            toks = wl.requests[i]
            try:
                want = ora.allocate_prefix(i, toks)
            except NoBlocks:
                with pytest.raises(pa.NoBlocksError):
                    nat.allocate_prefix(i, toks)
                continue
            slots, cached = nat.allocate_prefix(i, toks)
            assert slots.tolist() == want[0] and cached == want[1]
            hits += cached // B
            alive.append(i)
            if rng.random() < 0.2:                       # a parallel-sampling branch
                nat.fork(i, 10_000 + i); ora.fork(i, 10_000 + i); alive.append(10_000 + i)
        # a few decode steps of every live sequence
        for _ in range(int(rng.integers(0, 3))):
            seqs = sorted(alive)
            try:
                want = [ora.append_slot(s) for s in seqs]
            except NoBlocks:
                pytest.skip("pool too small for this draw")
            slots, pairs = nat.append_slots(seqs)
            assert slots.tolist() == [w[0] for w in want]
            assert [tuple(p) for p in pairs.tolist()] == [w[1] for w in want if w[1] is not None]
        compare(nat, ora, wl.num_blocks)
    assert hits > 0
    for s in list(alive):
        nat.free_seq(s); ora.free_seq(s)
    compare(nat, ora, wl.num_blocks)
    assert nat.num_free() == wl.num_blocks
    nat.close()


def test_failed_batch_keeps_cached_blocks(pa):
    """A batch of appends that takes a cached free block and then fails is
    undone completely: the block is back at the front of the free list with
    its prefix still entered, and a later prompt hits it."""
    B = 4
    nat = pa.BlockManager(4, B)
    nat.allocate_prefix(0, list(range(4)))            # block 0, cached
    nat.allocate(1, 3)                                # block 1
    nat.allocate(2, 4)                                # block 2, full
    nat.free_seq(0)                                   # free: 3 0
    assert nat.num_cached() == 1 and nat.num_free() == 2
    with pytest.raises(pa.NoBlocksError):
        nat.append_slots([1] + [2] * 9)               # 1 in place; 2 takes 3, then 0, then fails
    assert nat.num_cached() == 1 and nat.num_free() == 2
    assert nat.seq_len(1) == 3 and nat.seq_len(2) == 4
    slots, cached = nat.allocate_prefix(3, list(range(4)) + [9])
    assert cached == 4 and nat.block_table(3) == [0, 3]
    assert slots.tolist() == [-1, -1, -1, -1, 12]
    # a successful batch that takes the cached block drops its entry
    nat.free_seq(3)                                   # free: 0 3 (0 still cached)
    nat.append_slots([2, 2, 2, 2, 2])                 # 2 takes 0 then 3
    assert nat.num_cached() == 0
    slots, cached = nat.allocate_prefix(4, [])
    assert cached == 0 and slots.tolist() == []
    nat.close()


def test_prefix_arguments(pa):
    nat = pa.BlockManager(8, 4)
    nat.allocate_prefix(0, [1, 2, 3])
    with pytest.raises(pa.SeqError):
        nat.allocate_prefix(0, [1])
    with pytest.raises(pa.NoBlocksError):
        nat.allocate_prefix(1, list(range(100)))
    assert nat.num_free() == 7 and nat.num_cached() == 0
    nat.close()
