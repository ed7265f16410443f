"""The native (C++) block manager against the oracle's, bit for bit: the same
operations from the same free order give the same tables, slots, copy pairs,
reference counts and free-list length."""
import numpy as np
import pytest

from oracle.block_manager import BlockManager as OracleBM, NoBlocks, SeqExists, UnknownSeq
import workloads as W


def same_state(nat, ora, seqs):
    assert nat.num_free() == ora.num_free()
    assert nat.num_seqs() == len(ora.seqs())
    for s in seqs:
        assert nat.block_table(s) == ora.block_table(s)
        assert nat.seq_len(s) == ora.seq_len(s)
    for b in range(ora.num_blocks):
        assert nat.ref_count(b) == ora.ref_count(b)


def test_tiny_decode_batch(pa):
    b = W.standard_batch("tiny")
    nat = pa.BlockManager(b.num_blocks, 16, b.free_order)
    ora = OracleBM(b.num_blocks, 16, b.free_order)
    for s, L in enumerate(b.context_lens):
        a1 = nat.allocate(s, int(L) - 1)
        a2 = ora.allocate(s, int(L) - 1)
        assert a1.tolist() == a2
    slots, pairs = nat.append_slots(np.arange(4))
    want = [ora.append_slot(s) for s in range(4)]
    assert slots.tolist() == [w[0] for w in want] and len(pairs) == 0
    same_state(nat, ora, range(4))
    # the generator's own table is what FIFO allocation of whole sequences,
    # in order, from its free order gives
    nat2 = pa.BlockManager(b.num_blocks, 16, b.free_order)
    for s, L in enumerate(b.context_lens):
        nat2.allocate(s, int(L))
        n = -(-int(L) // 16)
        assert nat2.block_table(s) == b.block_tables[s, :n].tolist()


def test_parallel_sampling_workload(pa):
    wl = W.cow_workload(steps=8)
    B = wl.shape.block_size
    nat = pa.BlockManager(wl.num_blocks, B, wl.free_order)
    ora = OracleBM(wl.num_blocks, B, wl.free_order)
    for p, P in enumerate(wl.prompt_lens):
        nat.allocate(wl.seq_id(p, 0), int(P))
        ora.allocate(wl.seq_id(p, 0), int(P))
        for br in range(1, wl.branches):
            nat.fork(wl.seq_id(p, 0), wl.seq_id(p, br))
            ora.fork(wl.seq_id(p, 0), wl.seq_id(p, br))
    seqs = np.arange(wl.num_seqs)
    for step in range(wl.steps):
        slots, pairs = nat.append_slots(seqs)
        want_slots, want_pairs = [], []
        for s in seqs:
            sl, cow = ora.append_slot(int(s))
            want_slots.append(sl)
            if cow is not None:
                want_pairs.append(cow)
        assert slots.tolist() == want_slots
        assert [tuple(x) for x in pairs.tolist()] == want_pairs
    same_state(nat, ora, seqs)
    tables, lens = nat.block_tables(seqs, 64)
    for s in seqs:
        t = ora.block_table(int(s))
        assert tables[s, :len(t)].tolist() == t and (tables[s, len(t):] == -1).all()
        assert lens[s] == ora.seq_len(int(s))


def test_random_churn_matches(pa):
    rng = np.random.default_rng(11)
    order = rng.permutation(300)
    nat = pa.BlockManager(300, 8, order)
    ora = OracleBM(300, 8, order)
    live, nxt = [], 0
    for it in range(4000):
        op = int(rng.integers(5))
        if op == 0 or not live:
            n = int(rng.integers(0, 60))
            r1 = r2 = None
            try:
                r1 = nat.allocate(nxt, n).tolist()
            except pa.NoBlocksError:
                r1 = "nb"
            try:
                r2 = ora.allocate(nxt, n)
            except NoBlocks:
                r2 = "nb"
            assert r1 == r2
            if r1 != "nb":
                live.append(nxt)
            nxt += 1
        elif op == 1:
            par = live[int(rng.integers(len(live)))]
            nat.fork(par, nxt)
            ora.fork(par, nxt)
            live.append(nxt)
            nxt += 1
        elif op in (2, 3):
            batch = [live[int(i)] for i in rng.integers(len(live), size=int(rng.integers(1, 6)))]
            try:
                r1 = nat.append_slots(batch)
                r1 = (r1[0].tolist(), [tuple(x) for x in r1[1].tolist()])
            except pa.NoBlocksError:
                r1 = "nb"
            # the oracle has no batch call: emulate all-or-nothing with a copy
            import copy
            snap = copy.deepcopy(ora.__dict__)
            try:
                res = [ora.append_slot(s) for s in batch]
                r2 = ([r[0] for r in res], [r[1] for r in res if r[1] is not None])
            except NoBlocks:
                ora.__dict__.update(snap)
                r2 = "nb"
            assert r1 == r2
        else:
            s = live.pop(int(rng.integers(len(live))))
            nat.free_seq(s)
            ora.free_seq(s)
        if it % 200 == 0:
            same_state(nat, ora, live)
    same_state(nat, ora, live)


def test_native_errors_leave_state_unchanged(pa):
    nat = pa.BlockManager(4, 4)
    nat.allocate(0, 10)
    with pytest.raises(pa.NoBlocksError):
        nat.allocate(1, 9)
    with pytest.raises(pa.SeqError):
        nat.allocate(0, 1)
    with pytest.raises(pa.SeqError):
        nat.append_slot(7)
    with pytest.raises(pa.SeqError):
        nat.fork(9, 10)
    with pytest.raises(pa.SeqError):
        nat.free_seq(3)
    assert nat.num_free() == 1 and nat.block_table(0) == [0, 1, 2]
    nat.allocate(1, 3)            # takes block 3
    nat.append_slot(1)            # fills it
    before = (nat.num_free(), nat.block_table(0), nat.block_table(1), nat.seq_len(0), nat.seq_len(1))
    with pytest.raises(pa.NoBlocksError):
        nat.append_slots([0, 0, 1])   # the third append needs a block: all undone
    assert before == (nat.num_free(), nat.block_table(0), nat.block_table(1), nat.seq_len(0),
                      nat.seq_len(1))
    with pytest.raises(ValueError):
        pa.BlockManager(4, 4, [0, 1, 1, 2])


def test_outputs_into_caller_buffers(pa):
    """append_slots / block_tables write into caller arrays (numpy or a CPU
    torch tensor, as a pinned upload buffer would be) exactly what they
    return otherwise; a wrong shape or dtype is refused."""
    import torch
    wl = W.cow_workload(steps=4)
    B = wl.shape.block_size
    mk = []
    for _ in range(2):
        bm = pa.BlockManager(wl.num_blocks, B, wl.free_order)
        for p, P in enumerate(wl.prompt_lens):
            bm.allocate(wl.seq_id(p, 0), int(P))
            for br in range(1, wl.branches):
                bm.fork(wl.seq_id(p, 0), wl.seq_id(p, br))
        mk.append(bm)
    a, b = mk
    seqs = np.arange(wl.num_seqs)
    n = len(seqs)
    slots_buf = np.full(n, -7, dtype=np.int64)
    pairs_buf = torch.full((n, 2), -7, dtype=torch.int64)
    tab_buf = torch.full((n, 64), -7, dtype=torch.int32)
    lens_buf = np.full(n, -7, dtype=np.int32)
    for _ in range(wl.steps):
        s1, p1 = a.append_slots(seqs)
        s2, p2 = b.append_slots(seqs, slots_out=slots_buf, pairs_out=pairs_buf)
        assert np.array_equal(s1, s2) and np.array_equal(s1, slots_buf)
        assert np.array_equal(p1, p2) and np.array_equal(p1, pairs_buf.numpy()[:len(p1)])
        t1, l1 = a.block_tables(seqs, 64)
        b.block_tables(seqs, 64, out=tab_buf, lens_out=lens_buf)
        assert np.array_equal(t1, tab_buf.numpy()) and np.array_equal(l1, lens_buf)
    with pytest.raises(ValueError):
        b.block_tables(seqs, 64, out=np.empty((n, 63), dtype=np.int32))
    with pytest.raises(ValueError):
        b.append_slots(seqs, slots_out=np.empty(n, dtype=np.int32))
    a.close(); b.close()
