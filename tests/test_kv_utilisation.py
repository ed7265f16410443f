"""KV memory accounting: the native manager's pa_bm_stats against the
oracle's accounting, and the pages' claims on real length mixes."""
import numpy as np
import pytest

from oracle import utilisation as U
from oracle.block_manager import BlockManager as OracleBM
import workloads as W


def oracle_shared(ora):
    tables = {s: ora.block_table(s) for s in ora.seqs()}
    lens = {s: ora.seq_len(s) for s in ora.seqs()}
    return U.shared_report(tables, lens, ora.block_size)


def test_stats_match_the_oracle_on_the_parallel_sampling_workload(pa):
    wl = W.cow_workload(steps=20)
    B = wl.shape.block_size
    nat = pa.BlockManager(wl.num_blocks, B, wl.free_order)
    ora = OracleBM(wl.num_blocks, B, wl.free_order)
    for p_, P in enumerate(wl.prompt_lens):
        for bm in (nat, ora):
            bm.allocate(wl.seq_id(p_, 0), int(P))
            for br in range(1, wl.branches):
                bm.fork(wl.seq_id(p_, 0), wl.seq_id(p_, br))
    for step in range(wl.steps):
        nat.append_slots(np.arange(wl.num_seqs))
        for s in range(wl.num_seqs):
            ora.append_slot(s)
        if step in (0, 5, 19):
            st = nat.stats()
            want = oracle_shared(ora)
            assert st["used_blocks"] == want["physical_blocks"]
            assert st["filled_slots"] == want["filled_slots"]
            assert st["logical_tokens"] == want["logical_tokens"]
            assert st["free_blocks"] == ora.num_free()
            assert st["used_blocks"] + st["free_blocks"] == wl.num_blocks
            shared = sum(1 for b in range(wl.num_blocks) if ora.ref_count(b) > 1)
            assert st["shared_blocks"] == shared
    # branches share their prompt: far fewer slots than tokens
    assert nat.stats()["logical_tokens"] > 4 * nat.stats()["filled_slots"] / 2


@pytest.mark.parametrize("name", ["13b", "gqa8b", "long"])
def test_paged_versus_contiguous_reservation(pa, name):
    """[P1] sections 1 and 3: blocks taken on demand leave at most B-1 idle
    slots per sequence (waste under 4 % on these length mixes); a max-length
    contiguous reservation leaves most of its slots idle."""
    sh = W.SHAPES[name]
    rng = np.random.default_rng(W.SEEDS[name])
    lens = {"13b": W.lens_13b, "gqa8b": W.lens_gqa8b, "long": W.lens_long}[name](rng)
    nblk = int(sum(-(-int(L) // sh.block_size) for L in lens))
    bm = pa.BlockManager(nblk, sh.block_size)
    for s, L in enumerate(lens):
        bm.allocate(s, int(L))
    reserve = 32768 if name == "long" else 4096
    r = pa.utilisation_report(bm, reserve)
    want = U.report(lens, sh.block_size, reserve)
    assert r["paged_slots"] == want["paged_slots"]
    assert r["paged_idle_slots"] == want["paged_idle"] < len(lens) * sh.block_size
    assert r["contiguous_idle_slots"] == want["contiguous_idle"]
    assert 1 - r["paged_useful_fraction"] < 0.04
    assert r["contiguous_idle_slots"] > 10 * r["paged_idle_slots"]
    assert r["contiguous_useful_fraction"] < r["paged_useful_fraction"]
