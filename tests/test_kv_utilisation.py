"""KV memory accounting: the native manager's pa_bm_stats against the
oracle's accounting, and the pages' claims on real length mixes."""
import json
import os

import numpy as np
import pytest

import bench

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


def _cow_managers(pa, steps):
    """Native and oracle managers of the parallel-sampling workload after its
    prompts are forked and `steps` decode steps appended."""
    wl = W.cow_workload(steps=steps)
    B = wl.shape.block_size
    nat = pa.BlockManager(wl.num_blocks, B, wl.free_order)
    ora = OracleBM(wl.num_blocks, B, wl.free_order)
    for p_, P in enumerate(wl.prompt_lens):
        for bm in (nat, ora):
            bm.allocate(wl.seq_id(p_, 0), int(P))
            for br in range(1, wl.branches):
                bm.fork(wl.seq_id(p_, 0), wl.seq_id(p_, br))
    for _ in range(steps):
        nat.append_slots(np.arange(wl.num_seqs))
        for s in range(wl.num_seqs):
            ora.append_slot(s)
    return wl, nat, ora


@pytest.mark.parametrize("name", ["13b", "gqa8b", "long", "cow"])
def test_paged_versus_contiguous_reservation(pa, name):
    """[P1] sections 1 and 3: blocks taken on demand leave at most B-1 idle
    slots per sequence (waste under 4 % on the single-request length mixes);
    a max-length contiguous reservation leaves most of its slots idle.  The
    report's figures (from the native pa_bm_stats) equal the oracle's."""
    if name == "cow":
        wl, bm, ora = _cow_managers(pa, 64)
        B = wl.shape.block_size
        reserve = 2048
        tables = {s: ora.block_table(s) for s in ora.seqs()}
        lens = [ora.seq_len(s) for s in ora.seqs()]
        sh_rep = U.shared_report(tables, {s: ora.seq_len(s) for s in ora.seqs()}, B)
        want = {"paged_slots": sh_rep["physical_slots"],
                "paged_idle": sh_rep["physical_slots"] - sh_rep["filled_slots"],
                "contiguous_idle": U.contiguous_idle(lens, reserve)}
    else:
        sh = W.SHAPES[name]
        B = sh.block_size
        rng = np.random.default_rng(W.SEEDS[name])
        lens = {"13b": W.lens_13b, "gqa8b": W.lens_gqa8b, "long": W.lens_long}[name](rng)
        nblk = int(sum(-(-int(L) // B) for L in lens))
        bm = pa.BlockManager(nblk, B)
        for s, L in enumerate(lens):
            bm.allocate(s, int(L))
        reserve = 32768 if name == "long" else 4096
        want = U.report(lens, B, reserve)
        assert 1 - bench.kv_accounting(bm.stats(), reserve)["paged_useful_fraction"] < 0.04
    r = bench.kv_accounting(bm.stats(), reserve)
    assert r["paged_slots"] == want["paged_slots"]
    assert r["paged_idle_slots"] == want["paged_idle"] < len(lens) * B
    assert r["contiguous_idle_slots"] == want["contiguous_idle"]
    assert r["contiguous_idle_slots"] > 10 * r["paged_idle_slots"]
    assert r["contiguous_useful_fraction"] < r["paged_useful_fraction"]
    if name == "cow":
        # branches share their prompts: several logical tokens per filled slot
        assert r["sharing_ratio"] > 2 and r["shared_blocks"] > 0


def test_kv_report_covers_the_workloads_and_the_pages_example(pa):
    """bench.py --report kv: every length mix, set beside the pages' figures;
    the pages' one worked example (a 150-token request in a 2,048-token
    reservation leaves 1,898 slots idle; P1 section 1) comes out of the native
    manager's accounting exactly."""
    rep = bench.kv_report(pa)
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "contiguous_reservation_example.json")))
    ex = rep["workloads"]["example_150_tokens"]
    assert ex["contiguous_idle_slots"] == g["idle_slots"]
    assert ex["contiguous_slots"] == g["reserved_tokens"]
    assert ex["paged_idle_slots"] == 10 < g["example_block_size"]
    for name in ("13b", "gqa8b", "long", "cow_after_fork", "cow_after_64_steps"):
        r = rep["workloads"][name]
        assert r["paged_useful_fraction"] > r["contiguous_useful_fraction"]
        assert r["paged_idle_slots"] < r["sequences"] * 16
    assert rep["pages"]["paged_waste_fraction_below"] == 0.04
    json.dumps(rep)   # printable as one JSON line
