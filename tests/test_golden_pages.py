"""Figures the pages print, checked against the oracle's accounting and gather.
Each fixture under tests/golden/ names the page and section it comes from."""
import json
import os

import numpy as np

from oracle import attention as A
from oracle import utilisation as U
import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_internal_fragmentation_example():
    g = load("contiguous_reservation_example.json")
    assert U.contiguous_idle([g["used_tokens"]], g["reserved_tokens"]) == g["idle_slots"]
    # the same request in blocks of the example size idles only its last
    # block's tail
    B = g["example_block_size"]
    idle = U.paged_idle([g["used_tokens"]], B)
    assert idle == 10 and idle < B
    assert U.paged_slots([g["used_tokens"]], B) == 160


def test_decode_reads_every_earlier_token():
    """The step that produces token #501 attends over the 500 tokens whose K/V
    are cached; the oracle gathers exactly those rows, from ceil(500/16) blocks."""
    g = load("decode_lookback_example.json")
    L = g["tokens_looked_back"]
    B = 16
    sh = W.Shape(1, 1, 8, B, "f16")
    b = W.make_decode_batch(sh, [L], 3)
    K = A.gather_logical_kv(W.bits(b.k_cache), b.block_tables[0], L, 0, B, "f16")
    assert K.shape == (L, 8)
    assert int((b.block_tables[0] >= 0).sum()) == -(-L // B) == 32


def test_paged_waste_below_four_percent_on_realistic_lengths():
    g = load("waste_figures.json")
    for name in ("13b", "gqa8b", "long", "long32"):
        sh = W.SHAPES[name]
        rng = np.random.default_rng(W.SEEDS[name])
        lens = {"13b": W.lens_13b, "gqa8b": W.lens_gqa8b}.get(name, W.lens_long)(rng)
        reserve = 32768 if name.startswith("long") else 4096
        r = U.report(lens, sh.block_size, reserve)
        assert r["paged_waste_fraction"] < g["paged_waste_fraction_below"], (name, r)
        # a max-length reservation wastes far more than blocks do
        assert r["contiguous_idle"] > 10 * r["paged_idle"]
