"""KV memory accounting (oracle; test infrastructure).

* [P1] section 1 "The Contiguous Allocation Problem": an engine that reserves
  a contiguous buffer of the maximum request length (e.g. 2,048 or 4,096
  tokens) leaves every slot past the request's actual length idle (internal
  fragmentation); worked example: 2,048 reserved, 150 used, 1,898 idle.
* [P2] section 01 "The Problem": with such reservations only a fraction of KV
  memory holds useful tokens.
* [P1] section 2 / section 3: with fixed-size blocks taken on demand the only
  idle slots of a sequence are the unused tail of its last block, fewer than
  one block; waste falls under 4 %.

Definitions used here, for sequences of lengths L_s:
  paged allocation     = sum_s ceil(L_s / B) * B slots
  paged idle           = sum_s (ceil(L_s / B) * B - L_s), each term < B
  contiguous allocation= N * R slots for a reservation of R tokens each
  contiguous idle      = sum_s (R - L_s)
  useful fraction      = sum_s L_s / allocation
With shared blocks (forked branches) the allocation counts distinct physical
blocks while the useful tokens count each distinct block's filled slots once.
"""
from __future__ import annotations


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def paged_slots(lens, block_size: int) -> int:
    return sum(ceil_div(int(L), block_size) * block_size for L in lens)


def paged_idle(lens, block_size: int) -> int:
    return sum(ceil_div(int(L), block_size) * block_size - int(L) for L in lens)


def contiguous_slots(lens, reserve: int) -> int:
    return len(lens) * reserve


def contiguous_idle(lens, reserve: int) -> int:
    return sum(reserve - int(L) for L in lens)


def report(lens, block_size: int, reserve: int) -> dict:
    used = sum(int(L) for L in lens)
    ps = paged_slots(lens, block_size)
    cs = contiguous_slots(lens, reserve)
    return {
        "tokens": used,
        "paged_slots": ps,
        "paged_idle": ps - used,
        "paged_useful_fraction": used / ps if ps else 1.0,
        "paged_waste_fraction": (ps - used) / ps if ps else 0.0,
        "contiguous_slots": cs,
        "contiguous_idle": cs - used,
        "contiguous_useful_fraction": used / cs if cs else 1.0,
    }


def shared_report(tables: dict, lens: dict, block_size: int) -> dict:
    """Accounting for a set of block tables that may share blocks.

    ``tables[seq]`` is the list of physical blocks, ``lens[seq]`` the token
    count.  A shared block is allocated once; its filled slots are the largest
    fill any holder gives it."""
    fill: dict[int, int] = {}
    for seq, table in tables.items():
        L = int(lens[seq])
        for j, b in enumerate(table):
            n = min(block_size, L - j * block_size)
            fill[b] = max(fill.get(b, 0), n)
    slots = len(fill) * block_size
    useful = sum(fill.values())
    logical = sum(int(L) for L in lens.values())
    return {
        "physical_blocks": len(fill),
        "physical_slots": slots,
        "filled_slots": useful,
        "logical_tokens": logical,
        "waste_fraction": (slots - useful) / slots if slots else 0.0,
        "sharing_ratio": logical / useful if useful else 1.0,
    }
