"""Cache writes and copy-on-write block copies on raw bits (oracle; test infrastructure).

* reshape_and_cache -- [P1] section 2 "The PagedAttention Architecture",
  on-demand allocation: each generated token's K/V goes into the slot its
  sequence's block table assigns.  Slot numbering: slot = block * B + offset,
  the token then lives at cache[block, :, offset, :].  A negative slot means
  "no slot" and the token is skipped.
* copy_blocks -- [P1] section 3 "Copy-on-Write for Prompt Sharing": a branch
  that writes into a block it shares gets a private block; the private block
  starts as a copy of the shared one.  Each (src, dst) pair copies the whole
  block, every kv head, in both the K and the V pool.

Both operate on uint16 bit arrays of the pool layout
[num_blocks, num_kv_heads, block_size, head_dim], so equality is bit equality.
"""
from __future__ import annotations

import numpy as np


def reshape_and_cache(key_bits, value_bits, k_cache_bits, v_cache_bits, slot_mapping,
                      block_size: int) -> None:
    """In place: cache[slot // B, h, slot % B, :] = new[t, h, :] for every token t."""
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        blk, off = divmod(int(slot), block_size)
        k_cache_bits[blk, :, off, :] = key_bits[t]
        v_cache_bits[blk, :, off, :] = value_bits[t]


def copy_blocks(k_cache_bits, v_cache_bits, block_mapping) -> None:
    """In place: cache[dst] = cache[src] for every (src, dst) pair, K and V."""
    for src, dst in np.asarray(block_mapping).reshape(-1, 2).tolist():
        k_cache_bits[int(dst)] = k_cache_bits[int(src)]
        v_cache_bits[int(dst)] = v_cache_bits[int(src)]
