"""Paged decode attention, written out plainly in float64 (oracle; test infrastructure).

What is computed, per the pages:

* [P1] section 2 "The PagedAttention Architecture": the KV cache is cut into
  fixed-size blocks (e.g. 16 tokens); a block table maps a sequence's logical
  token positions to physical blocks; for a newly generated token the kernel
  looks the physical blocks up in the table and fetches K/V from wherever the
  blocks lie.
* [P3] second paragraph: attention runs block by block, so the blocks need
  not be contiguous; the result is that of ordinary attention over the
  sequence's logical K/V.

So for sequence s, query head h (kv head kh = h // G, G = Hq / Hkv) and the
sequence's L tokens (the token appended this step included):

1. gather: K_s[t] = k_cache[table[s][t // B], kh, t % B, :], same for V,
   for t = 0 .. L-1, in logical order;
2. z_t = scale * <q[s, h], K_s[t]>;
3. w = exp(z - max z) / sum(exp(z - max z));
4. out[s, h] = sum_t w_t V_s[t].

An empty sequence (L = 0) has no tokens to attend to; its output row is zero.

The split-context partial/merge algebra (a sequence cut into partitions whose
(max, sum, unnormalised accumulator) are merged afterwards) is not on the pages;
it is the exact rewriting of steps 2-4 that long sequences use.  It is written
here so the tests can pin it: merging the partials of any partition of 0..L-1
equals step 4.
"""
from __future__ import annotations

import numpy as np

from .fp import decode


def gather_logical_kv(cache_bits: np.ndarray, table_row, length: int, kv_head: int,
                      block_size: int, dtype: str) -> np.ndarray:
    """Step 1: the sequence's K (or V) rows in logical order, as float64 [L, D]."""
    t = np.arange(length)
    phys = np.asarray(table_row, dtype=np.int64)[t // block_size]
    off = t % block_size
    return decode(cache_bits[phys, kv_head, off, :], dtype)


def softmax_attention(qvec: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Steps 2-4 for one query vector over contiguous K, V [L, D] (float64)."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    z = scale * (K @ qvec)
    z = z - z.max()
    w = np.exp(z)
    w = w / w.sum()
    return w @ V


def paged_decode_attention(q_bits, k_cache_bits, v_cache_bits, block_tables, context_lens,
                           scale: float, num_kv_heads: int, block_size: int, dtype: str,
                           seqs=None) -> np.ndarray:
    """out [S, Hq, D] float64.  ``seqs`` restricts the work to some sequences
    (rows of other sequences are left NaN)."""
    S, Hq, D = q_bits.shape
    assert Hq % num_kv_heads == 0
    G = Hq // num_kv_heads
    out = np.full((S, Hq, D), np.nan, dtype=np.float64)
    todo = range(S) if seqs is None else seqs
    for s in todo:
        L = int(context_lens[s])
        qs = decode(q_bits[s], dtype)
        for kh in range(num_kv_heads):
            K = gather_logical_kv(k_cache_bits, block_tables[s], L, kh, block_size, dtype)
            V = gather_logical_kv(v_cache_bits, block_tables[s], L, kh, block_size, dtype)
            for h in range(kh * G, (kh + 1) * G):
                out[s, h] = softmax_attention(qs[h], K, V, scale)
    return out


# ----------------------------------------------------------------------------
# split-context partials
# ----------------------------------------------------------------------------

def partial_attention(qvec: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """(m, l, acc) of one partition: m = max z, l = sum exp(z - m),
    acc = sum exp(z - m) V."""
    z = scale * (K @ qvec)
    m = z.max()
    p = np.exp(z - m)
    return m, p.sum(), p @ V


def merge_partials(parts) -> np.ndarray:
    """Merge partition results: with M = max_i m_i,
    out = sum_i exp(m_i - M) acc_i / sum_i exp(m_i - M) l_i."""
    M = max(m for m, _, _ in parts)
    num = sum(np.exp(m - M) * acc for m, _, acc in parts)
    den = sum(np.exp(m - M) * l for m, l, _ in parts)
    return num / den


def split_context_attention(qvec, K, V, scale: float, partition: int) -> np.ndarray:
    """Steps 2-4 computed partition by partition (``partition`` tokens each)
    and merged."""
    L = K.shape[0]
    parts = [partial_attention(qvec, K[a:a + partition], V[a:a + partition], scale)
             for a in range(0, L, partition)]
    return merge_partials(parts)


# ----------------------------------------------------------------------------
# chunked prefill: several new tokens of a sequence at once
# ----------------------------------------------------------------------------

def paged_prefill_attention(q_bits, k_cache_bits, v_cache_bits, block_tables, context_lens,
                            query_start, scale: float, num_kv_heads: int, block_size: int,
                            dtype: str, seqs=None) -> np.ndarray:
    """Attention of a chunk of new tokens per sequence over the paged cache.

    Not on the pages beyond their statement that attention runs block by
    block over non-contiguous blocks ([P3] second paragraph) and that the
    KV cache is filled as tokens arrive ([P1] section 2); written here as the
    plainest multi-token form of steps 1-4.  Sequence s owns the query rows
    query_start[s] .. query_start[s+1]-1 of ``q_bits`` [T, Hq, D]: its last
    C_s = query_start[s+1] - query_start[s] tokens, whose K/V are already in
    the cache (the cache write comes first, as in decode), so its context
    holds L_s = context_lens[s] >= C_s tokens.  Row i (0 <= i < C_s) is the
    token at position p = L_s - C_s + i and, causally, attends to positions
    0 .. p only.  C_s = 1 is a decode step.  Returns out [T, Hq, D] float64
    (rows of sequences not in ``seqs`` left NaN)."""
    T, Hq, D = q_bits.shape
    assert Hq % num_kv_heads == 0
    G = Hq // num_kv_heads
    out = np.full((T, Hq, D), np.nan, dtype=np.float64)
    todo = range(len(context_lens)) if seqs is None else seqs
    for s in todo:
        a, b = int(query_start[s]), int(query_start[s + 1])
        C, L = b - a, int(context_lens[s])
        assert 0 <= C <= L
        for kh in range(num_kv_heads):
            K = gather_logical_kv(k_cache_bits, block_tables[s], L, kh, block_size, dtype)
            V = gather_logical_kv(v_cache_bits, block_tables[s], L, kh, block_size, dtype)
            for i in range(C):
                p = L - C + i
                qs = decode(q_bits[a + i], dtype)
                for h in range(kh * G, (kh + 1) * G):
                    out[a + i, h] = softmax_attention(qs[h], K[:p + 1], V[:p + 1], scale)
    return out
