"""Shared plumbing of the GPU parity tests (not a test module).

The expected side of every comparison is computed by oracle/ code only, from
the generator's inputs as drawn (copied to the host before any library kernel
touches them).  The library side runs the native block manager and the CUDA
kernels through the binding.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as OA
from oracle import cache_ops as OC
from oracle.block_manager import BlockManager as OracleBM
import workloads as W

TOL = 2e-3   # max-abs error allowed for attention outputs (fp32 accumulate vs fp64)


class Expected:
    """Oracle result of one decode step on (a sample of) a generated batch.
    With ``whole_pool`` the oracle's cache write is also applied to a host
    copy of the entire pool (``k_pool``, ``v_pool``: bits after the step)."""

    def __init__(self, batch: W.DecodeBatch, seqs=None, whole_pool: bool = False):
        sh = batch.shape
        B = sh.block_size
        S = batch.num_seqs
        self.seqs = list(range(S)) if seqs is None else sorted(set(int(s) for s in seqs))
        # slots from the oracle's block manager: whole sequences, in order
        bm = OracleBM(batch.num_blocks, B, batch.free_order)
        self.slots = np.empty(S, dtype=np.int64)
        for s in range(S):
            L = int(batch.context_lens[s])
            sl = bm.allocate(s, L)
            self.slots[s] = sl[-1] if L > 0 else -1
        self.tables = {s: bm.block_table(s) for s in range(S)}
        if whole_pool:
            self.k_pool, self.v_pool = W.bits(batch.k_cache), W.bits(batch.v_cache)
            OC.reshape_and_cache(W.bits(batch.k_new), W.bits(batch.v_new), self.k_pool,
                                 self.v_pool, self.slots, B)
        # the needed part of the pool, as drawn
        need = sorted({b for s in self.seqs for b in self.tables[s]})
        self.blocks = np.array(need, dtype=np.int64)
        remap = {b: i for i, b in enumerate(need)}
        idx = torch.as_tensor(self.blocks, device=batch.k_cache.device)
        kb = W.bits(batch.k_cache.index_select(0, idx)) if len(need) else np.zeros((0,) + tuple(batch.k_cache.shape[1:]), np.uint16)
        vb = W.bits(batch.v_cache.index_select(0, idx)) if len(need) else kb.copy()
        qb = W.bits(batch.q)[self.seqs]
        knb = W.bits(batch.k_new)[self.seqs]
        vnb = W.bits(batch.v_new)[self.seqs]
        sub_slots = []
        for s in self.seqs:
            sl = int(self.slots[s])
            sub_slots.append(-1 if sl < 0 else remap[sl // B] * B + sl % B)
        OC.reshape_and_cache(knb, vnb, kb, vb, np.array(sub_slots), B)
        self.k_after, self.v_after = kb, vb
        maxb = max([len(self.tables[s]) for s in self.seqs] + [1])
        sub_tables = np.full((len(self.seqs), maxb), -1, dtype=np.int64)
        for i, s in enumerate(self.seqs):
            t = [remap[b] for b in self.tables[s]]
            sub_tables[i, :len(t)] = t
        lens = batch.context_lens[self.seqs]
        self.out = OA.paged_decode_attention(qb, kb, vb, sub_tables, lens, batch.scale,
                                             sh.num_kv_heads, B, sh.dtype)


def library_fused_step(pa, batch: W.DecodeBatch, max_context_len=None):
    """One decode step through the fused entry point pa_decode_step (cache
    write of the newest token + attention in one launch), with a workspace of
    pa_paged_decode_workspace_bytes as the benchmark allocates it.  Returns
    (tables, out)."""
    sh = batch.shape
    S = batch.num_seqs
    bm = pa.BlockManager(batch.num_blocks, sh.block_size, batch.free_order)
    for s in range(S):
        bm.allocate(s, int(batch.context_lens[s]))
    tables, lens = bm.block_tables(np.arange(S), batch.max_blocks_per_seq)
    dev = batch.q.device
    out = torch.empty(S, sh.num_q_heads, sh.head_dim, dtype=torch.float32, device=dev)
    if max_context_len is None:
        max_context_len = int(batch.context_lens.max(initial=0))
    ws = pa.alloc_workspace(S, sh.num_q_heads, sh.num_kv_heads, sh.head_dim, sh.block_size,
                            max_context_len, dev)
    pa.pa_decode_step(out, batch.q, batch.k_new, batch.v_new, batch.k_cache, batch.v_cache,
                      torch.as_tensor(tables, device=dev), torch.as_tensor(lens, device=dev),
                      batch.scale, sh.num_kv_heads, max_context_len=max_context_len,
                      workspace=ws)
    torch.cuda.synchronize()
    return tables, out


def library_step(pa, batch: W.DecodeBatch, tuning=None):
    """One decode step through the library: native manager slots, cache write,
    attention.  Returns (slots, tables, out)."""
    sh = batch.shape
    B = sh.block_size
    S = batch.num_seqs
    bm = pa.BlockManager(batch.num_blocks, B, batch.free_order)
    slots = np.empty(S, dtype=np.int64)
    for s in range(S):
        L = int(batch.context_lens[s])
        sl = bm.allocate(s, L)
        slots[s] = sl[-1] if L > 0 else -1
    maxb = batch.max_blocks_per_seq
    tables, lens = bm.block_tables(np.arange(S), maxb)
    dev = batch.q.device
    d_slots = torch.as_tensor(slots, device=dev)
    d_tables = torch.as_tensor(tables, device=dev)
    d_lens = torch.as_tensor(lens, device=dev)
    pa.pa_reshape_and_cache(batch.k_new, batch.v_new, batch.k_cache, batch.v_cache, d_slots)
    out = torch.empty(S, sh.num_q_heads, sh.head_dim, dtype=torch.float32, device=dev)
    if tuning is not None:
        pa.pa_decode_tuning(*tuning)
    try:
        pa.pa_paged_decode_attention(out, batch.q, batch.k_cache, batch.v_cache, d_tables, d_lens,
                                     batch.scale, sh.num_kv_heads,
                                     max_context_len=int(batch.context_lens.max(initial=0)))
    finally:
        if tuning is not None:
            pa.pa_decode_tuning(0, 0, 0)
    torch.cuda.synchronize()
    return slots, tables, out


def max_abs_err(got: np.ndarray, want: np.ndarray) -> float:
    return float(np.max(np.abs(got.astype(np.float64) - want))) if want.size else 0.0
