"""Python binding of libpa.so, the B200 paged-KV-cache attention library.

Argument marshalling only: every function here checks the torch tensors it is
given, passes their device pointers, sizes and the current CUDA stream to the
C ABI declared in include/pa.h, and raises on a non-zero status.  No step of
the computation runs in Python, and there is no fallback: if libpa.so is
missing or a call fails, an exception is raised.

Names follow the C ABI: ``pa_reshape_and_cache``, ``pa_paged_decode_attention``
(with ``pa_paged_decode_workspace_bytes``, and ``pa_paged_decode_attention_no_alloc``),
the fused ``pa_decode_step``, ``pa_paged_prefill_attention`` (chunked prefill),
``pa_copy_blocks``, ``pa_device_error``, ``pa_decode_tuning``, ``pa_set_wait_limit``,
and the host block manager ``BlockManager`` over the ``pa_bm_*`` calls (prefix
caching included).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_F16, PA_BF16 = 0, 1
STATUS = {0: "PA_OK", -1: "PA_ERR_ARG", -2: "PA_ERR_UNSUPPORTED", -3: "PA_ERR_NO_BLOCKS",
          -4: "PA_ERR_SEQ", -5: "PA_ERR_CUDA", -6: "PA_ERR_DEVICE_BOUNDS", -7: "PA_ERR_WORKSPACE"}
DEVERR = {"block_id": 0x1, "context_len": 0x2, "slot": 0x4, "copy_pair": 0x8, "timeout": 0x10,
          "range": 0x20}


class PAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class NoBlocksError(PAError):
    pass


class SeqError(PAError):
    pass


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if libpa.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} not found: build it with "
                              "`python -m paged_kv_cache_414_b200.build`")
        _lib = ctypes.CDLL(LIB_PATH)
        _declare(_lib)
    return _lib


class BmStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("num_blocks", "free_blocks", "used_blocks",
                                               "shared_blocks", "num_seqs", "logical_tokens",
                                               "filled_slots", "block_size")]


def _declare(L):
    c = ctypes
    vp, i32, i64, sz, f32 = c.c_void_p, c.c_int, c.c_int64, c.c_size_t, c.c_float
    P64, P32 = c.POINTER(c.c_int64), c.POINTER(c.c_int32)
    sig = {
        "pa_status_string": (c.c_char_p, [i32]),
        "pa_version": (i32, []),
        "pa_reshape_and_cache": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]),
        "pa_paged_decode_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
        "pa_paged_decode_attention": (i32, [vp, vp, vp, vp, vp, vp, f32, i32, i32, i32, i32, i32,
                                            i32, i32, i32, i32, vp, sz, vp]),
        "pa_paged_decode_attention_no_alloc": (i32, [vp, vp, vp, vp, vp, vp, f32, i32, i32, i32,
                                                     i32, i32, i32, i32, i32, i32, vp]),
        "pa_decode_step": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, f32, i32, i32, i32, i32, i32,
                                 i32, i32, i32, i32, vp, sz, vp]),
        "pa_decode_tuning": (i32, [i32, i32, i32]),
        "pa_set_wait_limit": (i32, [c.c_longlong]),
        "pa_paged_prefill_attention": (i32, [vp, vp, vp, vp, vp, vp, vp, f32, i32, i32, i32, i32,
                                             i32, i32, i32, i32, i32, i32, vp]),
        "pa_copy_blocks": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]),
        "pa_device_error": (i32, [c.POINTER(c.c_uint), i32]),
        "pa_bm_create": (vp, [i32, i32, P32]),
        "pa_bm_destroy": (None, [vp]),
        "pa_bm_allocate": (i32, [vp, i64, i32, P64]),
        "pa_bm_fork": (i32, [vp, i64, i64]),
        "pa_bm_append_slot": (i32, [vp, i64, P64, P32, P32]),
        "pa_bm_append_slots": (i32, [vp, P64, i32, P64, P64, c.POINTER(c.c_int)]),
        "pa_bm_free": (i32, [vp, i64]),
        "pa_bm_block_table": (i32, [vp, i64, P32, i32, c.POINTER(c.c_int)]),
        "pa_bm_block_tables": (i32, [vp, P64, i32, P32, i32, P32]),
        "pa_bm_seq_len": (i32, [vp, i64]),
        "pa_bm_num_free": (i32, [vp]),
        "pa_bm_ref_count": (i32, [vp, c.c_int32]),
        "pa_bm_num_seqs": (i32, [vp]),
        "pa_bm_stats": (i32, [vp, c.POINTER(BmStats)]),
        "pa_bm_allocate_prefix": (i32, [vp, i64, P32, i32, P64, c.POINTER(c.c_int)]),
        "pa_bm_num_cached": (i32, [vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def _check(status: int, what: str):
    if status != 0:
        if status == -3:
            raise NoBlocksError(status, what)
        if status == -4:
            raise SeqError(status, what)
        raise PAError(status, what)


# --------------------------------------------------------------------------- torch marshalling

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"K/V/q must be float16 or bfloat16, got {t.dtype}")


def _dev(t, name, dtype=None, ndim=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None):
    """cache[slot // B, :, slot % B, :] = key[t] (and value) for every token t."""
    torch = _torch()
    NB, Hkv, B, D = k_cache.shape
    T = key.shape[0]
    if tuple(key.shape) != (T, Hkv, D) or tuple(value.shape) != (T, Hkv, D):
        raise ValueError("key/value must be [num_tokens, num_kv_heads, head_dim]")
    if v_cache.shape != k_cache.shape or key.dtype != k_cache.dtype or value.dtype != k_cache.dtype:
        raise ValueError("cache/key/value shapes or dtypes disagree")
    if slot_mapping.shape != (T,):
        raise ValueError("slot_mapping must be [num_tokens]")
    st = lib().pa_reshape_and_cache(
        _dev(key, "key"), _dev(value, "value"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D, B, NB,
        _dtype_code(k_cache), _stream(stream))
    _check(st, "pa_reshape_and_cache")


def pa_paged_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                    max_context_len) -> int:
    n = lib().pa_paged_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              block_size, max_context_len)
    if n == 0:
        raise PAError(-1, "pa_paged_decode_workspace_bytes")
    return int(n)


def alloc_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                    device=None):
    """A device workspace tensor of the size the library asks for."""
    torch = _torch()
    n = pa_paged_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                        block_size, max_context_len)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def pa_paged_decode_attention(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                              num_kv_heads, max_context_len=None, workspace=None, stream=None):
    """out[s, h] = softmax(scale * q[s, h] K_s^T) V_s over the sequence's cached tokens."""
    torch = _torch()
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    if Hkv != num_kv_heads or D2 != D:
        raise ValueError("q / cache shapes disagree")
    if tuple(out.shape) != (S, Hq, D):
        raise ValueError("out must be [num_seqs, num_q_heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables [S, max_blocks] / context_lens [S] expected")
    maxb = int(block_tables.shape[1])
    if max_context_len is None:
        max_context_len = maxb * B
    if workspace is None:
        workspace = alloc_workspace(S, Hq, Hkv, D, B, max_context_len, q.device)
    st = lib().pa_paged_decode_attention(
        _dev(out, "out", torch.float32), _dev(q, "q", k_cache.dtype), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache", k_cache.dtype), _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), float(scale), Hkv, S, Hq, D, B, maxb,
        int(max_context_len), NB, _dtype_code(k_cache), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "pa_paged_decode_attention")
    return out


def pa_paged_decode_attention_no_alloc(out, q, k_cache, v_cache, block_tables, context_lens,
                                       scale, num_kv_heads, max_context_len=None, stream=None):
    """pa_paged_decode_attention without a workspace: the library's own fixed
    scratch array is used, and nothing is allocated (not even here), for
    callers that cannot allocate device memory.  Calls that may overlap on
    the GPU share that scratch and must be serialised by the caller."""
    torch = _torch()
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    if Hkv != num_kv_heads or D2 != D:
        raise ValueError("q / cache shapes disagree")
    if tuple(out.shape) != (S, Hq, D):
        raise ValueError("out must be [num_seqs, num_q_heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables [S, max_blocks] / context_lens [S] expected")
    maxb = int(block_tables.shape[1])
    if max_context_len is None:
        max_context_len = maxb * B
    st = lib().pa_paged_decode_attention_no_alloc(
        _dev(out, "out", torch.float32), _dev(q, "q", k_cache.dtype), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache", k_cache.dtype), _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), float(scale), Hkv, S, Hq, D, B, maxb,
        int(max_context_len), NB, _dtype_code(k_cache), _stream(stream))
    _check(st, "pa_paged_decode_attention_no_alloc")
    return out


def pa_decode_step(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, scale,
                   num_kv_heads, max_context_len=None, workspace=None, stream=None):
    """One fused decode step: store each sequence's newest token (k_new/v_new
    [S, Hkv, D]) at position L-1 of its block table and attend over all L
    tokens; equals pa_reshape_and_cache followed by pa_paged_decode_attention."""
    torch = _torch()
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    if Hkv != num_kv_heads or D2 != D:
        raise ValueError("q / cache shapes disagree")
    if tuple(k_new.shape) != (S, Hkv, D) or tuple(v_new.shape) != (S, Hkv, D):
        raise ValueError("k_new / v_new must be [num_seqs, num_kv_heads, head_dim]")
    if tuple(out.shape) != (S, Hq, D):
        raise ValueError("out must be [num_seqs, num_q_heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables [S, max_blocks] / context_lens [S] expected")
    maxb = int(block_tables.shape[1])
    if max_context_len is None:
        max_context_len = maxb * B
    if workspace is None:
        workspace = alloc_workspace(S, Hq, Hkv, D, B, max_context_len, q.device)
    dt = k_cache.dtype
    st = lib().pa_decode_step(
        _dev(out, "out", torch.float32), _dev(q, "q", dt), _dev(k_new, "k_new", dt),
        _dev(v_new, "v_new", dt), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache", dt),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), float(scale), Hkv, S, Hq, D, B, maxb,
        int(max_context_len), NB, _dtype_code(k_cache), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "pa_decode_step")
    return out


def pa_paged_prefill_attention(out, q, k_cache, v_cache, block_tables, context_lens,
                               query_start, scale, num_kv_heads, max_query_len, stream=None):
    """Chunked prefill: query row t of sequence s (rows query_start[s] ..
    query_start[s+1]-1, the sequence's last tokens, already in the cache) at
    position p attends to positions 0..p of its sequence.  q [T, Hq, D],
    out [T, Hq, D] fp32; max_query_len bounds every chunk (host int)."""
    torch = _torch()
    T, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    if Hkv != num_kv_heads or D2 != D:
        raise ValueError("q / cache shapes disagree")
    if tuple(out.shape) != (T, Hq, D):
        raise ValueError("out must be [num_tokens, num_q_heads, head_dim]")
    S = int(context_lens.shape[0])
    if block_tables.dim() != 2 or block_tables.shape[0] != S or query_start.shape != (S + 1,):
        raise ValueError("block_tables [S, max_blocks] / query_start [S + 1] expected")
    st = lib().pa_paged_prefill_attention(
        _dev(out, "out", torch.float32), _dev(q, "q", k_cache.dtype), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache", k_cache.dtype), _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32),
        _dev(query_start, "query_start", torch.int32), float(scale), Hkv, S, T, Hq, D, B,
        int(block_tables.shape[1]), int(max_query_len), NB, _dtype_code(k_cache),
        _stream(stream))
    _check(st, "pa_paged_prefill_attention")
    return out


def pa_decode_tuning(nstage=0, ctas_per_sm=0, min_tiles_per_warp=0):
    _check(lib().pa_decode_tuning(nstage, ctas_per_sm, min_tiles_per_warp), "pa_decode_tuning")


def pa_set_wait_limit(ns: int = 0):
    """Limit (ns) of every bounded wait in kernels launched afterwards; 0 = the default 2 s."""
    _check(lib().pa_set_wait_limit(int(ns)), "pa_set_wait_limit")


def pa_copy_blocks(k_cache, v_cache, block_mapping, stream=None):
    """k_cache[dst] = k_cache[src] (and V) for every (src, dst) row of block_mapping."""
    torch = _torch()
    NB, Hkv, B, D = k_cache.shape
    if block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise ValueError("block_mapping must be [num_pairs, 2]")
    st = lib().pa_copy_blocks(
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache", k_cache.dtype),
        _dev(block_mapping, "block_mapping", torch.int64), int(block_mapping.shape[0]), Hkv, D,
        B, NB, _dtype_code(k_cache), _stream(stream))
    _check(st, "pa_copy_blocks")


def pa_device_error(clear: bool = True) -> int:
    """Sticky device error bits (synchronises the device)."""
    v = ctypes.c_uint(0)
    st = lib().pa_device_error(ctypes.byref(v), 1 if clear else 0)
    if st not in (0, -6):
        _check(st, "pa_device_error")
    return int(v.value)


# --------------------------------------------------------------------------- block manager

def _out(a, shape, dtype):
    """A caller-provided output array (numpy, or a CPU torch tensor such as a
    pinned buffer) checked for shape, dtype and contiguity."""
    if not isinstance(a, np.ndarray):
        a = a.numpy()
    if a.shape != tuple(shape) or a.dtype != dtype or not a.flags.c_contiguous:
        raise ValueError(f"output array must be contiguous {np.dtype(dtype)} {tuple(shape)}, "
                         f"got {a.dtype} {a.shape}")
    return a


def _p64(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _p32(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


class BlockManager:
    """Host block manager (free list, reference counts, fork, copy-on-write)
    of libpa.so.  Methods mirror the pa_bm_* calls."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
            if order.shape != (self.num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
        h = lib().pa_bm_create(self.num_blocks, self.block_size,
                               None if order is None else _p32(order))
        if not h:
            raise ValueError("pa_bm_create rejected the pool description")
        self._h = ctypes.c_void_p(h)

    def close(self):
        if getattr(self, "_h", None):
            lib().pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def allocate(self, seq: int, num_tokens: int) -> np.ndarray:
        slots = np.empty(max(num_tokens, 0), dtype=np.int64)
        _check(lib().pa_bm_allocate(self._h, seq, num_tokens, _p64(slots)), "pa_bm_allocate")
        return slots

    def allocate_prefix(self, seq: int, tokens, slots_out=None):
        """Allocate a prompt of token ids, reusing cached full blocks whose
        whole token prefix matches.  Returns (slots int64 [n], -1 for the
        cached tokens; number of cached tokens)."""
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        n = toks.shape[0]
        slots = (np.empty(n, dtype=np.int64) if slots_out is None
                 else _out(slots_out, (n,), np.int64))
        got = ctypes.c_int(0)
        _check(lib().pa_bm_allocate_prefix(self._h, seq, _p32(toks), n, _p64(slots),
                                           ctypes.byref(got)), "pa_bm_allocate_prefix")
        return slots, int(got.value)

    def num_cached(self) -> int:
        """Blocks entered in the prefix cache (held by a sequence or free)."""
        return lib().pa_bm_num_cached(self._h)

    def fork(self, parent: int, child: int) -> None:
        _check(lib().pa_bm_fork(self._h, parent, child), "pa_bm_fork")

    def append_slot(self, seq: int):
        slot = ctypes.c_int64()
        cs, cd = ctypes.c_int32(-1), ctypes.c_int32(-1)
        r = lib().pa_bm_append_slot(self._h, seq, ctypes.byref(slot), ctypes.byref(cs),
                                    ctypes.byref(cd))
        if r < 0:
            _check(r, "pa_bm_append_slot")
        return int(slot.value), ((int(cs.value), int(cd.value)) if r == 1 else None)

    def append_slots(self, seqs, slots_out=None, pairs_out=None):
        """(slots int64 [n], cow_pairs int64 [k, 2]) for one append per entry.
        With `slots_out` ([n] int64) and `pairs_out` ([n, 2] int64), e.g. views
        of pinned host memory, the results are written there and views of them
        returned."""
        seqs = np.ascontiguousarray(seqs, dtype=np.int64)
        n = seqs.shape[0]
        slots = (np.empty(n, dtype=np.int64) if slots_out is None
                 else _out(slots_out, (n,), np.int64))
        pairs = (np.empty((max(n, 1), 2), dtype=np.int64) if pairs_out is None
                 else _out(pairs_out, (max(n, 1), 2), np.int64))
        k = ctypes.c_int(0)
        _check(lib().pa_bm_append_slots(self._h, _p64(seqs), n, _p64(slots), _p64(pairs),
                                        ctypes.byref(k)), "pa_bm_append_slots")
        return slots, (pairs[:k.value] if pairs_out is not None else pairs[:k.value].copy())

    def free_seq(self, seq: int) -> None:
        _check(lib().pa_bm_free(self._h, seq), "pa_bm_free")

    def block_table(self, seq: int) -> list:
        n = self.seq_len(seq)
        cap = max(1, -(-n // self.block_size))
        out = np.empty(cap, dtype=np.int32)
        got = ctypes.c_int(0)
        _check(lib().pa_bm_block_table(self._h, seq, _p32(out), cap, ctypes.byref(got)),
               "pa_bm_block_table")
        return out[:got.value].tolist()

    def block_tables(self, seqs, cap: int, out=None, lens_out=None):
        """(tables int32 [n, cap] padded with -1, lens int32 [n]); written into
        `out` / `lens_out` when given (contiguous int32 arrays of those shapes)."""
        seqs = np.ascontiguousarray(seqs, dtype=np.int64)
        n = seqs.shape[0]
        out = np.empty((n, cap), dtype=np.int32) if out is None else _out(out, (n, cap), np.int32)
        lens = np.empty(n, dtype=np.int32) if lens_out is None else _out(lens_out, (n,), np.int32)
        _check(lib().pa_bm_block_tables(self._h, _p64(seqs), n, _p32(out), cap, _p32(lens)),
               "pa_bm_block_tables")
        return out, lens

    def seq_len(self, seq: int) -> int:
        r = lib().pa_bm_seq_len(self._h, seq)
        if r < 0:
            _check(r, "pa_bm_seq_len")
        return r

    def num_free(self) -> int:
        return lib().pa_bm_num_free(self._h)

    def ref_count(self, block: int) -> int:
        r = lib().pa_bm_ref_count(self._h, block)
        if r < 0:
            _check(r, "pa_bm_ref_count")
        return r

    def num_seqs(self) -> int:
        return lib().pa_bm_num_seqs(self._h)

    def stats(self) -> dict:
        """pa_bm_stats as a dict: blocks (total, free, used, shared), live
        sequences, logical tokens, filled slots, block size."""
        st = BmStats()
        _check(lib().pa_bm_stats(self._h, ctypes.byref(st)), "pa_bm_stats")
        return {name: int(getattr(st, name)) for name, _ in BmStats._fields_}
