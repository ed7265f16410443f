"""Seeded synthetic inputs for paged decode attention.

This module only draws random numbers and lays them out in the shapes of the
decode workloads below; it performs no step of the attention method itself
(no block-table lookup for attention, no softmax, no cache write).  Both the
CPU oracle (``oracle/``) and the CUDA library are fed from here, so that the
two sides see the same bits while sharing no arithmetic.

Workloads (sizes follow the decode shapes the library is built for):

* ``tiny``   4 sequences, context lengths {1, 17, 33, 100}, block size 16,
             4 q heads = 4 kv heads, head_dim 64, fp16, pool of 32 blocks.
* ``13b``    64 sequences, 40 q heads = 40 kv heads, head_dim 128, block 16,
             fp16, lengths uniform on 1..2048, pool = used blocks + 10 %.
* ``gqa8b``  256 sequences, 32 q heads over 8 kv heads, head_dim 128, block 16,
             bf16, lengths lognormal (median 512, sigma 1) clipped to 16..4096.
* ``cow``    32 prompts of length uniform 64..512, each forked into 8 branches
             sharing the prompt's blocks, gqa8b head shapes, 64 decode steps.
* ``long``   8 sequences, lengths uniform 16384..32768, 64 q heads over 8 kv
             heads, head_dim 128, bf16, block 16 or 32, K given a large offset
             along the group's mean query at 8 positions per sequence so the
             softmax is peaked.
* ``prefix`` chat-like requests sharing a few system prompts (or an earlier
             request plus a new turn), at most 12 alive at once, with K/V
             rows that depend only on the token prefix (prefix caching).

Draw order for every batch: context lengths, then the physical block
permutation (numpy PCG64 seeded with ``seed``); then q, K pool, V pool, new K,
new V (torch generator seeded with ``seed`` on the requested device), each drawn
in fp32 from N(0, 1) and rounded to nearest-even into the storage dtype.

Conventions shared by both sides:

* ``context_lens[s]`` counts every token of sequence ``s`` including the one
  appended this step; the cache holds stale random values in that token's slot
  until the step's new K/V is written.
* The pool layout is ``[num_blocks, num_kv_heads, block_size, head_dim]``.
* Blocks are handed out as consecutive runs of one random permutation of the
  pool, sequence by sequence; ``free_order`` is that permutation, so a
  first-in-first-out free list seeded with it hands out the same blocks.
* Unused block-table entries are ``-1``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}
NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a 16-bit tensor (copied to host)."""
    assert t.element_size() == 2
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(a: np.ndarray, dtype: str, device="cpu") -> torch.Tensor:
    """Inverse of :func:`bits`."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.view(TORCH_DTYPES[dtype]).to(device)


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


# --------------------------------------------------------------------------
# context-length recipes
# --------------------------------------------------------------------------

def lens_tiny(rng: np.random.Generator) -> np.ndarray:
    return np.array([1, 17, 33, 100], dtype=np.int32)


def lens_13b(rng: np.random.Generator, num_seqs: int = 64) -> np.ndarray:
    return rng.integers(1, 2048, size=num_seqs, endpoint=True).astype(np.int32)


def lens_gqa8b(rng: np.random.Generator, num_seqs: int = 256) -> np.ndarray:
    raw = 512.0 * np.exp(rng.standard_normal(num_seqs))
    return np.clip(np.rint(raw), 16, 4096).astype(np.int32)


def lens_long(rng: np.random.Generator, num_seqs: int = 8) -> np.ndarray:
    return rng.integers(16384, 32768, size=num_seqs, endpoint=True).astype(np.int32)


@dataclass(frozen=True)
class Shape:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


SHAPES = {
    "tiny": Shape(4, 4, 64, 16, "f16"),
    "13b": Shape(40, 40, 128, 16, "f16"),
    "gqa8b": Shape(32, 8, 128, 16, "bf16"),
    "cow": Shape(32, 8, 128, 16, "bf16"),
    "long": Shape(64, 8, 128, 16, "bf16"),
    "long32": Shape(64, 8, 128, 32, "bf16"),
}
SEEDS = {"tiny": 0, "13b": 1, "gqa8b": 2, "cow": 3, "long": 4, "long32": 5}


# --------------------------------------------------------------------------
# one decode batch
# --------------------------------------------------------------------------

@dataclass
class DecodeBatch:
    shape: Shape
    context_lens: np.ndarray          # int32 [S]
    block_tables: np.ndarray          # int32 [S, max_blocks_per_seq], -1 = unused
    free_order: np.ndarray            # int32 [num_blocks], the pool permutation
    num_blocks: int
    q: torch.Tensor                   # [S, Hq, D]
    k_cache: torch.Tensor             # [num_blocks, Hkv, B, D]
    v_cache: torch.Tensor
    k_new: torch.Tensor               # [S, Hkv, D] the token appended this step
    v_new: torch.Tensor
    scale: float
    hot_positions: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    def blocks_in_use(self) -> int:
        return int(sum(_ceil_div(int(x), self.shape.block_size) for x in self.context_lens))


def make_decode_batch(shape: Shape, context_lens, seed: int, *, device="cpu",
                      num_blocks: int | None = None, spare_fraction: float = 0.10,
                      max_blocks_per_seq: int | None = None, poison: str | None = None,
                      rng: np.random.Generator | None = None) -> DecodeBatch:
    """Draw one decode batch.

    ``poison='nan'`` fills every slot that holds no token of any sequence (the
    tail of each last block and every unassigned block) with NaN, so a kernel
    that reads past a sequence's length shows it in the output.
    """
    rng = rng if rng is not None else np.random.default_rng(seed)
    lens = np.asarray(context_lens, dtype=np.int32)
    B = shape.block_size
    nb = [_ceil_div(int(x), B) for x in lens]
    used = int(sum(nb))
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(used * (1.0 + spare_fraction))))
    assert num_blocks >= used
    maxb = max_blocks_per_seq if max_blocks_per_seq is not None else max(1, max(nb, default=1))
    assert maxb >= max(nb, default=0)
    perm = rng.permutation(num_blocks).astype(np.int32)
    tables = np.full((len(lens), maxb), -1, dtype=np.int32)
    off = 0
    for s, n in enumerate(nb):
        tables[s, :n] = perm[off:off + n]
        off += n

    dt = TORCH_DTYPES[shape.dtype]
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    S, Hq, Hkv, D = len(lens), shape.num_q_heads, shape.num_kv_heads, shape.head_dim

    def draw(*dims):
        return torch.randn(*dims, generator=g, device=device, dtype=torch.float32).to(dt)

    q = draw(S, Hq, D)
    k_cache = draw(num_blocks, Hkv, B, D)
    v_cache = draw(num_blocks, Hkv, B, D)
    k_new = draw(S, Hkv, D)
    v_new = draw(S, Hkv, D)

    if poison == "nan":
        valid = torch.zeros(num_blocks, B, dtype=torch.bool)
        for s, n in enumerate(nb):
            for j in range(n):
                fill = min(B, int(lens[s]) - j * B)
                valid[int(tables[s, j]), :fill] = True
        valid = valid.to(device)
        nan = torch.tensor(NAN_BITS[shape.dtype], dtype=torch.int16, device=device).view(dt)
        mask = (~valid)[:, None, :, None].expand(num_blocks, Hkv, B, D)
        k_cache[mask] = nan
        v_cache[mask] = nan
    elif poison is not None:
        raise ValueError(poison)

    return DecodeBatch(shape=shape, context_lens=lens, block_tables=tables, free_order=perm,
                       num_blocks=num_blocks, q=q, k_cache=k_cache, v_cache=v_cache,
                       k_new=k_new, v_new=v_new, scale=1.0 / math.sqrt(D))


def add_peaked_offsets(batch: DecodeBatch, rng: np.random.Generator, hot_per_seq: int = 8,
                       edge: int = 512) -> None:
    """Make the softmax peaked: at ``hot_per_seq`` positions of each sequence add
    ``3*sqrt(D)*u`` to K, with ``u`` the unit vector along the mean of the
    group's query vectors (one position within the first ``edge`` tokens, one
    within the last ``edge`` tokens, the rest uniform).  Positions are placed in
    the blocks this module itself handed to the sequence."""
    sh = batch.shape
    B, G, D = sh.block_size, sh.group, sh.head_dim
    dt = TORCH_DTYPES[sh.dtype]
    for s, L in enumerate(batch.context_lens):
        L = int(L)
        first = int(rng.integers(0, min(edge, L)))
        last = int(rng.integers(max(0, L - edge), L))
        rest = rng.integers(0, L, size=max(0, hot_per_seq - 2)).tolist()
        pos = sorted(set([first, last] + [int(x) for x in rest]))
        batch.hot_positions[s] = pos
        qs = batch.q[s].float().view(sh.num_kv_heads, G, D).mean(dim=1)
        u = qs / qs.norm(dim=-1, keepdim=True).clamp_min(1e-12)
        for t in pos:
            blk = int(batch.block_tables[s, t // B])
            row = batch.k_cache[blk, :, t % B, :].float() + 3.0 * math.sqrt(D) * u
            batch.k_cache[blk, :, t % B, :] = row.to(dt)


def standard_batch(name: str, device="cpu", **kw) -> DecodeBatch:
    """The seeded batch of one named workload (not ``cow``)."""
    sh = SHAPES[name]
    seed = SEEDS[name]
    rng = np.random.default_rng(seed)
    if name == "tiny":
        lens = lens_tiny(rng)
        kw.setdefault("num_blocks", 32)
    elif name == "13b":
        lens = lens_13b(rng)
    elif name == "gqa8b":
        lens = lens_gqa8b(rng)
    elif name in ("long", "long32"):
        lens = lens_long(rng)
    else:
        raise ValueError(name)
    b = make_decode_batch(sh, lens, seed, device=device, rng=rng, **kw)
    if name in ("long", "long32"):
        add_peaked_offsets(b, rng)
    return b


# --------------------------------------------------------------------------
# parallel sampling with shared prompts
# --------------------------------------------------------------------------

@dataclass
class CowWorkload:
    shape: Shape
    prompt_lens: np.ndarray           # int32 [P]
    branches: int
    steps: int
    num_blocks: int
    free_order: np.ndarray            # int32 [num_blocks]
    prompt_k: torch.Tensor            # [sum(prompt_lens), Hkv, D] in prompt order
    prompt_v: torch.Tensor
    seed: int
    device: str = "cpu"

    @property
    def num_seqs(self) -> int:
        return int(len(self.prompt_lens) * self.branches)

    def seq_id(self, prompt: int, branch: int) -> int:
        return prompt * self.branches + branch

    def step_inputs(self, step: int):
        """(q [S, Hq, D], k_new [S, Hkv, D], v_new [S, Hkv, D]) for one decode
        step, sequences ordered by seq id (prompt-major, branch-minor)."""
        sh = self.shape
        g = torch.Generator(device=self.device)
        g.manual_seed(int(self.seed) * 1_000_003 + 7919 * (step + 1))
        dt = TORCH_DTYPES[sh.dtype]
        S = self.num_seqs

        def draw(*dims):
            return torch.randn(*dims, generator=g, device=self.device,
                               dtype=torch.float32).to(dt)

        q = draw(S, sh.num_q_heads, sh.head_dim)
        k = draw(S, sh.num_kv_heads, sh.head_dim)
        v = draw(S, sh.num_kv_heads, sh.head_dim)
        return q, k, v


def cow_workload(device="cpu", num_prompts: int = 32, branches: int = 8, steps: int = 64,
                 prompt_range=(64, 512), shape: Shape | None = None,
                 seed: int | None = None) -> CowWorkload:
    sh = shape if shape is not None else SHAPES["cow"]
    seed = SEEDS["cow"] if seed is None else seed
    rng = np.random.default_rng(seed)
    plens = rng.integers(prompt_range[0], prompt_range[1], size=num_prompts,
                         endpoint=True).astype(np.int32)
    B = sh.block_size
    prompt_blocks = sum(_ceil_div(int(p), B) for p in plens)
    # every branch can grow by ceil(steps/B)+1 blocks, plus one private copy each
    growth = num_prompts * branches * (_ceil_div(steps, B) + 2)
    num_blocks = int(math.ceil((prompt_blocks + growth) * 1.1))
    perm = rng.permutation(num_blocks).astype(np.int32)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    dt = TORCH_DTYPES[sh.dtype]
    total = int(plens.sum())
    pk = torch.randn(total, sh.num_kv_heads, sh.head_dim, generator=g, device=device,
                     dtype=torch.float32).to(dt)
    pv = torch.randn(total, sh.num_kv_heads, sh.head_dim, generator=g, device=device,
                     dtype=torch.float32).to(dt)
    return CowWorkload(shape=sh, prompt_lens=plens, branches=branches, steps=steps,
                       num_blocks=num_blocks, free_order=perm, prompt_k=pk, prompt_v=pv,
                       seed=seed, device=device)


def empty_pool(shape: Shape, num_blocks: int, seed: int, device="cpu"):
    """A K and V pool filled with random stale values (what a fresh pool holds
    before any token is written)."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) + 12345)
    dt = TORCH_DTYPES[shape.dtype]
    dims = (num_blocks, shape.num_kv_heads, shape.block_size, shape.head_dim)
    k = torch.randn(*dims, generator=g, device=device, dtype=torch.float32).to(dt)
    v = torch.randn(*dims, generator=g, device=device, dtype=torch.float32).to(dt)
    return k, v


# --------------------------------------------------------------------------
# requests sharing prompt prefixes (for prefix caching across requests)
# --------------------------------------------------------------------------
@dataclass
class PrefixWorkload:
    shape: Shape
    requests: list                    # token ids (np.int32 arrays), in arrival order
    events: list                      # ("alloc", i) / ("free", i), in order
    num_blocks: int
    free_order: np.ndarray            # int32 [num_blocks]
    seed: int


def prefix_workload(shape: Shape | None = None, num_requests: int = 48, num_system: int = 4,
                    system_range=(20, 300), suffix_range=(1, 120), vocab: int = 32000,
                    live: int = 12, repeat_fraction: float = 0.25, seed: int = 7,
                    num_blocks: int | None = None) -> PrefixWorkload:
    """Chat-like requests: each is one of a few system prompts (drawn with
    skewed weights) followed by its own suffix, or, with probability
    ``repeat_fraction``, an earlier request followed by a new turn.  At most
    ``live`` requests are held at once: before a request arrives a random live
    one finishes when the limit is reached.  The default pool holds about
    1.5 times the live requests' blocks, so freed blocks are reused and
    retained prefixes are eventually handed out again."""
    sh = shape if shape is not None else SHAPES["gqa8b"]
    rng = np.random.default_rng(seed)
    systems = [rng.integers(0, vocab, size=int(rng.integers(system_range[0], system_range[1],
                                                            endpoint=True))).astype(np.int32)
               for _ in range(num_system)]
    weights = rng.dirichlet(np.full(num_system, 0.7))
    requests, events, alive = [], [], []
    for i in range(num_requests):
        suffix = rng.integers(0, vocab, size=int(rng.integers(suffix_range[0], suffix_range[1],
                                                              endpoint=True))).astype(np.int32)
        if requests and rng.random() < repeat_fraction:
            base = requests[int(rng.integers(0, len(requests)))]
        else:
            base = systems[int(rng.choice(num_system, p=weights))]
        requests.append(np.concatenate([base, suffix]).astype(np.int32))
        if len(alive) >= live:
            j = alive.pop(int(rng.integers(0, len(alive))))
            events.append(("free", j))
        events.append(("alloc", i))
        alive.append(i)
    B = sh.block_size
    if num_blocks is None:
        biggest = sorted((_ceil_div(len(r), B) for r in requests), reverse=True)[:live]
        num_blocks = int(math.ceil(1.5 * sum(biggest))) + live * 4
    perm = rng.permutation(num_blocks).astype(np.int32)
    return PrefixWorkload(shape=sh, requests=requests, events=events, num_blocks=num_blocks,
                          free_order=perm, seed=seed)


def prefix_kv_rows(tokens, shape: Shape, seed: int, device="cpu"):
    """Synthetic K and V rows [n, Hkv, D] for a prompt, row t a function of
    (seed, tokens[0..t]) only -- as a model's K/V at a position depend on the
    whole prefix -- so requests with equal prefixes get bit-equal rows.  Row t
    is N(0, 1) drawn by a PCG64 generator seeded with (seed, running CRC-32 of
    the prefix), rounded to nearest-even into the storage dtype."""
    import zlib
    dims = (shape.num_kv_heads, shape.head_dim)
    n = len(tokens)
    k = np.empty((n,) + dims, dtype=np.float32)
    v = np.empty((n,) + dims, dtype=np.float32)
    crc = 0
    for t, tok in enumerate(np.asarray(tokens, dtype=np.int32).tolist()):
        crc = zlib.crc32(np.int32(tok).tobytes(), crc)
        g = np.random.default_rng([int(seed), crc])
        k[t] = g.standard_normal(dims, dtype=np.float32)
        v[t] = g.standard_normal(dims, dtype=np.float32)
    dt = TORCH_DTYPES[shape.dtype]
    return torch.from_numpy(k).to(dt).to(device), torch.from_numpy(v).to(dt).to(device)


# --------------------------------------------------------------------------
# chunked prefill: several new tokens per sequence
# --------------------------------------------------------------------------
@dataclass
class PrefillBatch:
    shape: Shape
    context_lens: np.ndarray          # int32 [S], tokens after this chunk
    chunk_lens: np.ndarray            # int32 [S], new tokens this step (<= context_lens)
    query_start: np.ndarray           # int32 [S+1], running sum of chunk_lens
    block_tables: np.ndarray          # int32 [S, max_blocks_per_seq], -1 = unused
    free_order: np.ndarray            # int32 [num_blocks]
    num_blocks: int
    q: torch.Tensor                   # [T, Hq, D], T = sum(chunk_lens)
    k_cache: torch.Tensor             # [num_blocks, Hkv, B, D]
    v_cache: torch.Tensor
    k_new: torch.Tensor               # [T, Hkv, D] the chunk's tokens
    v_new: torch.Tensor
    scale: float

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_tokens(self) -> int:
        return int(self.query_start[-1])


def make_prefill_batch(shape: Shape, context_lens, chunk_lens, seed: int, *, device="cpu",
                       spare_fraction: float = 0.10, max_blocks_per_seq: int | None = None,
                       poison: str | None = None) -> PrefillBatch:
    """Draw one chunked-prefill batch.  Sequence s already holds
    context_lens[s] - chunk_lens[s] tokens and adds chunk_lens[s] this step.
    Blocks are consecutive runs of one permutation, sequence by sequence, as
    a first-in-first-out manager seeded with ``free_order`` hands them out
    when each sequence is allocated and then extended by its chunk before the
    next one.  Draw order: permutation (numpy), then q, K pool, V pool, new K,
    new V (torch generator), N(0, 1) rounded into the storage dtype;
    ``poison='nan'`` as for decode batches."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(context_lens, dtype=np.int32)
    chunks = np.asarray(chunk_lens, dtype=np.int32)
    assert lens.shape == chunks.shape and (chunks >= 0).all() and (chunks <= lens).all()
    B = shape.block_size
    nb = [_ceil_div(int(x), B) for x in lens]
    used = int(sum(nb))
    num_blocks = max(1, int(math.ceil(used * (1.0 + spare_fraction))))
    maxb = max_blocks_per_seq if max_blocks_per_seq is not None else max(1, max(nb, default=1))
    perm = rng.permutation(num_blocks).astype(np.int32)
    tables = np.full((len(lens), maxb), -1, dtype=np.int32)
    off = 0
    for s, n in enumerate(nb):
        tables[s, :n] = perm[off:off + n]
        off += n
    qstart = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    T = int(qstart[-1])
    dt = TORCH_DTYPES[shape.dtype]
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    Hq, Hkv, D = shape.num_q_heads, shape.num_kv_heads, shape.head_dim

    def draw(*dims):
        return torch.randn(*dims, generator=g, device=device, dtype=torch.float32).to(dt)

    q = draw(T, Hq, D)
    k_cache = draw(num_blocks, Hkv, B, D)
    v_cache = draw(num_blocks, Hkv, B, D)
    k_new = draw(T, Hkv, D)
    v_new = draw(T, Hkv, D)
    if poison == "nan":
        valid = torch.zeros(num_blocks, B, dtype=torch.bool)
        for s, n in enumerate(nb):
            for j in range(n):
                valid[int(tables[s, j]), :min(B, int(lens[s]) - j * B)] = True
        mask = (~valid).to(device)[:, None, :, None].expand(num_blocks, Hkv, B, D)
        nan = torch.tensor(NAN_BITS[shape.dtype], dtype=torch.int16, device=device).view(dt)
        k_cache[mask] = nan
        v_cache[mask] = nan
    elif poison is not None:
        raise ValueError(poison)
    return PrefillBatch(shape=shape, context_lens=lens, chunk_lens=chunks, query_start=qstart,
                        block_tables=tables, free_order=perm, num_blocks=num_blocks, q=q,
                        k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
                        scale=1.0 / math.sqrt(D))


def prefill_lens(rng: np.random.Generator, num_seqs: int = 16, chunk: int = 512,
                 max_len: int = 4096):
    """Chunked-prefill mix: every sequence adds a chunk of ``chunk`` tokens on
    top of 0 .. max_len - chunk tokens already cached (uniform, in whole
    chunks, as a long prompt processed chunk by chunk)."""
    before = chunk * rng.integers(0, max_len // chunk, size=num_seqs)
    chunks = np.full(num_seqs, chunk, dtype=np.int32)
    return (before + chunks).astype(np.int32), chunks
