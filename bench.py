"""Benchmark of the paged decode hot path on B200.

One step = one decode step of one attention layer over a batch of sequences:
the host block manager reserves every sequence's next slot (copy-on-write
pairs if any -> copy_blocks), reshape_and_cache writes the new K/V, and
paged decode attention (+ the split-context merge) reads every cached token
of every sequence through the block tables.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gqa8b]
    python bench.py --impl reference ...     # the CPU oracle, timed on host cores
    python bench.py --workload prefill       # chunked prefill (tensor cores), TFLOP/s
    python bench.py --report kv              # paged vs contiguous KV memory (no GPU needed)

Prints one JSON line (rank 0).  `value` is the decode attention's algorithmic
HBM bytes (every K/V element of every cached token read once, plus the block
table entries used) divided by the device-timed step; `e2e` is the same
metric through the public API from pinned host buffers, with the block
manager, the host->device copy of the step's inputs and the device->host copy
of its output inside the timed region.  Inputs are larger than L2, so no L2
flush is needed between steps.  Data are synthetic (seeded, see workloads.py).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

WORKLOADS = {
    "gqa8b": "GQA 8B-class paged decode: 256 seqs, 32 q / 8 kv heads, head_dim 128, block 16, "
             "bf16 KV, lognormal context lengths (median 512, clip 16..4096), shuffled blocks",
    "13b": "13B-class paged decode: 64 seqs, 40 q = 40 kv heads, head_dim 128, block 16, fp16 KV, "
           "context lengths uniform 1..2048, shuffled blocks",
    "long": "long-context paged decode: 8 seqs, 64 q / 8 kv heads, head_dim 128, block 16, bf16, "
            "context lengths uniform 16384..32768, peaked softmax",
    "long32": "long-context paged decode, block 32",
    "cow": "parallel sampling with copy-on-write: 32 prompts (64..512 tokens) x 8 branches sharing "
           "the prompt blocks, 32 q / 8 kv heads, head_dim 128, block 16, bf16; the timed steps "
           "start at the first append (copy_blocks of every shared partial last block)",
    "prefill": "chunked prefill: 16 seqs, 512-token chunks on 0..3584 cached tokens, 32 q / 8 kv "
               "heads, head_dim 128, block 16, bf16 KV, shuffled blocks",
}
PREFILL_METRIC = "chunked prefill attention achieved TFLOP/s (% of measured bf16 tensor peak)"
METRIC = "paged decode attention achieved HBM GB/s (% of B200 peak); decode tokens/s"
# committed ncu summaries of the decode kernel, per workload
PROFILE_SUMMARIES = {w: os.path.join(ROOT, "profiles", f"decode_attention_{w}.md")
                     for w in ("gqa8b", "13b")}
# sources that decide a kernel's DRAM traffic: the kernel itself and the host
# code that picks its launch shape (grid, CTAs per SM, stages, scratch layout)
KERNEL_SOURCES = ["paged_kv_cache_414_b200/csrc/decode_attention.cuh",
                  "paged_kv_cache_414_b200/csrc/pa_device.cuh",
                  "paged_kv_cache_414_b200/csrc/pa_kernels.cu"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gqa8b", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--report", choices=["kv"], default=None,
                    help="print the KV memory report (paged vs contiguous) instead of timing")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers

PREFILL_PROFILE = os.path.join(ROOT, "profiles", "prefill_attention_16x512.md")
PREFILL_SOURCES = ["paged_kv_cache_414_b200/csrc/prefill_attention.cuh",
                   "paged_kv_cache_414_b200/csrc/umma.cuh",
                   "paged_kv_cache_414_b200/csrc/pa_device.cuh",
                   "paged_kv_cache_414_b200/csrc/prefill_launch.cuh"]


def kernel_source_sha(sources=None) -> str:
    h = hashlib.sha256()
    for f in (KERNEL_SOURCES if sources is None else sources):
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(bytes_per_launch: float, workload: str = "gqa8b"):
    """DRAM bytes (read + write) per launch from the workload's committed ncu
    summary, scaled from the profiled launch to this run's launches by
    algorithmic bytes; None without a summary for the workload or unless it
    was taken on the current kernel source."""
    try:
        text = open(PROFILE_SUMMARIES[workload]).read()
    except (KeyError, OSError):
        return None
    m_sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"dram_bytes_per_launch_full_workload:\s*([0-9.eE+]+)", text)
    m_alg = re.search(r"algorithmic_bytes_of_profiled_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_tr or not m_alg or m_sha.group(1) != kernel_source_sha():
        return None
    return round(float(m_tr.group(1)) * bytes_per_launch / float(m_alg.group(1)))


def prefill_profiled_traffic():
    """DRAM bytes (read + write) of one prefill launch of the bench workload
    from the committed ncu summary; None unless it was taken on the current
    kernel source."""
    try:
        text = open(PREFILL_PROFILE).read()
    except OSError:
        return None
    m_sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"dram_bytes_per_launch_full_workload:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_tr or m_sha.group(1) != kernel_source_sha(PREFILL_SOURCES):
        return None
    return int(float(m_tr.group(1)))


def measured_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_cores_used() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = max([int(x.get("num_threads", 1)) for x in threadpool_info()] + [1])
        return n
    except Exception:
        return os.cpu_count() or 1


def rank_reduce(x: float, op: str, world: int, device=None) -> float:
    """Max or sum of a scalar over all ranks (identity on one rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def decode_bytes(context_lens, num_kv_heads: int, head_dim: int, block_size: int,
                 elem_bytes: int = 2) -> int:
    """Algorithmic HBM bytes of one decode-attention call: every cached K and V
    element of every sequence read once, plus the block-table entries used."""
    total = 0
    for L in np.asarray(context_lens).tolist():
        L = int(L)
        total += 2 * L * num_kv_heads * head_dim * elem_bytes + 4 * math.ceil(L / block_size)
    return total


def prefill_flops(context_lens, chunk_lens, num_q_heads: int, head_dim: int) -> int:
    """Algorithmic FLOPs of one chunked-prefill attention call: a chunk token
    at position p costs 2*head_dim*(p+1) for its scores and as much for P.V,
    per query head; positions run L-C .. L-1, so a sequence contributes
    4*D*Hq * C*(2L - C + 1)/2."""
    total = 0
    for L, C in zip(np.asarray(context_lens).tolist(), np.asarray(chunk_lens).tolist()):
        total += 4 * head_dim * num_q_heads * (int(C) * (2 * int(L) - int(C) + 1) // 2)
    return total


def rank_seed(name: str, rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling)."""
    return W.SEEDS[name] + 1000 * rank


# ----------------------------------------------------------------------------- workload

class Workload:
    """A decode batch plus K+W steps of block-manager output prepared ahead."""

    def __init__(self, name: str, device, seed_offset: int, steps_total: int):
        import torch
        self.name = name
        self.cyclic = False
        self.steps_total = steps_total   # the block tables are sized for this many steps
        if name == "cow":
            self._init_cow(device, seed_offset, steps_total)
            return
        sh = W.SHAPES[name]
        self.shape = sh
        seed = rank_seed(name, seed_offset)
        rng = np.random.default_rng(seed)
        lens = {"gqa8b": W.lens_gqa8b, "13b": W.lens_13b}.get(name, W.lens_long)(rng)
        B = sh.block_size
        grow = math.ceil(steps_total / B) + 1
        need = sum(math.ceil(int(L) / B) + grow for L in lens)
        maxb = max(math.ceil((int(L) + steps_total) / B) for L in lens)
        self.batch = W.make_decode_batch(sh, lens, seed,
                                         device=device, num_blocks=int(need * 1.1),
                                         max_blocks_per_seq=maxb, rng=rng)
        self.lens0 = lens.astype(np.int64)
        self.maxb = maxb
        self.S = len(lens)
        self.device = device
        self.scale = 1.0 / math.sqrt(sh.head_dim)
        self.elem = 2

    def _init_cow(self, device, seed_offset: int, steps_total: int):
        """32 prompts forked into 8 branches each; the prompts' K/V are written
        into the pool when the first manager is built.  The step inputs are
        one seeded draw reused every step (the bytes moved are the same)."""
        from types import SimpleNamespace
        sh = W.SHAPES["cow"]
        self.shape = sh
        self.cyclic = True          # timed steps replay steps 0.. (copy-on-write first)
        seed = rank_seed("cow", seed_offset)
        cw = W.cow_workload(device=device, steps=steps_total, seed=seed)
        self.cw = cw
        B = sh.block_size
        k_cache, v_cache = W.empty_pool(sh, cw.num_blocks, seed, device=device)
        q, k_new, v_new = cw.step_inputs(0)
        self.batch = SimpleNamespace(k_cache=k_cache, v_cache=v_cache, q=q, k_new=k_new,
                                     v_new=v_new, num_blocks=cw.num_blocks,
                                     free_order=cw.free_order)
        # context after step 0's append: the prompt plus the branch's first token
        self.lens0 = np.repeat(cw.prompt_lens.astype(np.int64) + 1, cw.branches)
        self.maxb = max(math.ceil((int(P) + steps_total) / B) for P in cw.prompt_lens)
        self.S = cw.num_seqs
        self.device = device
        self.scale = 1.0 / math.sqrt(sh.head_dim)
        self.elem = 2
        self._prompts_written = False

    def bytes_per_step(self, step: int) -> int:
        """Algorithmic (logical) bytes: every cached token of every sequence;
        for shared prompt blocks that is once per branch reading them."""
        return decode_bytes(self.lens0 + step, self.shape.num_kv_heads, self.shape.head_dim,
                            self.shape.block_size, self.elem)

    def new_manager(self, pa):
        """A native manager in the state before step 0 (for the cow workload the
        prompts are allocated and forked, and their K/V written the first time)."""
        bm = pa.BlockManager(self.batch.num_blocks, self.shape.block_size, self.batch.free_order)
        if self.name != "cow":
            for s in range(self.S):
                bm.allocate(s, int(self.lens0[s]) - 1)
            return bm
        import torch
        cw = self.cw
        slots = []
        for pr, P in enumerate(cw.prompt_lens):
            slots.append(bm.allocate(cw.seq_id(pr, 0), int(P)))
            for br in range(1, cw.branches):
                bm.fork(cw.seq_id(pr, 0), cw.seq_id(pr, br))
        if not self._prompts_written:
            pa.pa_reshape_and_cache(cw.prompt_k, cw.prompt_v, self.batch.k_cache,
                                    self.batch.v_cache,
                                    torch.as_tensor(np.concatenate(slots), device=self.device))
            self._prompts_written = True
        return bm

    def oracle_manager(self, step: int):
        """The oracle's manager after `step` steps, and the slots of step `step`."""
        from oracle.block_manager import BlockManager as OracleBM
        bm = OracleBM(self.batch.num_blocks, self.shape.block_size, self.batch.free_order)
        if self.name != "cow":
            for s in range(self.S):
                bm.allocate(s, int(self.lens0[s]) - 1 + step)
        else:
            cw = self.cw
            for pr, P in enumerate(cw.prompt_lens):
                bm.allocate(cw.seq_id(pr, 0), int(P))
                for br in range(1, cw.branches):
                    bm.fork(cw.seq_id(pr, 0), cw.seq_id(pr, br))
            for _ in range(step):
                for s in range(self.S):
                    bm.append_slot(s)
        return bm, [bm.append_slot(s)[0] for s in range(self.S)]


def decode_config(wl, name: str, world: int, K: int, Wm: int) -> dict:
    """The `config` of a decode line; both arms print the same one."""
    sh = wl.shape
    timed = (lambda k: k) if wl.cyclic else (lambda k: Wm + k)  # noqa: E731
    b = wl.batch
    pool_bytes = 2 * b.k_cache.numel() * b.k_cache.element_size()
    flush = pool_bytes < 2 * 126 * 2 ** 20
    bytes_launch = float(np.mean([wl.bytes_per_step(timed(k)) for k in range(K)]))
    return {
        "workload": f"{name}: {WORKLOADS[name]}",
        "num_seqs_per_gpu": wl.S,
        "num_q_heads": sh.num_q_heads,
        "num_kv_heads": sh.num_kv_heads,
        "head_dim": sh.head_dim,
        "block_size": sh.block_size,
        "mean_context_len": float(np.mean(wl.lens0)) + float(np.mean([timed(k) for k in range(K)])),
        "bytes_per_step": bytes_launch,
        "parallelism": f"dp{world} (independent batches, no collective on the data path)",
        "l2": ("K/V pool %.0f MB, under twice L2: L2 flushed (256 MB memset) before "
               "every timed step, outside the per-step CUDA-event spans" % (pool_bytes / 1e6)
               if flush else "inputs larger than L2: %.2f GB of KV read per step, no flush"
               % (bytes_launch / 1e9)),
        "step": "host block manager (prepared ahead) -> copy_blocks if any -> pa_decode_step "
                "(cache write of the new token + paged decode attention) -> split merge",
    }


# ----------------------------------------------------------------------------- our arm

def run_b200(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from paged_kv_cache_414_b200 import build as pbuild
    pbuild.build()
    import paged_kv_cache_414_b200 as pa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    K, Wm = args.steps, args.warmup
    wl = Workload(args.workload, dev, rank, K + Wm + 1)
    sh = wl.shape
    B = sh.block_size
    S = wl.S
    b = wl.batch
    stream = torch.cuda.current_stream()

    # block manager output for every step, prepared ahead (device-resident arm)
    bm = wl.new_manager(pa)
    seqs = np.arange(S)
    d_tables, d_lens, d_pairs = [], [], []
    # step indices: warm-up steps, then the timed ones; a cyclic workload
    # (copy-on-write) times steps 0.. again after its warm-up, so that the
    # timed region starts with the copies of the first append
    nprep = K if wl.cyclic else K + Wm
    warm_idx = (lambda i: i % K) if wl.cyclic else (lambda i: i)   # noqa: E731
    timed_idx = (lambda k: k) if wl.cyclic else (lambda k: Wm + k)  # noqa: E731
    for step in range(nprep):
        slots, pairs = bm.append_slots(seqs)
        tables, lens = bm.block_tables(seqs, wl.maxb)

        d_tables.append(torch.as_tensor(tables, device=dev))
        d_lens.append(torch.as_tensor(lens, device=dev))
        d_pairs.append(torch.as_tensor(pairs, device=dev) if len(pairs) else None)
    bm.close()
    maxctx = wl.maxb * B
    ws = pa.alloc_workspace(S, sh.num_q_heads, sh.num_kv_heads, sh.head_dim, B, maxctx, dev)
    out = torch.empty(S, sh.num_q_heads, sh.head_dim, dtype=torch.float32, device=dev)
    # kernels launched per timed step: the fused decode step and its split
    # merge, plus copy_blocks on steps with copy-on-write pairs
    timed_launches = sum(2 + (d_pairs[timed_idx(k)] is not None) for k in range(K))
    # a pool smaller than twice L2 is flushed (a 256 MB memset) before every
    # timed step, outside per-step CUDA-event spans that then make the time
    pool_bytes = 2 * b.k_cache.numel() * b.k_cache.element_size()
    flush = pool_bytes < 2 * 126 * 2 ** 20
    flush_buf = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev) if flush else None
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]

    # Per-call events only when a step has other kernels (copy-on-write
    # copies) to separate from the decode call: an event recorded between two
    # launches ends the programmatic overlap of the second with the first.
    # Otherwise the decode call is the whole step and its average duration is
    # the timed region over K (launch gaps included, so never optimistic).
    per_call_events = flush or any(d_pairs[timed_idx(k)] is not None for k in range(K))
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(K)]

    def step(i, timed_idx=None):
        if d_pairs[i] is not None:
            pa.pa_copy_blocks(b.k_cache, b.v_cache, d_pairs[i])
        if timed_idx is not None and per_call_events:
            ev_a[timed_idx].record(stream)
        # fused: the newest token's cache write + decode attention (+ split merge)
        pa.pa_decode_step(out, b.q, b.k_new, b.v_new, b.k_cache, b.v_cache, d_tables[i],
                          d_lens[i], wl.scale, sh.num_kv_heads, max_context_len=maxctx,
                          workspace=ws)
        if timed_idx is not None and per_call_events:
            ev_b[timed_idx].record(stream)

    for i in range(Wm):
        step(warm_idx(i))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" in os.environ
                          else local_rank)
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0.record(stream)
    for k in range(K):
        if flush:
            flush_buf.zero_()
            ev_s[k].record(stream)
        step(timed_idx(k), k)
        if flush:
            ev_e[k].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    flags = pa.pa_device_error()
    ms_total = t0.elapsed_time(t1)
    if flush:   # the steps alone, without the flushes between them
        ms_total = float(sum(ev_s[k].elapsed_time(ev_e[k]) for k in range(K)))
    if per_call_events:
        attn_ms = [ev_a[k].elapsed_time(ev_b[k]) for k in range(K)]
    else:
        attn_ms = [ms_total / K] * K
    bytes_steps = [wl.bytes_per_step(timed_idx(k)) for k in range(K)]
    my_bytes = float(sum(bytes_steps))

    reduce_max = lambda x: rank_reduce(x, "max", world, dev)   # noqa: E731
    reduce_sum = lambda x: rank_reduce(x, "sum", world, dev)   # noqa: E731

    ms_max = reduce_max(ms_total)
    all_bytes = reduce_sum(my_bytes)
    value = all_bytes / (ms_max * 1e-3) / 1e9
    tokens_per_s = reduce_sum(float(S * K)) / (ms_max * 1e-3)

    # roofline of the decode attention call (attention + merge kernels)
    attn_avg_ms = float(np.mean(attn_ms))
    bytes_launch = float(np.mean(bytes_steps))
    achieved = bytes_launch / (attn_avg_ms * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    # from the committed ncu summary of this workload's launch, if there is
    # one (the others run other kernel instances or, with shared prefixes,
    # other DRAM/L2 splits)
    traffic = profiled_traffic(bytes_launch, args.workload)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(pa, wl, K, Wm, dev, world, reduce_max, reduce_sum)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": Wm,
            "ms_per_step": round(ms_max / K, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": sh.dtype,
            "data": "synthetic",
            "config": decode_config(wl, args.workload, world, K, Wm),
            "pct_of_measured_hbm_peak": round(100.0 * value / peak / world, 2),
            "pct_of_nominal_8tbs": round(100.0 * value / 8000.0 / world, 2),
            "decode_tokens_per_s": round(tokens_per_s, 1),
            "roofline": {
                "bound": "hbm",
                "kernel": "pa_decode_step (paged_decode_kernel with the newest token's cache write, + paged_decode_merge_kernel)",
                "achieved": round(achieved, 2),
                "peak": peak,
                "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback 6650 GB/s",
                "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": traffic,
                "bytes_per_launch": bytes_launch,
                "avg_launch_ms": round(attn_avg_ms, 5),
                "launch_timing": ("CUDA events around every call" if per_call_events else
                                  "the call is the whole step: timed region (CUDA events) / steps"),
            },
            "e2e": e2e,
            "cpu_baseline": cpu,
            "gpu_launches": timed_launches,
            "device_error_flags": flags,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)


def run_e2e(pa, wl, K, Wm, dev, world, reduce_max, reduce_sum):
    """Same metric through the public API from pinned host buffers: per step,
    the host block manager reserves the slots and writes the block tables
    straight into pinned memory, the step's inputs (q, new K/V, lengths,
    block tables, copy-on-write pairs) go host -> device as one packed copy,
    the library's kernels run, and the output comes back device -> host.
    Three streams (upload, compute, download) and three buffer sets let step
    i+1's upload and step i-1's download overlap step i's kernels; events
    order every reuse."""
    import torch
    import torch.distributed as dist
    sh = wl.shape
    S, B = wl.S, sh.block_size
    b = wl.batch
    seqs = np.arange(S)
    bm = wl.new_manager(pa)
    NBUF = 3

    # packed input layout: q | k_new | v_new | lens | tables | pairs (256-byte aligned)
    def al(n):
        return (n + 255) // 256 * 256
    parts = [("q", b.q.dtype, (S, sh.num_q_heads, sh.head_dim), 2),
             ("k", b.k_new.dtype, (S, sh.num_kv_heads, sh.head_dim), 2),
             ("v", b.v_new.dtype, (S, sh.num_kv_heads, sh.head_dim), 2),
             ("lens", torch.int32, (S,), 4),
             ("tables", torch.int32, (S, wl.maxb), 4),
             ("pairs", torch.int64, (S, 2), 8)]
    off, pos = {}, 0
    for name, _, shape, es in parts:
        off[name] = pos
        pos += al(int(np.prod(shape)) * es)
    total = pos

    def views(buf):
        v = {}
        for name, dt, shape, es in parts:
            n = int(np.prod(shape)) * es
            v[name] = buf[off[name]:off[name] + n].view(dt).view(shape)
        return v

    h_buf = [torch.empty(total, dtype=torch.uint8).pin_memory() for _ in range(NBUF)]
    d_buf = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(NBUF)]
    h_in = [views(x) for x in h_buf]
    d_in = [views(x) for x in d_buf]
    h_slots = [np.empty(S, dtype=np.int64) for _ in range(NBUF)]
    for hv in h_in:
        hv["q"].copy_(b.q.cpu())
        hv["k"].copy_(b.k_new.cpu())
        hv["v"].copy_(b.v_new.cpu())
    h_out = [torch.empty(S, sh.num_q_heads, sh.head_dim, dtype=torch.float32).pin_memory()
             for _ in range(NBUF)]
    d_out = [torch.empty(S, sh.num_q_heads, sh.head_dim, dtype=torch.float32, device=dev)
             for _ in range(NBUF)]
    maxctx = wl.maxb * B
    ws = pa.alloc_workspace(S, sh.num_q_heads, sh.num_kv_heads, sh.head_dim, B, maxctx, dev)
    s_up, s_cmp, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(NBUF)]    # upload of the set done
    ev_cmp = [torch.cuda.Event() for _ in range(NBUF)]   # kernels reading / writing the set done
    ev_dn = [torch.cuda.Event() for _ in range(NBUF)]    # download of the set's output done
    used = [False] * NBUF
    in_bytes = off["pairs"]                      # everything up to the (optional) pairs
    h2d_steps, d2h = [], h_out[0].numel() * 4

    def one(i):
        j = i % NBUF
        hv, dv = h_in[j], d_in[j]
        if used[j]:
            ev_up[j].synchronize()             # host buffers of set j are free again
        _, pairs = bm.append_slots(seqs, slots_out=h_slots[j], pairs_out=hv["pairs"])
        bm.block_tables(seqs, wl.maxb, out=hv["tables"], lens_out=hv["lens"])
        npairs = len(pairs)
        nbytes = in_bytes + npairs * 16
        h2d_steps.append(nbytes)
        with torch.cuda.stream(s_up):
            if used[j]:
                s_up.wait_event(ev_cmp[j])     # device inputs of set j no longer read
            d_buf[j][:nbytes].copy_(h_buf[j][:nbytes], non_blocking=True)
            ev_up[j].record(s_up)
        s_cmp.wait_event(ev_up[j])
        if used[j]:
            s_cmp.wait_event(ev_dn[j])         # output of set j downloaded
        if npairs:
            pa.pa_copy_blocks(b.k_cache, b.v_cache, dv["pairs"][:npairs], stream=s_cmp)
        pa.pa_decode_step(d_out[j], dv["q"], dv["k"], dv["v"], b.k_cache, b.v_cache,
                          dv["tables"], dv["lens"], wl.scale, sh.num_kv_heads,
                          max_context_len=maxctx, workspace=ws, stream=s_cmp)
        ev_cmp[j].record(s_cmp)
        with torch.cuda.stream(s_dn):
            s_dn.wait_event(ev_cmp[j])
            h_out[j].copy_(d_out[j], non_blocking=True)
            ev_dn[j].record(s_dn)
        used[j] = True

    for i in range(Wm):
        one(i)
    torch.cuda.synchronize()
    h2d_steps.clear()
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for i in range(Wm, Wm + K):
        one(i)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    bm.close()
    dt_max = reduce_max(dt)
    bytes_all = reduce_sum(float(sum(wl.bytes_per_step(i) for i in range(Wm, Wm + K))))
    return {"value": round(bytes_all / dt_max / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(round(sum(h2d_steps) / max(len(h2d_steps), 1))),
            "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(dt_max * 1e3 / K, 4),
            "timing": "host wall clock, synchronize on both sides, max over ranks; "
                      "upload (one packed copy) / compute / download on three streams, "
                      "three buffer sets"}


# ----------------------------------------------------------------------------- chunked prefill

class PrefillBench:
    """The chunked-prefill batch (16 sequences, 512-token chunks on top of
    0..3584 cached tokens, GQA 8B heads, bf16) with the block manager's
    output for it: each sequence's earlier context allocated, then its chunk
    appended token by token."""

    def __init__(self, pa, device, rank: int):
        self.shape = W.SHAPES["gqa8b"]
        seed = W.SEEDS["gqa8b"] + 100 + 1000 * rank
        lens, chunks = W.prefill_lens(np.random.default_rng(seed))
        self.batch = W.make_prefill_batch(self.shape, lens, chunks, seed, device=device)
        b = self.batch
        bm = pa.BlockManager(b.num_blocks, self.shape.block_size, b.free_order)
        slots = []
        for s in range(b.num_seqs):
            L, C = int(lens[s]), int(chunks[s])
            bm.allocate(s, L - C)
            sl, _ = bm.append_slots([s] * C)
            slots.append(sl)
        tables, ctx = bm.block_tables(np.arange(b.num_seqs), b.block_tables.shape[1])
        bm.close()
        assert np.array_equal(tables, b.block_tables) and np.array_equal(ctx, b.context_lens)
        self.slots = np.concatenate(slots).astype(np.int64)
        self.flops = prefill_flops(lens, chunks, self.shape.num_q_heads, self.shape.head_dim)
        self.max_query_len = int(chunks.max())


def prefill_config(pb, world: int) -> dict:
    """The `config` of a prefill line; both arms print the same one."""
    b, sh = pb.batch, pb.shape
    return {
        "workload": f"prefill: {WORKLOADS['prefill']}",
        "num_seqs_per_gpu": b.num_seqs,
        "num_tokens_per_step": b.num_tokens,
        "num_q_heads": sh.num_q_heads,
        "num_kv_heads": sh.num_kv_heads,
        "head_dim": sh.head_dim,
        "block_size": sh.block_size,
        "mean_context_len": float(np.mean(b.context_lens)),
        "flops_per_step": pb.flops,
        "parallelism": f"dp{world} (independent batches, no collective on the data path)",
        "l2": "inputs larger than L2 (%.0f MB of K/V pool, %.0f MB of q, %.0f MB of "
              "output per step), no flush" % (
                  2 * b.k_cache.numel() * 2 / 1e6, b.q.numel() * 2 / 1e6,
                  b.num_tokens * sh.num_q_heads * sh.head_dim * 4 / 1e6),
        "step": "reshape_and_cache of the chunk (slots prepared ahead by the host block "
                "manager) -> pa_paged_prefill_attention",
    }


def run_prefill_b200(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from paged_kv_cache_414_b200 import build as pbuild
    pbuild.build()
    import paged_kv_cache_414_b200 as pa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    K, Wm = args.steps, args.warmup
    pb = PrefillBench(pa, dev, rank)
    b, sh = pb.batch, pb.shape
    T = b.num_tokens
    d_slots = torch.as_tensor(pb.slots, device=dev)
    d_tables = torch.as_tensor(b.block_tables, device=dev)
    d_lens = torch.as_tensor(b.context_lens, device=dev)
    d_qs = torch.as_tensor(b.query_start, device=dev)
    out = torch.empty(T, sh.num_q_heads, sh.head_dim, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(K)]

    def step(k=None):
        # the chunk's cache write, then its attention over the paged context
        pa.pa_reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache, d_slots)
        if k is not None:
            ev_a[k].record(stream)
        pa.pa_paged_prefill_attention(out, b.q, b.k_cache, b.v_cache, d_tables, d_lens, d_qs,
                                      b.scale, sh.num_kv_heads, pb.max_query_len)
        if k is not None:
            ev_b[k].record(stream)

    for _ in range(Wm):
        step()
    torch.cuda.synchronize()
    pa.pa_device_error(clear=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(K):
        step(k)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    flags = pa.pa_device_error()
    ms_total = t0.elapsed_time(t1)
    attn_ms = float(np.mean([ev_a[k].elapsed_time(ev_b[k]) for k in range(K)]))

    def reduce_max(x):
        return rank_reduce(x, "max", world, dev)

    def reduce_sum(x):
        return rank_reduce(x, "sum", world, dev)

    ms_max = reduce_max(ms_total)
    flops_all = reduce_sum(float(pb.flops) * K)
    value = flops_all / (ms_max * 1e-3) / 1e12
    achieved = pb.flops / (attn_ms * 1e-3) / 1e12
    peak, peak_kind = measured_tensor_peak()

    e2e = None
    if not args.no_e2e:
        e2e = run_prefill_e2e(pa, pb, K, Wm, dev, world, reduce_max, reduce_sum)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = prefill_cpu_baseline(pb, args.cpu_seconds)
    if rank == 0:
        line = {
            "metric": PREFILL_METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": K,
            "warmup": Wm,
            "ms_per_step": round(ms_max / K, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": sh.dtype,
            "data": "synthetic",
            "config": prefill_config(pb, world),
            "pct_of_measured_bf16_peak": round(100.0 * value / peak / world, 2),
            "roofline": {
                "bound": "tensor",
                "kernel": "paged_prefill_kernel (tcgen05: S = Q K^T, O += P V, P in TMEM)",
                "achieved": round(achieved, 2),
                "peak": peak,
                "peak_source": (f"{peak_kind} bf16_tflops burst (MEASURED_PEAKS.json)"
                                if peak_kind == "measured" else "fallback 1590 TFLOP/s"),
                "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4),
                "traffic": prefill_profiled_traffic(),
                "traffic_note": "ncu dram__bytes_read + dram__bytes_write of one launch of this "
                                "workload (profiles/prefill_attention_16x512.md)",
                "flops_per_launch": pb.flops,
                "flops_note": "algorithmic: 4*D*Hq*(p+1) per chunk token; the kernel also "
                              "multiplies the masked part of diagonal tiles, which is not "
                              "counted",
                "avg_launch_ms": round(attn_ms, 5),
                "launch_timing": "CUDA events around every prefill call",
            },
            "e2e": e2e,
            "cpu_baseline": cpu,
            "gpu_launches": 2 * K,
            "device_error_flags": flags,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)


def run_prefill_e2e(pa, pb, K, Wm, dev, world, reduce_max, reduce_sum):
    """The prefill step through the public API from pinned host buffers: per
    step the chunk's q, new K/V, slots, block tables, context lengths and
    query offsets go host -> device as one packed copy, the two kernels run,
    the fp32 output comes back.  Upload, compute and download run on three
    streams with two buffer sets, so one step's download overlaps the next
    step's upload and kernels."""
    import torch
    import torch.distributed as dist
    b, sh = pb.batch, pb.shape
    T, S = b.num_tokens, b.num_seqs
    parts = [("q", b.q.dtype, tuple(b.q.shape), 2), ("k", b.k_new.dtype, tuple(b.k_new.shape), 2),
             ("v", b.v_new.dtype, tuple(b.v_new.shape), 2), ("slots", torch.int64, (T,), 8),
             ("tables", torch.int32, tuple(b.block_tables.shape), 4),
             ("lens", torch.int32, (S,), 4), ("qs", torch.int32, (S + 1,), 4)]
    off, pos = {}, 0
    for name, _, shape, es in parts:
        off[name] = pos
        pos += (int(np.prod(shape)) * es + 255) // 256 * 256
    total = pos

    def views(buf):
        return {name: buf[off[name]:off[name] + int(np.prod(shape)) * es].view(dt).view(shape)
                for name, dt, shape, es in parts}

    NBUF = 2
    h_buf = [torch.empty(total, dtype=torch.uint8).pin_memory() for _ in range(NBUF)]
    d_buf = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(NBUF)]
    h_in, d_in = [views(x) for x in h_buf], [views(x) for x in d_buf]
    for hv in h_in:
        hv["q"].copy_(b.q.cpu()); hv["k"].copy_(b.k_new.cpu()); hv["v"].copy_(b.v_new.cpu())
        hv["slots"].copy_(torch.from_numpy(pb.slots))
        hv["tables"].copy_(torch.from_numpy(b.block_tables))
        hv["lens"].copy_(torch.from_numpy(b.context_lens))
        hv["qs"].copy_(torch.from_numpy(b.query_start))
    h_out = [torch.empty(T, sh.num_q_heads, sh.head_dim).pin_memory() for _ in range(NBUF)]
    d_out = [torch.empty(T, sh.num_q_heads, sh.head_dim, device=dev) for _ in range(NBUF)]
    s_up, s_cmp, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(NBUF)]
    ev_cmp = [torch.cuda.Event() for _ in range(NBUF)]
    ev_dn = [torch.cuda.Event() for _ in range(NBUF)]
    used = [False] * NBUF

    def one(i):
        j = i % NBUF
        dv = d_in[j]
        with torch.cuda.stream(s_up):
            if used[j]:
                s_up.wait_event(ev_cmp[j])
            d_buf[j].copy_(h_buf[j], non_blocking=True)
            ev_up[j].record(s_up)
        s_cmp.wait_event(ev_up[j])
        if used[j]:
            s_cmp.wait_event(ev_dn[j])
        pa.pa_reshape_and_cache(dv["k"], dv["v"], b.k_cache, b.v_cache, dv["slots"],
                                stream=s_cmp)
        pa.pa_paged_prefill_attention(d_out[j], dv["q"], b.k_cache, b.v_cache, dv["tables"],
                                      dv["lens"], dv["qs"], b.scale, sh.num_kv_heads,
                                      pb.max_query_len, stream=s_cmp)
        ev_cmp[j].record(s_cmp)
        with torch.cuda.stream(s_dn):
            s_dn.wait_event(ev_cmp[j])
            h_out[j].copy_(d_out[j], non_blocking=True)
            ev_dn[j].record(s_dn)
        used[j] = True

    for i in range(Wm):
        one(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for i in range(Wm, Wm + K):
        one(i)
    torch.cuda.synchronize()
    dt = reduce_max(time.perf_counter() - t0)
    flops_all = reduce_sum(float(pb.flops) * K)
    return {"value": round(flops_all / dt / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(total), "d2h_bytes_per_step": int(h_out[0].numel() * 4),
            "ms_per_step": round(dt * 1e3 / K, 4),
            "timing": "host wall clock, synchronize on both sides, max over ranks; one packed "
                      "upload, two kernels, one download per step on three streams, two buffer "
                      "sets (PCIe-bound: the step moves its q and fp32 output)"}


def prefill_oracle_sample(pb, seqs, kb, vb):
    """The oracle's chunked prefill for some sequences on the pool bits after
    the chunk's cache write.  Returns (seconds, flops)."""
    from oracle import attention as OA
    b, sh = pb.batch, pb.shape
    t0 = time.perf_counter()
    OA.paged_prefill_attention(W.bits(b.q), kb, vb, b.block_tables, b.context_lens,
                               b.query_start, b.scale, sh.num_kv_heads, sh.block_size, sh.dtype,
                               seqs=seqs)
    dt = time.perf_counter() - t0
    return dt, prefill_flops(b.context_lens[seqs], b.chunk_lens[seqs], sh.num_q_heads,
                             sh.head_dim)


def prefill_oracle_pool(pb):
    from oracle import cache_ops as OC
    b = pb.batch
    kb, vb = W.bits(b.k_cache), W.bits(b.v_cache)
    OC.reshape_and_cache(W.bits(b.k_new), W.bits(b.v_new), kb, vb, pb.slots, pb.shape.block_size)
    return kb, vb


def prefill_cpu_baseline(pb, seconds: float):
    """The oracle on whole sequences of the prefill batch until about
    `seconds` of CPU work are spent (shortest contexts first)."""
    kb, vb = prefill_oracle_pool(pb)
    order = np.argsort(pb.batch.context_lens).tolist()
    spent, flops, done = 0.0, 0, 0
    for s in order:
        dt, f = prefill_oracle_sample(pb, [int(s)], kb, vb)
        spent += dt
        flops += f
        done += 1
        if spent >= seconds:
            break
    return {"value": round(flops / spent / 1e12, 6), "unit": "TFLOP/s",
            "cores": cpu_cores_used(), "kind": "oracle",
            "sample": f"{done} of {pb.batch.num_seqs} sequences of the prefill batch (fp64 "
                      f"attention of every chunk token), {spent:.1f} s of CPU work"}


def run_prefill_reference(args, rank, world):
    """The reference arm for the prefill workload: the CPU oracle."""
    if rank != 0:
        return
    import paged_kv_cache_414_b200 as pa
    from paged_kv_cache_414_b200 import build as pbuild
    pbuild.build()
    K, Wm = args.steps, args.warmup
    pb = PrefillBench(pa, "cpu", 0)
    kb, vb = prefill_oracle_pool(pb)
    order = np.argsort(pb.batch.context_lens).tolist()
    times, flops = [], []
    for i in range(Wm + K):
        dt, f = prefill_oracle_sample(pb, [int(order[i % len(order)])], kb, vb)
        if i >= Wm:
            times.append(dt)
            flops.append(f)
    value = sum(flops) / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": PREFILL_METRIC, "value": round(value, 6),
        "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": Wm,
        "ms_per_step": round(1e3 * sum(times) / K, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": prefill_config(pb, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_cores_used(),
                         "kind": "oracle",
                         "sample": "one sequence of the prefill batch per step (fp64 attention "
                                   "of every chunk token)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- KV memory report

# The pages' figures the report is set beside (context, not targets).
PAGES_KV_FIGURES = {
    "prior_systems_useful_kv_fraction": [0.20, 0.38],
    "prior_systems_useful_source": "vLLM & PagedAttention: OS Ideas for LLM Serving, section 01 "
                                   "'The Problem' (the 2023 paper's measurement)",
    "prior_systems_memory_wasted_fraction": [0.60, 0.80],
    "prior_systems_wasted_source": "Why OS Virtual Memory Paging Saved LLM Inference, "
                                   "introduction; vLLM & PagedAttention, introduction",
    "paged_waste_fraction_below": 0.04,
    "paged_waste_source": "Why OS Virtual Memory Paging Saved LLM Inference, section 3",
    "example": {"reserved_tokens": 2048, "used_tokens": 150, "idle_slots": 1898,
                "source": "Why OS Virtual Memory Paging Saved LLM Inference, section 1"},
}


def kv_accounting(stats: dict, reserve: int) -> dict:
    """KV memory of a block manager's live sequences (its pa_bm_stats) against
    a contiguous reservation of `reserve` tokens per sequence, the allocation
    paged blocks replace: slots allocated, the fraction holding tokens, idle
    slots.  A block shared by several sequences is one allocation whose
    filled slots count once; a contiguous reservation shares nothing, so
    every sequence's tokens are stored (and useful) in its own buffer."""
    B = stats["block_size"]
    paged = stats["used_blocks"] * B
    filled = stats["filled_slots"]
    tokens = stats["logical_tokens"]
    contiguous = stats["num_seqs"] * reserve
    return {
        "sequences": stats["num_seqs"],
        "logical_tokens": tokens,
        "paged_slots": paged,
        "paged_filled_slots": filled,
        "paged_idle_slots": paged - filled,
        "paged_useful_fraction": filled / paged if paged else 1.0,
        "paged_waste_fraction": (paged - filled) / paged if paged else 0.0,
        "shared_blocks": stats["shared_blocks"],
        "sharing_ratio": tokens / filled if filled else 1.0,
        "contiguous_reserve_tokens": reserve,
        "contiguous_slots": contiguous,
        "contiguous_idle_slots": contiguous - tokens,
        "contiguous_useful_fraction": tokens / contiguous if contiguous else 1.0,
        "paged_slots_per_contiguous_slot": paged / contiguous if contiguous else 0.0,
    }


def kv_report(pa) -> dict:
    """Paged versus contiguous KV memory on the workloads' length mixes, from
    the native block manager's own accounting (pa_bm_stats)."""
    out = {"report": "kv_utilisation", "source": "pa_bm_stats of the native block manager",
           "pages": PAGES_KV_FIGURES, "workloads": {}}
    # the pages' worked example through the manager: one 150-token request
    bm = pa.BlockManager(16, 16)
    bm.allocate(0, 150)
    out["workloads"]["example_150_tokens"] = dict(
        kv_accounting(bm.stats(), 2048), reserve_reason="the pages' 2,048-token reservation")
    bm.close()
    reserves = {"13b": (2048, "the workload's longest context"),
                "gqa8b": (4096, "the workload's longest context"),
                "long": (32768, "the workload's longest context")}
    for name, (reserve, why) in reserves.items():
        sh = W.SHAPES[name]
        lens = {"13b": W.lens_13b, "gqa8b": W.lens_gqa8b,
                "long": W.lens_long}[name](np.random.default_rng(W.SEEDS[name]))
        nblk = int(sum(-(-int(L) // sh.block_size) for L in lens))
        bm = pa.BlockManager(nblk, sh.block_size)
        for s, L in enumerate(lens):
            bm.allocate(s, int(L))
        out["workloads"][name] = dict(kv_accounting(bm.stats(), reserve), reserve_reason=why)
        bm.close()
    # parallel sampling: prompts shared by their 8 branches, then 64 decode
    # steps with copy-on-write of the shared partial last blocks
    cw = W.cow_workload()
    B = cw.shape.block_size
    bm = pa.BlockManager(cw.num_blocks, B, cw.free_order)
    for p_, P in enumerate(cw.prompt_lens):
        bm.allocate(cw.seq_id(p_, 0), int(P))
        for br in range(1, cw.branches):
            bm.fork(cw.seq_id(p_, 0), cw.seq_id(p_, br))
    why = "the pages' 2,048-token reservation per branch (contexts reach 576 tokens)"
    out["workloads"]["cow_after_fork"] = dict(kv_accounting(bm.stats(), 2048), reserve_reason=why)
    seqs = np.arange(cw.num_seqs)
    for _ in range(cw.steps):
        bm.append_slots(seqs)
    out["workloads"]["cow_after_64_steps"] = dict(kv_accounting(bm.stats(), 2048),
                                                  reserve_reason=why)
    bm.close()
    return out


# ----------------------------------------------------------------------------- oracle (CPU)

def oracle_step_sample(wl, step: int, seqs):
    """The oracle's decode step for some sequences: its own block manager's
    slots, its own cache write, its own attention.  Returns (out, bytes)."""
    from oracle import attention as OA
    from oracle import cache_ops as OC
    sh = wl.shape
    B = sh.block_size
    b = wl.batch
    bm, slots = wl.oracle_manager(step)
    need = sorted({x for s in seqs for x in bm.block_table(s)})
    remap = {x: i for i, x in enumerate(need)}
    import torch
    idx = torch.as_tensor(need, device=b.k_cache.device)
    kb = W.bits(b.k_cache.index_select(0, idx))
    vb = W.bits(b.v_cache.index_select(0, idx))
    qb, knb, vnb = W.bits(b.q)[seqs], W.bits(b.k_new)[seqs], W.bits(b.v_new)[seqs]
    sub = [remap[slots[s] // B] * B + slots[s] % B for s in seqs]
    t0 = time.perf_counter()
    OC.reshape_and_cache(knb, vnb, kb, vb, np.array(sub), B)
    tabs = np.full((len(seqs), wl.maxb), -1, dtype=np.int64)
    lens = np.zeros(len(seqs), dtype=np.int64)
    for i, s in enumerate(seqs):
        t = [remap[x] for x in bm.block_table(s)]
        tabs[i, :len(t)] = t
        lens[i] = bm.seq_len(s)
    OA.paged_decode_attention(qb, kb, vb, tabs, lens, wl.scale, sh.num_kv_heads, B, sh.dtype)
    dt = time.perf_counter() - t0
    return dt, decode_bytes(lens, sh.num_kv_heads, sh.head_dim, B, 2)


def cpu_baseline(wl, seconds: float):
    """The oracle on a bounded sample of the workload: whole steps of random
    sequences until about `seconds` of CPU work are spent."""
    rng = np.random.default_rng(0)
    spent, nbytes, done, step = 0.0, 0, 0, 0
    while spent < seconds and step < wl.steps_total:
        for s in rng.permutation(wl.S):
            dt, nb = oracle_step_sample(wl, step, [int(s)])
            spent += dt
            nbytes += nb
            done += 1
            if spent >= seconds:
                break
        step += 1
    return {"value": round(nbytes / spent / 1e9, 4), "unit": "GB/s", "cores": cpu_cores_used(),
            "kind": "oracle",
            "sample": f"{done} sequence-steps of the same workload ({wl.S} sequences per step; "
                      f"oracle cache write + fp64 attention), {spent:.1f} s of CPU work"}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, on bounded samples of the same workload."""
    if rank != 0:
        return
    import torch
    K, Wm = args.steps, args.warmup
    wl = Workload(args.workload, "cpu", 0, K + Wm + 1)
    per_step_budget = max(0.5, min(6.0, 150.0 / max(1, K + Wm)))
    rng = np.random.default_rng(1)
    order = rng.permutation(wl.S).tolist()
    # size one step's sample so it takes about per_step_budget seconds
    dt, _ = oracle_step_sample(wl, 0, order[:1])
    nseq = max(1, min(wl.S, int(per_step_budget / max(dt, 1e-3))))
    times, nbytes = [], []
    for i in range(Wm + K):
        seqs = [order[(i * nseq + j) % wl.S] for j in range(nseq)]
        dt, nb = oracle_step_sample(wl, i, seqs)
        if i >= Wm:
            times.append(dt)
            nbytes.append(nb)
    value = sum(nbytes) / sum(times) / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": round(1e3 * sum(times) / K, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": decode_config(wl, args.workload, world, K, Wm),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cpu_cores_used(),
                         "kind": "oracle",
                         "sample": f"{nseq} of {wl.S} sequences per step (oracle cache write + "
                                   f"fp64 attention)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.report == "kv":
        if rank == 0:
            from paged_kv_cache_414_b200 import build as pbuild
            pbuild.build()
            import paged_kv_cache_414_b200 as pa
            print(json.dumps(kv_report(pa)), flush=True)
        return
    if args.impl == "reference":
        if args.workload == "prefill":
            run_prefill_reference(args, rank, world)
        else:
            run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.workload == "prefill":
            run_prefill_b200(args, rank, world, local_rank)
        else:
            run_b200(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
