"""The C ABI: libpa.so loads, exports every function include/pa.h declares,
and rejects bad arguments on the host before touching the GPU."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(pa_\w+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("pa_reshape_and_cache", "pa_paged_decode_attention", "pa_copy_blocks",
                 "pa_paged_decode_workspace_bytes", "pa_bm_create", "pa_bm_allocate",
                 "pa_bm_fork", "pa_bm_append_slot", "pa_bm_free", "pa_bm_block_table"):
        assert want in names


def test_every_declared_symbol_is_exported(pa):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(pa_\w+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    L = pa.lib()
    for n in declared_functions():
        assert hasattr(L, n)


def test_status_strings(pa):
    L = pa.lib()
    assert L.pa_status_string(0) == b"PA_OK"
    assert L.pa_status_string(-3).startswith(b"PA_ERR_NO_BLOCKS")
    assert L.pa_version() >= 100


def test_host_argument_checks(pa):
    L = pa.lib()
    nul = None
    # negative sizes, bad dtype, unsupported shapes: rejected before any CUDA call
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, -1, 8, 128, 16, 10, 1, nul) == -1
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, 4, 8, 128, 16, 10, 7, nul) == -1
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, 4, 8, 96, 16, 10, 1, nul) == -2
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, 4, 8, 128, 16, 10, 1, nul) == -1
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, 0, 8, 128, 16, 10, 1, nul) == 0
    def attn(kv=8, seqs=4, qh=32, hd=128, bs=16, maxb=4, maxctx=64, nblk=10, dt=1):
        return L.pa_paged_decode_attention(nul, nul, nul, nul, nul, nul, 1.0, kv, seqs, qh, hd,
                                           bs, maxb, maxctx, nblk, dt, nul, 0, nul)
    assert attn(qh=30) == -1            # q heads not a multiple of kv heads
    assert attn(bs=24) == -2            # unsupported block size
    assert attn(kv=1, qh=32) == -2      # group of 32 > 16
    assert attn(seqs=0) == 0            # nothing to do
    assert attn(maxctx=65) == -1        # longer than the table can hold
    assert attn() == -1                 # null pointers
    assert attn(dt=3) == -1
    assert L.pa_copy_blocks(nul, nul, nul, 0, 8, 128, 16, 10, 1, nul) == 0
    assert L.pa_copy_blocks(nul, nul, nul, 3, 8, 128, 16, 10, 1, nul) == -1
    assert L.pa_copy_blocks(nul, nul, nul, 3, 8, 100, 16, 10, 1, nul) == -2
    assert L.pa_copy_blocks(nul, nul, nul, 70000, 8, 128, 16, 10, 1, nul) == -2   # > 65535 pairs
    assert L.pa_copy_blocks(nul, nul, nul, 3, 8, 128, 16, 10, 2, nul) == -1      # fp32 pool
    assert L.pa_decode_tuning(-1, 0, 0) == -1
    assert L.pa_decode_tuning(0, 0, 0) == 0


def test_binding_refuses_cpu_tensors(pa):
    import torch
    k = torch.zeros(4, 2, 16, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        pa.pa_reshape_and_cache(torch.zeros(1, 2, 64, dtype=torch.float16),
                                torch.zeros(1, 2, 64, dtype=torch.float16), k, k.clone(),
                                torch.zeros(1, dtype=torch.int64))


def test_no_oracle_on_the_product_path():
    """The package never imports the oracle."""
    pkg = os.path.join(ROOT, "paged_kv_cache_414_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.replace("no oracle", ""), f


def test_prefill_host_argument_checks(pa):
    """pa_paged_prefill_attention refuses bad shapes on the host, and an empty
    call is a no-op, before any CUDA call."""
    L = pa.lib()
    nul = None

    def pf(kv=8, seqs=4, toks=16, qh=32, hd=128, bs=16, maxb=4, mq=4, nblk=10, dt=1):
        return L.pa_paged_prefill_attention(nul, nul, nul, nul, nul, nul, nul, 1.0, kv, seqs,
                                            toks, qh, hd, bs, maxb, mq, nblk, dt, nul)
    assert pf(qh=30) == -1              # q heads not a multiple of kv heads
    assert pf(hd=96) == -2              # unsupported head_dim
    assert pf(bs=8) == -2               # unsupported block size
    assert pf(kv=1, qh=32) == -2        # group of 32 > 16
    assert pf(dt=2) == -1               # fp32 cache
    assert pf(toks=-1) == -1
    assert pf(seqs=0) == 0 and pf(toks=0) == 0 and pf(mq=0) == 0
    assert pf() == -1                   # null pointers
