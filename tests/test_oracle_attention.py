"""Pins for the attention oracle: everything here checks oracle/attention.py and
oracle/fp.py against something other than themselves (known bit patterns,
closed forms, brute force, torch's own attention routine, invariants the pages
state)."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle.fp import bf16_bits_to_f64, decode, f16_bits_to_f64
import workloads as W


# ---------------------------------------------------------------- fp decoding

F16_KNOWN = [  # IEEE 754 binary16 encodings
    (0x3C00, 1.0), (0xC000, -2.0), (0x0001, 2.0 ** -24), (0x0400, 2.0 ** -14),
    (0x7BFF, 65504.0), (0x3555, 0.333251953125), (0x8000, -0.0), (0x7C00, math.inf),
    (0x3800, 0.5), (0x4248, 3.140625),
]
BF16_KNOWN = [  # bfloat16 = upper half of binary32
    (0x3F80, 1.0), (0xC040, -3.0), (0x3EAB, 0.333984375), (0x0001, 2.0 ** -133),
    (0x0080, 2.0 ** -126), (0x7F7F, (2 - 2.0 ** -7) * 2.0 ** 127), (0x7F80, math.inf),
    (0x4049, 3.140625), (0xBF00, -0.5),
]


@pytest.mark.parametrize("bits,val", F16_KNOWN)
def test_f16_decode_known(bits, val):
    got = f16_bits_to_f64(np.array([bits], dtype=np.uint16))[0]
    assert got == val and math.copysign(1, got) == math.copysign(1, val)


@pytest.mark.parametrize("bits,val", BF16_KNOWN)
def test_bf16_decode_known(bits, val):
    assert bf16_bits_to_f64(np.array([bits], dtype=np.uint16))[0] == val


def test_decode_matches_torch_widening():
    rng = np.random.default_rng(5)
    b = rng.integers(0, 0x7C00, size=4096, dtype=np.uint16)
    t16 = torch.from_numpy(b.view(np.int16)).view(torch.float16).double().numpy()
    assert np.array_equal(decode(b, "f16"), t16)
    b2 = rng.integers(0, 0x7F80, size=4096, dtype=np.uint16)
    tb = torch.from_numpy(b2.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(decode(b2, "bf16"), tb)


# ---------------------------------------------------------------- helpers

def _contiguous_pool(K, V, B, rng=None):
    """Lay logical K/V [L, Hkv, D] (float64, exactly fp16-representable) into a
    pool with a random (or identity) physical placement.  Returns pool bits and
    the block table row."""
    L, Hkv, D = K.shape
    nb = -(-L // B)
    num_blocks = nb + 3
    perm = np.arange(num_blocks) if rng is None else rng.permutation(num_blocks)
    table = perm[:nb]
    kp = rng.standard_normal((num_blocks, Hkv, B, D)) if rng is not None else np.zeros((num_blocks, Hkv, B, D))
    vp = kp.copy()
    for t in range(L):
        kp[table[t // B], :, t % B, :] = K[t]
        vp[table[t // B], :, t % B, :] = V[t]
    kb = kp.astype(np.float16).view(np.uint16)
    vb = vp.astype(np.float16).view(np.uint16)
    return kb, vb, table


def _f16(x):
    return np.asarray(x, dtype=np.float16).astype(np.float64)


def _rand_case(rng, L, Hq, Hkv, D):
    q = _f16(rng.standard_normal((Hq, D)))
    K = _f16(rng.standard_normal((L, Hkv, D)))
    V = _f16(rng.standard_normal((L, Hkv, D)))
    return q, K, V


def _run_oracle(q, kb, vb, table, L, scale, Hkv, B):
    qb = q.astype(np.float16).view(np.uint16)[None]
    return A.paged_decode_attention(qb, kb, vb, table[None], np.array([L]), scale, Hkv, B, "f16")[0]


# ---------------------------------------------------------------- brute force

def test_brute_force_tiny():
    """Scalar loops with math.exp on a 5-token, 2-head case."""
    rng = np.random.default_rng(1)
    L, Hq, Hkv, D, B = 5, 2, 1, 3, 2
    q, K, V = _rand_case(rng, L, Hq, Hkv, D)
    kb, vb, table = _contiguous_pool(K, V, B, rng)
    scale = 0.7
    got = _run_oracle(q, kb, vb, table, L, scale, Hkv, B)
    for h in range(Hq):
        z = [scale * sum(q[h, d] * K[t, 0, d] for d in range(D)) for t in range(L)]
        e = [math.exp(x - max(z)) for x in z]
        tot = sum(e)
        for d in range(D):
            want = sum(e[t] / tot * V[t, 0, d] for t in range(L))
            assert abs(got[h, d] - want) < 1e-13


@pytest.mark.parametrize("L,B,Hq,Hkv,D", [(1, 16, 4, 4, 64), (17, 16, 4, 4, 64), (100, 16, 8, 2, 32),
                                          (33, 8, 6, 3, 16), (250, 32, 8, 1, 128)])
def test_matches_torch_sdpa(L, B, Hq, Hkv, D):
    """The contiguous special case ([P1] section 1: ordinary attention over
    contiguous K/V) is torch's scaled_dot_product_attention; with grouped
    heads query head h reads kv head h // (Hq/Hkv) (enable_gqa)."""
    rng = np.random.default_rng(L * 7 + B)
    q, K, V = _rand_case(rng, L, Hq, Hkv, D)
    kb, vb, table = _contiguous_pool(K, V, B, rng)
    scale = 1.0 / math.sqrt(D)
    got = _run_oracle(q, kb, vb, table, L, scale, Hkv, B)
    qt = torch.from_numpy(q)[None, :, None, :]                  # [1, Hq, 1, D]
    kt = torch.from_numpy(K).permute(1, 0, 2)[None]             # [1, Hkv, L, D]
    vt = torch.from_numpy(V).permute(1, 0, 2)[None]
    want = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, scale=scale, enable_gqa=(Hq != Hkv))[0, :, 0, :].numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_identity_table_one_block():
    """Block size >= L with an identity table: one block holds the sequence."""
    rng = np.random.default_rng(2)
    L, D = 40, 16
    q, K, V = _rand_case(rng, L, 2, 2, D)
    kb, vb, table = _contiguous_pool(K, V, 64, None)
    got = _run_oracle(q, kb, vb, table, L, 0.25, 2, 64)
    want = np.stack([A.softmax_attention(q[h], K[:, h], V[:, h], 0.25) for h in range(2)])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- closed forms

def test_length_one_returns_own_v_exactly():
    rng = np.random.default_rng(3)
    q, K, V = _rand_case(rng, 1, 4, 2, 64)
    kb, vb, table = _contiguous_pool(K, V, 16, rng)
    got = _run_oracle(q, kb, vb, table, 1, 0.125, 2, 16)
    for h in range(4):
        assert np.array_equal(got[h], V[0, h // 2])


def test_constant_v():
    rng = np.random.default_rng(4)
    q, K, V = _rand_case(rng, 37, 2, 1, 8)
    V[:] = _f16(rng.standard_normal(8))[None, None, :]
    kb, vb, table = _contiguous_pool(K, V, 16, rng)
    got = _run_oracle(q, kb, vb, table, 37, 0.3, 1, 16)
    np.testing.assert_allclose(got, np.broadcast_to(V[0, 0], got.shape), rtol=0, atol=1e-14)


def test_scale_zero_is_mean_of_v():
    rng = np.random.default_rng(5)
    q, K, V = _rand_case(rng, 29, 2, 2, 8)
    kb, vb, table = _contiguous_pool(K, V, 8, rng)
    got = _run_oracle(q, kb, vb, table, 29, 0.0, 2, 8)
    for h in range(2):
        np.testing.assert_allclose(got[h], V[:, h].mean(axis=0), rtol=0, atol=1e-14)


def test_identical_keys_is_mean_of_v():
    rng = np.random.default_rng(6)
    q, K, V = _rand_case(rng, 21, 1, 1, 8)
    K[:] = K[0]
    kb, vb, table = _contiguous_pool(K, V, 4, rng)
    got = _run_oracle(q, kb, vb, table, 21, 0.9, 1, 4)
    np.testing.assert_allclose(got[0], V[:, 0].mean(axis=0), rtol=0, atol=1e-14)


def test_peaked_softmax_selects_the_hot_token():
    """A key whose score exceeds all others by a margin g makes the output the
    hot token's V up to a weight of at most (L-1) e^{-g} on the rest."""
    rng = np.random.default_rng(7)
    L, D = 64, 16
    q, K, V = _rand_case(rng, L, 1, 1, D)
    K[:] = 0.0
    K[13, 0] = _f16(30.0 * q[0] / np.linalg.norm(q[0]))
    kb, vb, table = _contiguous_pool(K, V, 16, rng)
    got = _run_oracle(q, kb, vb, table, L, 1.0, 1, 16)
    gap = float(K[13, 0] @ q[0])
    bound = (L - 1) * math.exp(-gap) * 2 * np.abs(V).max()
    np.testing.assert_allclose(got[0], V[13, 0], rtol=0, atol=bound + 1e-15)


def test_empty_sequence_is_zero():
    qb = np.zeros((1, 2, 8), dtype=np.uint16)
    kb = np.zeros((2, 1, 4, 8), dtype=np.uint16)
    out = A.paged_decode_attention(qb, kb, kb, np.array([[-1]]), np.array([0]), 1.0, 1, 4, "f16")
    assert np.array_equal(out, np.zeros_like(out))


def test_softmax_weights_translation_invariant():
    """Adding a constant to every score does not change the softmax: a key
    offset along q by c shifts every z by c*|q|^2*scale."""
    rng = np.random.default_rng(8)
    qv = rng.standard_normal(8)
    K = rng.standard_normal((10, 8))
    V = rng.standard_normal((10, 8))
    a = A.softmax_attention(qv, K, V, 0.5)
    b = A.softmax_attention(qv, K + 3.0 * qv / (qv @ qv), V, 0.5)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- invariants from the pages

def _batch(rng, lens, Hq, Hkv, D, B):
    sh = W.Shape(Hq, Hkv, D, B, "bf16")
    return W.make_decode_batch(sh, lens, int(rng.integers(1 << 30)), num_blocks=None)


def test_permutation_of_physical_blocks_is_invisible():
    """[P1] section 2, [P3] second paragraph: blocks may sit anywhere; only the
    logical order matters.  Permuting the pool and the table together leaves
    the output bit-identical."""
    rng = np.random.default_rng(9)
    b = _batch(rng, [1, 16, 17, 70, 129], 8, 2, 32, 16)
    kb, vb, qb = W.bits(b.k_cache), W.bits(b.v_cache), W.bits(b.q)
    out1 = A.paged_decode_attention(qb, kb, vb, b.block_tables, b.context_lens, b.scale, 2, 16, "bf16")
    perm = rng.permutation(b.num_blocks)         # new position of every block
    kb2 = np.empty_like(kb); vb2 = np.empty_like(vb)
    kb2[perm] = kb; vb2[perm] = vb
    t2 = np.where(b.block_tables >= 0, perm[np.maximum(b.block_tables, 0)], -1)
    out2 = A.paged_decode_attention(qb, kb2, vb2, t2, b.context_lens, b.scale, 2, 16, "bf16")
    assert np.array_equal(out1, out2)


@pytest.mark.parametrize("B", [1, 2, 8, 16, 32])
def test_block_size_is_a_storage_choice(B):
    """[P1] section 2 ("e.g., 16 tokens per block"): the same logical K/V
    stored with any block size gives a bit-identical result."""
    rng = np.random.default_rng(10)
    L, Hkv, D = 45, 2, 16
    q, K, V = _rand_case(rng, L, 4, Hkv, D)
    ref = None
    for BB in (B, 64):
        kb, vb, table = _contiguous_pool(K, V, BB, np.random.default_rng(BB))
        out = _run_oracle(q, kb, vb, table, L, 0.25, Hkv, BB)
        ref = out if ref is None else ref
        assert np.array_equal(out, ref)


@pytest.mark.parametrize("part", [1, 3, 16, 512, 10_000])
def test_split_context_merge_is_exact(part):
    """Merging per-partition (max, sum, accumulator) reproduces attention over
    the whole sequence (the algebra the split-context reduce relies on)."""
    rng = np.random.default_rng(11)
    L, D = 700, 32
    qv = rng.standard_normal(D)
    K = 3 * rng.standard_normal((L, D))
    V = rng.standard_normal((L, D))
    want = A.softmax_attention(qv, K, V, 0.4)
    got = A.split_context_attention(qv, K, V, 0.4, part)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_merge_single_partial_is_normalisation():
    m, l, acc = 2.0, 4.0, np.array([8.0, -2.0])
    assert np.array_equal(A.merge_partials([(m, l, acc)]), np.array([2.0, -0.5]))


def test_merge_weights_partials_by_exp_of_max_difference():
    """Two partials whose maxima differ by ln 2: the first counts twice."""
    p1 = (math.log(2.0), 1.0, np.array([1.0]))
    p2 = (0.0, 1.0, np.array([4.0]))
    # exp(m - M): 1 for p1, 1/2 for p2 -> (1 + 2) / (1 + 0.5) = 2
    assert A.merge_partials([p1, p2])[0] == pytest.approx(2.0, abs=1e-15)


def test_unused_slots_are_not_read():
    """Everything outside a sequence's tokens may be NaN."""
    rng = np.random.default_rng(12)
    sh = W.Shape(4, 2, 16, 16, "f16")
    b = W.make_decode_batch(sh, [3, 16, 33], 1, poison="nan")
    out = A.paged_decode_attention(W.bits(b.q), W.bits(b.k_cache), W.bits(b.v_cache),
                                   b.block_tables, b.context_lens, b.scale, 2, 16, "f16")
    assert np.isfinite(out).all()
