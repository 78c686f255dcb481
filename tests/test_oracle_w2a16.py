"""Pins for the oracle's INT2 (W2A16) container, dequantization, GEMM and
packed layout: a hand-built word, closed forms over every code and zero
point, exact rational brute force, a reduction to a plain fp64 matmul, and
the layout's bijection, round trip, hand example and bf16 decoding
property."""

import struct
from fractions import Fraction

import numpy as np
import torch

from oracle import formats as F
from oracle import gemm as G
from oracle import layout as L
from quantized_gemm_bit_b200 import synth


def _bf16_exact(bits):
    return Fraction(struct.unpack("<f", struct.pack("<I", int(bits) << 16))[0])


def _a_bits(m, k, seed):
    return synth.bf16_normal(m, k, seed).view(torch.int16).numpy().view(np.uint16)


def _decode_python(qrow):
    """Codes of one row by plain Python integer arithmetic."""
    out = []
    for w in qrow.tolist():
        w &= 0xFFFFFFFF
        out.extend((w >> (2 * e)) & 3 for e in range(16))
    return out


def test_int2_words_hand_example():
    # codes 3, 0, 1, 2 then zeros: word = 0b10_01_00_11 = 0x93
    codes = np.zeros((1, 16), dtype=np.uint8)
    codes[0, :4] = [3, 0, 1, 2]
    w = F.int2_pack_words(codes)
    assert w.view(np.uint32).tolist() == [[0x93]]
    assert np.array_equal(F.int2_unpack_words(w), codes)


def test_w2a16_dequant_closed_form_every_code_and_zero():
    codes = np.tile(np.arange(4, dtype=np.uint8), 32)[None, :].repeat(4, axis=0)    # [4, 128]
    q = F.int2_pack_words(codes)
    s = np.full((4, 1), 0.25, dtype=np.float16)
    z = np.arange(4, dtype=np.uint8)[:, None]
    assert np.array_equal(G.w2a16_dequant(q, s, z, 128), (codes.astype(np.float64) - z) / 4)
    assert np.array_equal(G.w2a16_dequant(q, s, None, 128), (codes.astype(np.float64) - 2) / 4)


def test_w2a16_brute_force_in_rationals():
    m, n, k = 2, 3, 256
    q, s, z = synth.w2a16_weights(n, k, 128, True, seed=41)
    a = _a_bits(m, k, 42)
    got = G.w2a16_ref(a, q.numpy(), s.numpy(), z.numpy(), 128)
    for r in range(n):
        codes = _decode_python(q.numpy()[r])
        for i in range(m):
            acc = Fraction(0)
            for kk in range(k):
                g = kk // 128
                acc += _bf16_exact(a[i, kk]) * (codes[kk] - int(z.numpy()[r, g])) * Fraction(float(s.numpy()[r, g]))
            assert abs(got[i, r] - float(acc)) <= 1e-12 * max(1.0, abs(float(acc)))


def test_w2a16_unit_scale_zero_zero_is_plain_matmul():
    m, n, k = 5, 40, 384
    q, _, _ = synth.w2a16_weights(n, k, 128, False, seed=43)
    s = np.ones((n, k // 128), dtype=np.float16)
    z = np.zeros((n, k // 128), dtype=np.uint8)
    a = _a_bits(m, k, 44)
    got = G.w2a16_ref(a, q.numpy(), s, z, 128)
    w = torch.tensor([_decode_python(q.numpy()[r]) for r in range(n)], dtype=torch.float64)
    at = torch.from_numpy(a.astype(np.int32) << 16).view(torch.float32).double()
    assert np.array_equal(got, (at @ w.T).numpy())


def test_grouped_w2a16_equals_dense_per_expert():
    e, n, k = 3, 24, 128
    q, s, z = synth.w2a16_weights(n, k, 128, True, seed=45, experts=e)
    off = np.array([0, 0, 6, 11])
    a = _a_bits(11, k, 46)
    _, got = G.grouped_w2a16_ref(a, off, q.numpy(), s.numpy(), z.numpy(), 128)
    for x in range(e):
        lo, hi = off[x], off[x + 1]
        if hi > lo:
            assert np.array_equal(got[lo:hi], G.w2a16_ref(a[lo:hi], q.numpy()[x], s.numpy()[x], z.numpy()[x], 128))


def test_w2a16_layout_is_a_bijection():
    for n, k, hz in ((128, 256, False), (200, 384, True)):
        nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
        word, bit = L.w2a16_code_word_and_bit(nn.ravel(), kk.ravel(), k, hz)
        slots = word * 8 + bit                       # low bit of each 2-bit field
        assert len(np.unique(slots)) == slots.size and np.all(bit % 2 == 0)
        ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
        sb = L.w2a16_scale_byte(ng.ravel(), gg.ravel(), k, hz)
        code_bytes = set(np.unique(word).tolist()) | set(np.unique(word + 3).tolist())
        assert not code_bytes & set(sb.tolist())
        if hz:
            assert not code_bytes & set(L.w2a16_zero_byte(ng.ravel(), gg.ravel(), k).tolist())
        if n % 128 == 0:
            assert len(np.unique(word)) * 4 == (n // 128) * (k // 128) * 4096


def test_w2a16_pack_unpack_roundtrip_and_padding():
    for hz in (False, True):
        q, s, z = synth.w2a16_weights(136, 256, 128, hz, seed=47)
        blob = L.w2a16_pack(q.numpy(), s.numpy(), None if z is None else z.numpy())
        assert blob.size == L.w2a16_packed_bytes(136, 256, hz)
        c2, s2, z2 = L.w2a16_unpack(blob, 136, 256, hz)
        assert np.array_equal(c2, F.int2_unpack_words(q.numpy()))
        assert np.array_equal(s2.view(np.uint16), s.numpy().view(np.uint16))
        if hz:
            assert np.array_equal(z2, z.numpy())
        rec = L.w2a16_record_bytes(hz)
        tile1 = blob[2 * rec:].reshape(2, rec)
        assert np.all(tile1[:, :4096].reshape(2, 2, 128, 16)[:, :, 8:, :] == 0)


def test_w2a16_layout_small_hand_example():
    """Code (n=1, k=45): chunk 1, pair 6, odd half -> word q = 2 at byte
    (0*128 + 1)*16 + 8 = 24, bits 28..29.  Code (n=0, k=60): chunk 1, pair
    14 -> word q = 3 at byte 12, bits 12..13."""
    word, bit = L.w2a16_code_word_and_bit(1, 45, 128, False)
    assert (int(word), int(bit)) == (24, 28)
    word, bit = L.w2a16_code_word_and_bit(0, 60, 128, False)
    assert (int(word), int(bit)) == (12, 12)
    assert int(L.w2a16_scale_byte(1, 0, 128, True)) == 4098
    assert int(L.w2a16_zero_byte(1, 0, 128)) == 4096 + 256 + 1


def test_w2a16_pairs_decode_as_bf16_128_plus_code():
    """Pair i of a chunk sits at bits 2j / 16 + 2j of word 2c + i // 8
    (j = i % 8): a shift by 2j, the mask 0x00030003 and the bits of bf16
    128.0 give the bf16 pair (128 + q_even, 128 + q_odd)."""
    rng = np.random.default_rng(48)
    codes = rng.integers(0, 4, size=(128, 128)).astype(np.uint8)
    blob = L.w2a16_pack(F.int2_pack_words(codes), np.ones((128, 1), dtype=np.float16), None)
    words = blob[:4096].view(np.uint32)
    for r in (0, 50, 127):
        rw = [int(words[(qq // 4 * 128 + r) * 4 + qq % 4]) for qq in range(8)]
        for c in range(4):
            for i in range(16):
                x = ((rw[2 * c + i // 8] >> (2 * (i % 8))) & 0x00030003) | 0x43004300
                for h in range(2):
                    assert _bf16_exact((x >> (16 * h)) & 0xFFFF) == 128 + int(codes[r, 32 * c + 2 * i + h])
