"""Pins for the oracle's INT3 (W3A16) container, dequantization, GEMM and
packed layout: hand-built bit streams, closed forms over every code and
zero point, exact rational brute force, an independent big-integer decode
feeding a plain fp64 matmul, and the layout's bijection, round trip, hand
example and bf16 decoding property."""

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


def _decode_bigint(qrow):
    """One row's words -> codes through one Python integer (stream bit b =
    bit b of the integer): independent of formats.int3_unpack_stream."""
    big = 0
    for i, w in enumerate(np.asarray(qrow).astype(np.int64) & 0xFFFFFFFF):
        big |= int(w) << (32 * i)
    k = len(qrow) * 32 // 3
    return [(big >> (3 * j)) & 7 for j in range(k)]


def test_int3_stream_hand_examples():
    # code 10 = 0b101 at stream bits 30, 31, 32; code 21 = 0b110 at 63, 64, 65
    q = np.zeros((1, 3), dtype=np.uint32)
    q[0, 0] = 1 << 30
    q[0, 1] = 1
    q[0, 2] = 3
    codes = F.int3_unpack_stream(q.view(np.int32))
    want = np.zeros(32, dtype=np.uint8)
    want[10], want[21] = 5, 6
    assert np.array_equal(codes[0], want)
    assert np.array_equal(F.int3_pack_stream(codes).view(np.uint32), q)
    # all codes 7: every bit set
    assert np.all(F.int3_pack_stream(np.full((2, 64), 7, np.uint8)).view(np.uint32) == 0xFFFFFFFF)


def test_int3_stream_matches_bigint_decode():
    q, _, _ = synth.w3a16_weights(4, 256, seed=31)
    codes = F.int3_unpack_stream(q.numpy())
    for r in range(4):
        assert codes[r].tolist() == _decode_bigint(q.numpy()[r])


def test_w3a16_dequant_closed_form_every_code_and_zero():
    """Codes 0..7 against zero points 0..7 with scale 2^-3: W = (q - z)/8."""
    codes = np.tile(np.arange(8, dtype=np.uint8), 16)[None, :].repeat(8, axis=0)   # [8, 128]
    q = F.int3_pack_stream(codes)
    s = np.full((8, 1), 0.125, dtype=np.float16)
    z = np.arange(8, dtype=np.uint8)[:, None]
    w = G.w3a16_dequant(q, s, z, 128)
    assert np.array_equal(w, (codes.astype(np.float64) - z) / 8)
    sym = G.w3a16_dequant(q, s, None, 128)
    assert np.array_equal(sym, (codes.astype(np.float64) - 4) / 8)


def test_w3a16_brute_force_in_rationals():
    m, n, k = 2, 3, 256
    q, s, z = synth.w3a16_weights(n, k, 128, True, seed=32)
    a = _a_bits(m, k, 33)
    got = G.w3a16_ref(a, q.numpy(), s.numpy(), z.numpy(), 128)
    for r in range(n):
        codes = _decode_bigint(q.numpy()[r])
        for i in range(m):
            acc = Fraction(0)
            for kk in range(k):
                g = kk // 128
                sc = Fraction(float(s.numpy()[r, g]))
                acc += _bf16_exact(a[i, kk]) * (codes[kk] - int(z.numpy()[r, g])) * sc
            assert abs(got[i, r] - float(acc)) <= 1e-12 * max(1.0, abs(float(acc)))


def test_w3a16_unit_scale_zero_zero_is_plain_matmul():
    m, n, k = 5, 40, 384
    q, _, _ = synth.w3a16_weights(n, k, 128, False, seed=34)
    s = np.ones((n, k // 128), dtype=np.float16)
    z = np.zeros((n, k // 128), dtype=np.uint8)
    a = _a_bits(m, k, 35)
    got = G.w3a16_ref(a, q.numpy(), s, z, 128)
    w = torch.tensor([_decode_bigint(q.numpy()[r]) for r in range(n)], dtype=torch.float64)
    at = torch.from_numpy(a.astype(np.int32) << 16).view(torch.float32).double()
    assert np.array_equal(got, (at @ w.T).numpy())


def test_grouped_w3a16_equals_dense_per_expert():
    e, n, k = 3, 24, 128
    q, s, z = synth.w3a16_weights(n, k, 128, True, seed=36, experts=e)
    off = np.array([0, 4, 4, 9])
    a = _a_bits(9, k, 37)
    _, got = G.grouped_w3a16_ref(a, off, q.numpy(), s.numpy(), z.numpy(), 128)
    for x in range(e):
        lo, hi = off[x], off[x + 1]
        if hi > lo:
            assert np.array_equal(got[lo:hi], G.w3a16_ref(a[lo:hi], q.numpy()[x], s.numpy()[x], z.numpy()[x], 128))


def test_w3a16_layout_is_a_bijection():
    for n, k, hz in ((128, 256, False), (200, 384, True)):
        nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
        word, bit = L.w3a16_code_bits(nn.ravel(), kk.ravel(), k, hz)
        slots = (word * 8 + bit).ravel()
        assert len(np.unique(slots)) == slots.size == 3 * n * k
        ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
        sb = L.w3a16_scale_byte(ng.ravel(), gg.ravel(), k, hz)
        code_bytes = set(np.unique(slots // 8).tolist())
        assert not code_bytes & set(sb.tolist()) and not code_bytes & set((sb + 1).tolist())
        if hz:
            zb = L.w3a16_zero_byte(ng.ravel(), gg.ravel(), k)
            assert not code_bytes & set(zb.tolist())
        if n % 128 == 0:   # full tiles: the code area is used completely
            assert len(code_bytes) == (n // 128) * (k // 128) * 6144


def test_w3a16_pack_unpack_roundtrip_and_padding():
    for hz in (False, True):
        q, s, z = synth.w3a16_weights(136, 256, 128, hz, seed=38)
        blob = L.w3a16_pack(q.numpy(), s.numpy(), None if z is None else z.numpy())
        assert blob.size == L.w3a16_packed_bytes(136, 256, hz)
        c2, s2, z2 = L.w3a16_unpack(blob, 136, 256, hz)
        assert np.array_equal(c2, F.int3_unpack_stream(q.numpy()))
        assert np.array_equal(s2.view(np.uint16), s.numpy().view(np.uint16))
        if hz:
            assert np.array_equal(z2, z.numpy())
        rec = L.w3a16_record_bytes(hz)
        tile1 = blob[2 * rec:].reshape(2, rec)
        assert np.all(tile1[:, :6144].reshape(2, 3, 128, 16)[:, :, 8:, :] == 0)


def test_w3a16_layout_small_hand_example():
    """Code (n=1, k=37): chunk 1, pair 2 (part 0, slot 2), odd half -> word
    q = 3 at byte (0*128 + 1)*16 + 12 = 28, bits 22..24.  Code (n=0, k=62):
    chunk 1, pair 15, even half -> bit 15 of words 3, 4, 5 at bytes 12,
    (1*128 + 0)*16 = 2048 and 2052."""
    word, bit = L.w3a16_code_bits(1, 37, 128, False)
    assert word.tolist() == [28, 28, 28] and bit.tolist() == [22, 23, 24]
    word, bit = L.w3a16_code_bits(0, 62, 128, False)
    assert word.tolist() == [12, 2048, 2052] and bit.tolist() == [15, 15, 15]
    assert int(L.w3a16_scale_byte(1, 0, 128, True)) == 6146
    assert int(L.w3a16_zero_byte(1, 0, 128)) == 6144 + 256 + 1


def test_w3a16_pairs_decode_as_bf16_128_plus_code():
    """The property the layout is built for: in each chunk, pairs 0..14 sit
    at bits 3j and 16 + 3j of their word (j = pair % 5), so a shift by 3j,
    the mask 0x00070007 and the bits of bf16 128.0 in both halves give the
    bf16 pair (128 + q_even, 128 + q_odd); pair 15 collects bit p of each
    code from bits 15 and 31 of the chunk's word p."""
    rng = np.random.default_rng(39)
    codes = rng.integers(0, 8, size=(128, 128)).astype(np.uint8)
    q = F.int3_pack_stream(codes)
    s = np.ones((128, 1), dtype=np.float16)
    blob = L.w3a16_pack(q, s, None)
    words = blob[:6144].view(np.uint32)
    for r in (0, 77, 127):
        rw = [int(words[(qq // 4 * 128 + r) * 4 + qq % 4]) for qq in range(12)]
        for c in range(4):
            w3 = rw[3 * c: 3 * c + 3]
            for i in range(16):
                if i < 15:
                    x = ((w3[i // 5] >> (3 * (i % 5))) & 0x00070007) | 0x43004300
                else:
                    x = 0x43004300
                    for p in range(3):
                        x |= ((w3[p] >> (15 - p)) & (0x00010001 << p))
                for h in range(2):
                    v = _bf16_exact((x >> (16 * h)) & 0xFFFF)
                    assert v == 128 + int(codes[r, 32 * c + 2 * i + h])
