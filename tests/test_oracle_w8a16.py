"""Pins for the oracle's INT8 (W8A16) container, dequantization, GEMM and
packed layout: a hand-built word and numpy's own little-endian byte view,
closed forms over every code and several zero points, exact rational brute
force, a reduction to a plain fp64 matmul, the grouped form against the
dense one, and the layout's bijection, round trip and hand example."""

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


def test_int8_words_hand_example_and_byte_view():
    codes = np.zeros((1, 8), dtype=np.uint8)
    codes[0, :5] = [0x01, 0xFE, 0x80, 0x7F, 0xAB]
    w = F.int8_pack_words(codes)
    assert w.view(np.uint32).tolist() == [[0x7F80FE01, 0x000000AB]]
    assert np.array_equal(F.int8_unpack_words(w), codes)
    # the container is the little-endian byte order of the words
    q, _, _ = synth.w8a16_weights(3, 128, 128, False, seed=60)
    assert np.array_equal(F.int8_unpack_words(q.numpy()), q.numpy().view(np.uint8).reshape(3, 128))


def test_w8a16_dequant_closed_form_every_code():
    codes = np.arange(256, dtype=np.int64).reshape(2, 128).astype(np.uint8)      # every code once
    q = F.int8_pack_words(codes)
    s = np.array([[0.125], [2.0]], dtype=np.float16)
    for z in (0, 1, 128, 255):
        zz = np.full((2, 1), z, dtype=np.uint8)
        assert np.array_equal(G.w8a16_dequant(q, s, zz, 128), (codes.astype(np.float64) - z) * s.astype(np.float64))
    assert np.array_equal(G.w8a16_dequant(q, s, None, 128), (codes.astype(np.float64) - 128) * s.astype(np.float64))


def test_w8a16_brute_force_in_rationals():
    m, n, k = 2, 3, 256
    q, s, z = synth.w8a16_weights(n, k, 128, True, seed=61)
    a = _a_bits(m, k, 62)
    got = G.w8a16_ref(a, q.numpy(), s.numpy(), z.numpy(), 128)
    for r in range(n):
        codes = [(int(w) & 0xFFFFFFFF) >> (8 * e) & 0xFF for w in q.numpy()[r].tolist() for e in range(4)]
        for i in range(m):
            acc = Fraction(0)
            for kk in range(k):
                g = kk // 128
                acc += _bf16_exact(a[i, kk]) * (codes[kk] - int(z.numpy()[r, g])) * Fraction(float(s.numpy()[r, g]))
            assert abs(got[i, r] - float(acc)) <= 1e-12 * max(1.0, abs(float(acc)))


def test_w8a16_unit_scale_zero_zero_is_plain_matmul():
    m, n, k = 5, 40, 384
    q, _, _ = synth.w8a16_weights(n, k, 128, False, seed=63)
    s = np.ones((n, k // 128), dtype=np.float16)
    z = np.zeros((n, k // 128), dtype=np.uint8)
    a = _a_bits(m, k, 64)
    got = G.w8a16_ref(a, q.numpy(), s, z, 128)
    w = torch.from_numpy(q.numpy().view(np.uint8).reshape(n, k).astype(np.float64))
    at = torch.from_numpy(a.astype(np.int32) << 16).view(torch.float32).double()
    assert np.array_equal(got, (at @ w.T).numpy())


def test_grouped_w8a16_equals_dense_per_expert():
    e, n, k = 3, 24, 128
    q, s, z = synth.w8a16_weights(n, k, 128, True, seed=65, experts=e)
    off = np.array([0, 4, 4, 11])
    a = _a_bits(11, k, 66)
    _, got = G.grouped_w8a16_ref(a, off, q.numpy(), s.numpy(), z.numpy(), 128)
    for x in range(e):
        lo, hi = off[x], off[x + 1]
        if hi > lo:
            assert np.array_equal(got[lo:hi], G.w8a16_ref(a[lo:hi], q.numpy()[x], s.numpy()[x], z.numpy()[x], 128))


def test_w8a16_layout_is_a_bijection():
    for n, k, hz in ((128, 256, False), (200, 384, True)):
        nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
        cb = L.w8a16_code_byte(nn.ravel(), kk.ravel(), k, hz)
        assert len(np.unique(cb)) == cb.size
        ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
        sb = L.w8a16_scale_byte(ng.ravel(), gg.ravel(), k, hz)
        assert not set(cb.tolist()) & (set(sb.tolist()) | set((sb + 1).tolist()))
        if hz:
            assert not set(cb.tolist()) & set(L.w8a16_zero_byte(ng.ravel(), gg.ravel(), k).tolist())


def test_w8a16_pack_unpack_roundtrip_and_padding():
    for hz in (False, True):
        q, s, z = synth.w8a16_weights(136, 256, 128, hz, seed=67)
        blob = L.w8a16_pack(q.numpy(), s.numpy(), None if z is None else z.numpy())
        assert blob.size == L.w8a16_packed_bytes(136, 256, hz)
        c2, s2, z2 = L.w8a16_unpack(blob, 136, 256, hz)
        assert np.array_equal(c2, F.int8_unpack_words(q.numpy()))
        assert np.array_equal(s2.view(np.uint16), s.numpy().view(np.uint16))
        if hz:
            assert np.array_equal(z2, z.numpy())
        rec = L.w8a16_record_bytes(hz)
        tile1 = blob[2 * rec:].reshape(2, rec)
        assert np.all(tile1[:, :16384].reshape(2, 8, 128, 16)[:, :, 8:, :] == 0)   # rows 136.. are padding


def test_w8a16_layout_small_hand_example():
    """Code (n=1, k=17): 16-K chunk 1, byte 1 of it -> (1*128 + 1)*16 + 1 =
    2065; code (n=130, k=200) of a K=256 blob: tile 1, block 1 (record 3),
    chunk 4, byte 8 -> 3*16640 + (4*128 + 2)*16 + 8."""
    assert int(L.w8a16_code_byte(1, 17, 128, False)) == 2065
    assert int(L.w8a16_code_byte(130, 200, 256, False)) == 3 * 16640 + (4 * 128 + 2) * 16 + 8
    assert int(L.w8a16_scale_byte(1, 0, 128, True)) == 16386
    assert int(L.w8a16_zero_byte(1, 0, 128)) == 16384 + 256 + 1
