"""Pins for the oracle's MXFP4-weight x bf16-activation GEMM and its packed
layout: brute force in exact rationals, one-hot activations against the OCP
value table, the grouped form against the dense form, and the layout's
bijection, round trip, a hand example and its bf16 decoding property."""

import struct
from fractions import Fraction

import numpy as np
import torch

from oracle import formats as F
from oracle import gemm as G
from oracle import layout as L
from quantized_gemm_bit_b200 import synth

# OCP MX v1.0 FP4 (E2M1) magnitudes of codes 0..7; bit 3 is the sign
E2M1 = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _bf16_exact(bits):
    """bf16 bit pattern -> exact Fraction (through the fp32 with the same
    upper half, via struct)."""
    return Fraction(struct.unpack("<f", struct.pack("<I", int(bits) << 16))[0])


def _e2m1_exact(code):
    v = Fraction(E2M1[code & 7]).limit_denominator(2)
    return -v if code & 8 else v


def _a_bits(m, k, seed):
    return synth.bf16_normal(m, k, seed).view(torch.int16).numpy().view(np.uint16)


def test_mxfp4_a16_brute_force_in_rationals():
    m, n, k = 3, 5, 96
    rng = np.random.default_rng(91)
    codes = rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    e8 = rng.integers(110, 140, size=(n, k // 32), dtype=np.uint8)
    a = _a_bits(m, k, 92)
    got = G.mxfp4_a16_ref(a, codes, e8)
    for i in range(m):
        for j in range(n):
            acc = Fraction(0)
            for kk in range(k):
                byte = int(codes[j, kk // 2])
                code = byte & 0xF if kk % 2 == 0 else byte >> 4
                scale = Fraction(2) ** (int(e8[j, kk // 32]) - 127)
                acc += _bf16_exact(a[i, kk]) * _e2m1_exact(code) * scale
            assert abs(got[i, j] - float(acc)) <= 1e-12 * max(1.0, abs(float(acc)))


def test_mxfp4_a16_one_hot_rows_read_back_the_weights():
    """A row that is 1 at k and 0 elsewhere returns column k of W_hat, which
    must be the OCP value of the code times 2^(e - 127)."""
    n, k = 7, 64
    rng = np.random.default_rng(93)
    codes = rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    e8 = rng.integers(0, 253, size=(n, k // 32), dtype=np.uint8)
    one = 0x3F80                                               # bf16 1.0
    a = np.zeros((k, k), dtype=np.uint16)
    a[np.arange(k), np.arange(k)] = one
    got = G.mxfp4_a16_ref(a, codes, e8)                        # [k, n]
    for kk in range(k):
        for j in range(n):
            byte = int(codes[j, kk // 2])
            code = byte & 0xF if kk % 2 == 0 else byte >> 4
            want = (-1.0 if code & 8 else 1.0) * E2M1[code & 7] * 2.0 ** (int(e8[j, kk // 32]) - 127)
            assert got[kk, j] == want


def test_grouped_mxfp4_a16_equals_dense_per_expert():
    e, n, k = 4, 40, 128
    rng = np.random.default_rng(94)
    codes = rng.integers(0, 256, size=(e, n, k // 2), dtype=np.uint8)
    e8 = rng.integers(118, 126, size=(e, n, k // 32), dtype=np.uint8)
    off = np.array([0, 3, 3, 10, 17])                           # expert 1 empty
    a = _a_bits(17, k, 95)
    rows, got = G.grouped_mxfp4_a16_ref(a, off, codes, e8)
    assert np.array_equal(rows, np.arange(17))
    for x in range(e):
        lo, hi = off[x], off[x + 1]
        if hi > lo:
            assert np.array_equal(got[lo:hi], G.mxfp4_a16_ref(a[lo:hi], codes[x], e8[x]))


def test_mxa16_layout_is_a_bijection():
    n, k = 256, 256
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    word, bits = L.mxa16_code_word_and_bits(nn.ravel(), kk.ravel(), k)
    slots = (word[:, None] * 8 + bits).ravel()                  # bit index in the blob
    assert len(np.unique(slots)) == slots.size == 4 * n * k
    total = L.mxa16_packed_bytes(n, k)
    ns, bs = np.meshgrid(np.arange(n), np.arange(k // 32), indexing="ij")
    sb = L.mxa16_scale_byte(ns.ravel(), bs.ravel(), k)
    assert len(np.unique(sb)) == sb.size
    code_bytes = np.unique(slots // 8)
    assert not set(code_bytes.tolist()) & set(sb.tolist())
    assert code_bytes.size + sb.size == total                   # every byte used once


def test_mxa16_pack_unpack_roundtrip_and_padding():
    n, k = 136, 256
    codes, e8 = synth.mxfp4_weights(n, k, seed=96)
    blob = L.mxa16_pack(codes.numpy(), e8.numpy())
    assert blob.size == L.mxa16_packed_bytes(n, k)
    c2, s2 = L.mxa16_unpack(blob, n, k)
    assert np.array_equal(c2, F.fp4_unpack_bytes(codes.numpy()))
    assert np.array_equal(s2, e8.numpy())
    tile1 = blob[2 * L.MXA16_REC:].reshape(2, L.MXA16_REC)
    assert np.all(tile1[:, :8192].reshape(2, 4, 128, 16)[:, :, 8:, :] == 0)
    assert np.all(tile1[:, 8192:].reshape(2, 128, 4)[:, 8:, :] == 0)


def test_mxa16_layout_small_hand_example():
    """Code (n=1, k=37): chunk 1, word 0, pair 2, odd half -> word at byte
    (1*128 + 1)*16 = 2064, sign at bit 9; its scale (block 1) at 8192 + 4 + 1."""
    word, bits = L.mxa16_code_word_and_bits(1, 37, 128)
    assert int(word) == 2064 and tuple(int(b) for b in bits) == (0, 1, 2, 9)
    assert int(L.mxa16_scale_byte(1, 1, 128)) == 8197
    # k = 128 + 7 of row 129 (tile 1, record kb=1): pair 3, odd half
    word, bits = L.mxa16_code_word_and_bits(129, 135, 256)
    assert int(word) == (1 * 2 + 1) * L.MXA16_REC + (0 * 128 + 1) * 16
    assert tuple(int(b) for b in bits) == (20, 21, 30, 29)


def _rotr(x, n):
    return ((x >> n) | (x << (32 - n))) & 0xFFFFFFFF if n else x


def test_mxa16_pairs_decode_as_bf16_after_fixed_rotations():
    """The property the layout is built for: after rotating the word right
    by 0, 4 or 10 bits (pairs 0-2), or taking the mantissa, exponent bit 0
    and sign of pair 3 from a left rotation by 2 and its exponent bit 1
    from a right rotation by 6, each pair's two codes sit in a bf16x2 word
    (low half: even k) with the sign at bit 15, the exponent bits at 8..7
    and the mantissa bit at 6, i.e. the bf16 values e2m1(c) * 2^-126."""
    mask = 0x81C081C0
    for j in range(4):
        for c0 in range(16):
            for c1 in range(16):
                w = 0
                for h, c in ((0, c0), (1, c1)):
                    for b in range(4):
                        if (c >> b) & 1:
                            w |= 1 << L.MXA16_BITS[j][h][b]
                if j < 3:
                    x = _rotr(w, (0, 4, 10)[j]) & mask
                else:
                    x = (_rotr(w, 30) & 0x80C080C0) | (_rotr(w, 6) & 0x01000100)
                for h, c in ((0, c0), (1, c1)):
                    half = (x >> (16 * h)) & 0xFFFF
                    assert _bf16_exact(half) * Fraction(2) ** 126 == _e2m1_exact(c), (j, h, c)
