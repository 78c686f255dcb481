"""Pins for the oracle's MXINT4 weights (two's-complement 4-bit integers
with an E8M0 scale per 32 K) with bf16 activations: the two's-complement
table typed by hand, closed forms over every code and many exponents, an
exact rational brute force, a unit-scale reduction to a plain fp64 matmul,
one-hot rows that read back each weight, the grouped form against the dense
one, and the packed layout's bijection, round trip and hand example."""

import struct
from fractions import Fraction

import numpy as np
import torch

from oracle import formats as F
from oracle import gemm as G
from oracle import layout as L
from quantized_gemm_bit_b200 import synth

TWOS = [0, 1, 2, 3, 4, 5, 6, 7, -8, -7, -6, -5, -4, -3, -2, -1]   # 4-bit two's complement, by hand


def _bf16_exact(bits):
    return Fraction(struct.unpack("<f", struct.pack("<I", int(bits) << 16))[0])


def _a_bits(m, k, seed):
    return synth.bf16_normal(m, k, seed).view(torch.int16).numpy().view(np.uint16)


def test_twos_complement_table():
    assert F.int4_twos_complement(np.arange(16)).tolist() == TWOS


def test_mxint4_dequant_closed_form_every_code_and_exponent():
    codes = np.tile(np.arange(16, dtype=np.uint8), 2)[None, :]            # [1, 32]: every code twice
    packed = F.fp4_pack_bytes(codes)
    for e in (0, 1, 100, 120, 127, 128, 200, 251):
        got = G.mxint4_dequant(packed, np.array([[e]], dtype=np.uint8))
        want = [Fraction(TWOS[c]) * Fraction(2) ** (e - 127) for c in codes[0].tolist()]
        assert [Fraction(v) for v in got[0].tolist()] == want


def test_mxint4_brute_force_in_rationals():
    m, n, k = 2, 3, 128
    codes, e8 = synth.mxint4_weights(n, k, seed=70)
    a = _a_bits(m, k, 71)
    got = G.mxint4_a16_ref(a, codes.numpy(), e8.numpy())
    cb = codes.numpy()
    for r in range(n):
        for i in range(m):
            acc = Fraction(0)
            for kk in range(k):
                byte = int(cb[r, kk // 2])
                c = (byte >> (4 * (kk % 2))) & 0xF
                acc += _bf16_exact(a[i, kk]) * TWOS[c] * Fraction(2) ** (int(e8.numpy()[r, kk // 32]) - 127)
            assert abs(got[i, r] - float(acc)) <= 1e-12 * max(1e-30, abs(float(acc)))


def test_mxint4_unit_scale_is_plain_matmul():
    m, n, k = 4, 24, 256
    codes, _ = synth.mxint4_weights(n, k, seed=72)
    e8 = np.full((n, k // 32), 127, dtype=np.uint8)
    a = _a_bits(m, k, 73)
    got = G.mxint4_a16_ref(a, codes.numpy(), e8)
    lo = torch.from_numpy(codes.numpy().astype(np.int64) & 0xF)
    hi = torch.from_numpy(codes.numpy().astype(np.int64) >> 4)
    table = torch.tensor(TWOS, dtype=torch.float64)
    w = torch.stack([table[lo], table[hi]], dim=2).reshape(n, k)
    at = torch.from_numpy(a.astype(np.int32) << 16).view(torch.float32).double()
    assert np.array_equal(got, (at @ w.T).numpy())


def test_mxint4_one_hot_rows_read_back_weights():
    n, k = 8, 64
    codes, e8 = synth.mxint4_weights(n, k, seed=74)
    one = np.uint16(0x3F80)                                  # bf16 1.0
    a = np.zeros((k, k), dtype=np.uint16)
    a[np.arange(k), np.arange(k)] = one
    got = G.mxint4_a16_ref(a, codes.numpy(), e8.numpy())
    assert np.array_equal(got.T, G.mxint4_dequant(codes.numpy(), e8.numpy()))


def test_grouped_mxint4_equals_dense_per_expert():
    e, n, k = 3, 16, 64
    codes, e8 = synth.mxint4_weights(n, k, seed=75, experts=e)
    off = np.array([0, 5, 5, 9])
    a = _a_bits(9, k, 76)
    _, got = G.grouped_mxint4_a16_ref(a, off, codes.numpy(), e8.numpy())
    for x in range(e):
        lo, hi = off[x], off[x + 1]
        if hi > lo:
            assert np.array_equal(got[lo:hi], G.mxint4_a16_ref(a[lo:hi], codes.numpy()[x], e8.numpy()[x]))


def test_mxi4_layout_bijection_roundtrip_and_hand_example():
    for n, k in ((128, 256), (200, 384)):
        nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
        byte, nib = L.mxi4_code_byte_and_nibble(nn.ravel(), kk.ravel(), k)
        slots = byte * 2 + nib
        assert len(np.unique(slots)) == slots.size
        ns, bs = np.meshgrid(np.arange(n), np.arange(k // 32), indexing="ij")
        sb = L.mxi4_scale_byte(ns.ravel(), bs.ravel(), k)
        assert len(np.unique(sb)) == sb.size and not set(byte.tolist()) & set(sb.tolist())
    codes, e8 = synth.mxint4_weights(136, 256, seed=77)
    blob = L.mxi4_pack(codes.numpy(), e8.numpy())
    assert blob.size == L.mxi4_packed_bytes(136, 256)
    c2, s2 = L.mxi4_unpack(blob, 136, 256)
    assert np.array_equal(c2, F.fp4_unpack_bytes(codes.numpy())) and np.array_equal(s2, e8.numpy())
    # code (n=1, k=45): chunk 1, word 1, element 5 -> nibble p = 6: byte
    # (1*128 + 1)*16 + 4 + 3, high nibble; scale of (n=1, 32-K block 5) in
    # record 1 of a K=256 row tile: 8704 + 8192 + 4 + 1
    b, h = L.mxi4_code_byte_and_nibble(1, 45, 128)
    assert (int(b), int(h)) == ((128 + 1) * 16 + 7, 0)
    assert int(L.mxi4_scale_byte(1, 5, 256)) == 8704 + 8192 + 4 + 1


def test_mxi4_pairs_decode_as_bf16_136_plus_integer():
    """The INT4 nibble placement: shifting word w of a chunk right by 4j,
    keeping 0x000F000F and flipping bit 3 of each nibble into bf16 128.0
    gives the bf16 pair (136 + c_even, 136 + c_odd) of the two's-complement
    integers c of codes 32c' + 8w + 2j and + 1."""
    rng = np.random.default_rng(78)
    codes = rng.integers(0, 16, size=(128, 128)).astype(np.uint8)
    blob = L.mxi4_pack(F.fp4_pack_bytes(codes), np.full((128, 4), 127, dtype=np.uint8))
    words = blob[:8192].view(np.uint32)
    for r in (0, 77, 127):
        for c in range(4):
            for w in range(4):
                word = int(words[(c * 128 + r) * 4 + w])
                for j in range(4):
                    x = ((word >> (4 * j)) & 0x000F000F) ^ 0x43084308
                    for h in range(2):
                        want = 136 + TWOS[int(codes[r, 32 * c + 8 * w + 2 * j + h])]
                        assert _bf16_exact((x >> (16 * h)) & 0xFFFF) == want
