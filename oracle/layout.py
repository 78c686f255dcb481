"""Packed (device) weight layouts, written as elementwise index formulas.
Test infrastructure only: the library's own packer must produce exactly
these bytes.

The pages say the library turns every format into one standard description
with the weight, scale and zero point described separately ("Humming:
open-source kernel library for quantized inference", summary, second
paragraph).  The concrete device layout is this library's own choice and is
specified here, one formula per field.

INT4 W4A16, layout version 1 (group size 128):
  NT = ceil(N / 128) tiles of 128 rows; KB = K / 128 blocks of 128 k.
  One record per (tile nt, block kb), records in (nt, kb) row-major order,
  record size REC = 8192 + 256 (+ 128 with zero points) bytes:
    codes  : byte (c*128 + r)*16 + w*4 + p//2, nibble p%2 (0 = low), where
             r = n - 128*nt, kk = k - 128*kb, c = kk // 32, w = (kk % 32)//8,
             e = kk % 8 and p = (e % 2)*4 + e // 2;
    scale  : fp16 bits, little endian, at byte 8192 + 2*r;
    zero   : uint8 at byte 8192 + 256 + r (only with zero points).
  Rows n >= N (tile padding) hold code 0, scale 0 and zero 0.
  Experts (MoE) are stored one after another, each NT*KB*REC bytes.

MXFP4 / NVFP4 for the block-scaled kernels, and MXFP4 for the W4A16
kernels (bf16 activations), follow further down, each with its formulas.
"""

import numpy as np

from . import formats as F

W4_TILE_N = 128
W4_BLOCK_K = 128


def w4a16_record_bytes(has_zero):
    return 8192 + 256 + (128 if has_zero else 0)


def w4a16_packed_bytes(n, k, has_zero, num_experts=1):
    nt = -(-n // W4_TILE_N)
    return num_experts * nt * (k // W4_BLOCK_K) * w4a16_record_bytes(has_zero)


def w4a16_code_byte_and_nibble(n, k, kdim, has_zero):
    """Elementwise formula: (byte offset in the expert blob, nibble 0/1) of
    code q[n, k].  Works on numpy arrays of indices."""
    n = np.asarray(n, dtype=np.int64)
    k = np.asarray(k, dtype=np.int64)
    kb_count = kdim // W4_BLOCK_K
    rec = w4a16_record_bytes(has_zero)
    nt, r = n // W4_TILE_N, n % W4_TILE_N
    kb, kk = k // W4_BLOCK_K, k % W4_BLOCK_K
    c, w, e = kk // 32, (kk % 32) // 8, kk % 8
    p = (e % 2) * 4 + e // 2
    byte = (nt * kb_count + kb) * rec + (c * 128 + r) * 16 + w * 4 + p // 2
    return byte, p % 2


def w4a16_scale_byte(n, kb, kdim, has_zero):
    n = np.asarray(n, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    rec = w4a16_record_bytes(has_zero)
    nt, r = n // W4_TILE_N, n % W4_TILE_N
    return (nt * (kdim // W4_BLOCK_K) + kb) * rec + 8192 + 2 * r


def w4a16_zero_byte(n, kb, kdim):
    n = np.asarray(n, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    rec = w4a16_record_bytes(True)
    nt, r = n // W4_TILE_N, n % W4_TILE_N
    return (nt * (kdim // W4_BLOCK_K) + kb) * rec + 8192 + 256 + r


def w4a16_pack(qweight, scales, zeros, group=128):
    """Canonical (int32 [N, K/8], fp16 [N, K/128], uint8 [N, K/128] | None)
    -> packed uint8 blob, by scattering every element to the position the
    formulas above give."""
    assert group == W4_BLOCK_K
    codes = F.int4_unpack_words(qweight)
    n, k = codes.shape
    has_zero = zeros is not None
    out = np.zeros(w4a16_packed_bytes(n, k, has_zero), dtype=np.uint8)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    byte, nib = w4a16_code_byte_and_nibble(nn.ravel(), kk.ravel(), k, has_zero)
    vals = codes.ravel().astype(np.uint8) << (4 * nib).astype(np.uint8)
    np.bitwise_or.at(out, byte, vals)
    sb = np.asarray(scales, dtype=np.float16).view(np.uint16)
    ng, gg = np.meshgrid(np.arange(n), np.arange(k // group), indexing="ij")
    off = w4a16_scale_byte(ng.ravel(), gg.ravel(), k, has_zero)
    out[off] = (sb.ravel() & 0xFF).astype(np.uint8)
    out[off + 1] = (sb.ravel() >> 8).astype(np.uint8)
    if has_zero:
        zo = w4a16_zero_byte(ng.ravel(), gg.ravel(), k)
        out[zo] = np.asarray(zeros, dtype=np.uint8).ravel()
    return out


def w4a16_unpack(blob, n, k, has_zero):
    """Inverse of w4a16_pack: packed blob -> (codes uint8 [N, K],
    scales fp16 [N, K/128], zeros uint8 [N, K/128] | None)."""
    blob = np.asarray(blob, dtype=np.uint8)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    byte, nib = w4a16_code_byte_and_nibble(nn.ravel(), kk.ravel(), k, has_zero)
    codes = ((blob[byte] >> (4 * nib).astype(np.uint8)) & 0xF).reshape(n, k)
    ng, gg = np.meshgrid(np.arange(n), np.arange(k // W4_BLOCK_K), indexing="ij")
    off = w4a16_scale_byte(ng.ravel(), gg.ravel(), k, has_zero)
    sbits = blob[off].astype(np.uint16) | (blob[off + 1].astype(np.uint16) << 8)
    scales = sbits.reshape(n, k // W4_BLOCK_K).view(np.float16)
    zeros = None
    if has_zero:
        zeros = blob[w4a16_zero_byte(ng.ravel(), gg.ravel(), k)].reshape(n, k // W4_BLOCK_K)
    return codes.astype(np.uint8), scales, zeros


# ---------------------------------------------------------------------------
# MXFP4 / NVFP4, layout version 1
#   codes  : [NP][K/2] bytes, row major, even k low nibble (NP = N rounded up
#            to 128, extra rows zero)
#   scales : from byte NP*K/2; per (tile nt, group g of 4 scale blocks) a
#            512-byte block in (nt, g) order; scale of row n, block b sits at
#            block (nt = n//128, g = b//4), byte (n%32)*16 + ((n%128)//32)*4 + b%4
#   NVFP4 adds a 16-byte tail holding the fp32 tensor scale.
# ---------------------------------------------------------------------------


def fp4_packed_bytes(n, k, block, with_tail):
    np_ = -(-n // 128) * 128
    nt = np_ // 128
    groups = (k // block) // 4
    return np_ * k // 2 + nt * groups * 512 + (16 if with_tail else 0)


def fp4_scale_byte_np(n, b, k, block, np_rows):
    n = np.asarray(n, dtype=np.int64)
    b = np.asarray(b, dtype=np.int64)
    groups = (k // block) // 4
    nt, g = n // 128, b // 4
    return (np_rows * k // 2 + (nt * groups + g) * 512 + (n % 32) * 16 + ((n % 128) // 32) * 4 + b % 4)


def fp4_pack(codes_packed, scales, block, global_scale=None):
    """Canonical (uint8 [N, K/2], uint8 [N, K/block]) -> packed blob."""
    codes_packed = np.asarray(codes_packed, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    n, kh = codes_packed.shape
    k = kh * 2
    np_rows = -(-n // 128) * 128
    out = np.zeros(fp4_packed_bytes(n, k, block, global_scale is not None), dtype=np.uint8)
    out[: n * kh] = codes_packed.ravel()
    nn, bb = np.meshgrid(np.arange(n), np.arange(k // block), indexing="ij")
    out[fp4_scale_byte_np(nn.ravel(), bb.ravel(), k, block, np_rows)] = scales.ravel()
    if global_scale is not None:
        out[-16:-12] = np.frombuffer(np.float32(global_scale).tobytes(), dtype=np.uint8)
    return out


# ---------------------------------------------------------------------------
# MXFP4 weights for bf16 activations (W4A16 kernels), layout version 1
#   Records as for INT4: one per (tile nt of 128 rows, block kb of 128 K), in
#   (nt, kb) order, experts one after another; record size 8192 + 512 bytes.
#   codes : the 32-bit little-endian word at byte (c*128 + r)*16 + 4*w of the
#           record holds the 8 codes kk = 32c + 8w + 2j + h (j < 4, h < 2),
#           where r = n - 128*nt and kk = k - 128*kb.  Bit b of code
#           (b = 0 mantissa, 1 and 2 exponent, 3 sign) sits at word bit
#           MXA16_BITS[j][h][b].
#   scales: the E8M0 byte of row n, 32-K block 4*kb + c at byte 8192 + 4*r + c.
#   Rows n >= N (tile padding) hold code 0 and scale byte 0.
# ---------------------------------------------------------------------------

MXA16_REC = 8192 + 512

# [pair j][half h] -> word bit of (mantissa, exponent bit 0, exponent bit 1, sign)
MXA16_BITS = (
    ((6, 7, 8, 15), (22, 23, 24, 31)),
    ((10, 11, 12, 19), (26, 27, 28, 3)),
    ((16, 17, 18, 25), (0, 1, 2, 9)),
    ((4, 5, 14, 13), (20, 21, 30, 29)),
)


def mxa16_packed_bytes(n, k, num_experts=1):
    return num_experts * (-(-n // 128)) * (k // 128) * MXA16_REC


def mxa16_code_word_and_bits(n, k, kdim):
    """Elementwise formula: (byte offset of the 32-bit word in the expert
    blob, [4] word bits of code bits 0..3) for code (n, k)."""
    n = np.asarray(n, dtype=np.int64)
    k = np.asarray(k, dtype=np.int64)
    nt, r = n // 128, n % 128
    kb, kk = k // 128, k % 128
    c, w, j, h = kk // 32, (kk % 32) // 8, (kk % 8) // 2, kk % 2
    word = (nt * (kdim // 128) + kb) * MXA16_REC + (c * 128 + r) * 16 + 4 * w
    table = np.asarray(MXA16_BITS, dtype=np.int64)        # [4, 2, 4]
    return word, table[j, h]


def mxa16_scale_byte(n, blk, kdim):
    n = np.asarray(n, dtype=np.int64)
    blk = np.asarray(blk, dtype=np.int64)
    nt, r = n // 128, n % 128
    kb, c = blk // 4, blk % 4
    return (nt * (kdim // 128) + kb) * MXA16_REC + 8192 + 4 * r + c


def mxa16_pack(codes_packed, scales):
    """Canonical (uint8 [N, K/2] even k low nibble, uint8 E8M0 [N, K/32])
    -> packed blob of one expert, by placing every code bit and every scale
    byte where the formulas above say."""
    codes = F.fp4_unpack_bytes(np.asarray(codes_packed, dtype=np.uint8)).astype(np.uint32)
    n, k = codes.shape
    out = np.zeros(mxa16_packed_bytes(n, k), dtype=np.uint8)
    words = np.zeros(out.size // 4, dtype=np.uint32)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    word, bits = mxa16_code_word_and_bits(nn.ravel(), kk.ravel(), k)
    c = codes.ravel()
    for b in range(4):
        np.bitwise_or.at(words, word // 4, ((c >> b) & 1) << bits[:, b].astype(np.uint32))
    out[:] = words.view(np.uint8)                          # little endian words
    ns, bs = np.meshgrid(np.arange(n), np.arange(k // 32), indexing="ij")
    out[mxa16_scale_byte(ns.ravel(), bs.ravel(), k)] = np.asarray(scales, dtype=np.uint8).ravel()
    return out


def mxa16_unpack(blob, n, k):
    """Inverse of mxa16_pack: blob -> (codes uint8 [N, K], scales uint8 [N, K/32])."""
    words = np.asarray(blob, dtype=np.uint8).view(np.uint32)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    word, bits = mxa16_code_word_and_bits(nn.ravel(), kk.ravel(), k)
    wv = words[word // 4]
    codes = np.zeros(n * k, dtype=np.uint32)
    for b in range(4):
        codes |= ((wv >> bits[:, b].astype(np.uint32)) & 1) << b
    ns, bs = np.meshgrid(np.arange(n), np.arange(k // 32), indexing="ij")
    scales = np.asarray(blob, dtype=np.uint8)[mxa16_scale_byte(ns.ravel(), bs.ravel(), k)]
    return codes.reshape(n, k).astype(np.uint8), scales.reshape(n, k // 32)


# ---------------------------------------------------------------------------
# INT3 W3A16 (group 128), layout version 1
#   Records as for INT4: one per (tile nt of 128 rows, block kb of 128 K), in
#   (nt, kb) order, experts one after another; record size
#   6144 + 256 (+ 128 with zero points) bytes.
#   codes : row r's 12 code words; word q (q = 3c + p: 32-K chunk c, part
#           p < 3) is the 32-bit little-endian word at byte
#           (q // 4 * 128 + r) * 16 + 4 * (q % 4).  Code kk = k - 128*kb of
#           chunk c = kk // 32, pair i = (kk % 32) // 2, half h = kk % 2:
#             i < 15: word 3c + i // 5, code bit b at bit 3*(i % 5) + b + 16*h;
#             i = 15: code bit b in word 3c + b, at bit 15 + 16*h.
#   scale : fp16 bits at byte 6144 + 2*r;  zero: uint8 at 6144 + 256 + r.
#   Rows n >= N (tile padding) hold code 0, scale 0 and zero 0.
# ---------------------------------------------------------------------------


def w3a16_record_bytes(has_zero):
    return 6144 + 256 + (128 if has_zero else 0)


def w3a16_packed_bytes(n, k, has_zero, num_experts=1):
    return num_experts * (-(-n // 128)) * (k // 128) * w3a16_record_bytes(has_zero)


def w3a16_code_bits(n, k, kdim, has_zero):
    """Elementwise formula: ([.., 3] byte offsets of the words holding code
    bits 0..2 of code (n, k) in the expert blob, [.., 3] bit positions)."""
    n = np.asarray(n, dtype=np.int64)
    k = np.asarray(k, dtype=np.int64)
    rec = w3a16_record_bytes(has_zero)
    nt, r = n // 128, n % 128
    kb, kk = k // 128, k % 128
    c, i, h = kk // 32, (kk % 32) // 2, kk % 2
    b = np.arange(3, dtype=np.int64)
    last = (i == 15)[..., None]
    q = np.where(last, 3 * c[..., None] + b, (3 * c + np.minimum(i, 14) // 5)[..., None] + 0 * b)
    bit = np.where(last, 15 + 16 * h[..., None] + 0 * b, (3 * (np.minimum(i, 14) % 5) + 16 * h)[..., None] + b)
    base = ((nt * (kdim // 128) + kb) * rec)[..., None]
    word = base + (q // 4 * 128 + r[..., None]) * 16 + 4 * (q % 4)
    return word, bit


def w3a16_scale_byte(n, kb, kdim, has_zero):
    n = np.asarray(n, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    nt, r = n // 128, n % 128
    return (nt * (kdim // 128) + kb) * w3a16_record_bytes(has_zero) + 6144 + 2 * r


def w3a16_zero_byte(n, kb, kdim):
    n = np.asarray(n, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    nt, r = n // 128, n % 128
    return (nt * (kdim // 128) + kb) * w3a16_record_bytes(True) + 6144 + 256 + r


def w3a16_pack(qweight, scales, zeros, group=128):
    """Canonical (int32 [N, 3K/32] bit streams, fp16 [N, K/128], uint8
    [N, K/128] | None) -> packed blob of one expert, every code bit, scale
    and zero point placed where the formulas above say."""
    assert group == 128
    codes = F.int3_unpack_stream(qweight).astype(np.uint32)
    n, k = codes.shape
    has_zero = zeros is not None
    out = np.zeros(w3a16_packed_bytes(n, k, has_zero), dtype=np.uint8)
    words = np.zeros(out.size // 4, dtype=np.uint32)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    word, bit = w3a16_code_bits(nn.ravel(), kk.ravel(), k, has_zero)
    c = codes.ravel()
    for b in range(3):
        np.bitwise_or.at(words, word[:, b] // 4, ((c >> b) & 1) << bit[:, b].astype(np.uint32))
    out[:] = words.view(np.uint8)
    sb = np.asarray(scales, dtype=np.float16).view(np.uint16)
    ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
    off = w3a16_scale_byte(ng.ravel(), gg.ravel(), k, has_zero)
    out[off] = (sb.ravel() & 0xFF).astype(np.uint8)
    out[off + 1] = (sb.ravel() >> 8).astype(np.uint8)
    if has_zero:
        out[w3a16_zero_byte(ng.ravel(), gg.ravel(), k)] = np.asarray(zeros, dtype=np.uint8).ravel()
    return out


def w3a16_unpack(blob, n, k, has_zero):
    """Inverse of w3a16_pack: blob -> (codes uint8 [N, K], scales fp16
    [N, K/128], zeros uint8 [N, K/128] | None)."""
    blob = np.asarray(blob, dtype=np.uint8)
    words = blob.view(np.uint32)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    word, bit = w3a16_code_bits(nn.ravel(), kk.ravel(), k, has_zero)
    codes = np.zeros(n * k, dtype=np.uint32)
    for b in range(3):
        codes |= ((words[word[:, b] // 4] >> bit[:, b].astype(np.uint32)) & 1) << b
    ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
    off = w3a16_scale_byte(ng.ravel(), gg.ravel(), k, has_zero)
    sbits = blob[off].astype(np.uint16) | (blob[off + 1].astype(np.uint16) << 8)
    zeros = blob[w3a16_zero_byte(ng.ravel(), gg.ravel(), k)].reshape(n, k // 128) if has_zero else None
    return codes.reshape(n, k).astype(np.uint8), sbits.reshape(n, k // 128).view(np.float16), zeros


# ---------------------------------------------------------------------------
# INT2 W2A16 (group 128), layout version 1
#   Records as for INT4: one per (tile nt of 128 rows, block kb of 128 K), in
#   (nt, kb) order, experts one after another; record size
#   4096 + 256 (+ 128 with zero points) bytes.
#   codes : row r's 8 code words; word q (q = 2c + p: 32-K chunk c, part
#           p < 2) is the 32-bit little-endian word at byte
#           (q // 4 * 128 + r) * 16 + 4 * (q % 4).  Code kk = k - 128*kb of
#           chunk c = kk // 32, pair i = (kk % 32) // 2, half h = kk % 2
#           sits in word 2c + i // 8 at bits 2*(i % 8) + 16*h .. +1.
#   scale : fp16 bits at byte 4096 + 2*r;  zero: uint8 at 4096 + 256 + r.
#   Rows n >= N (tile padding) hold code 0, scale 0 and zero 0.
# ---------------------------------------------------------------------------


def w2a16_record_bytes(has_zero):
    return 4096 + 256 + (128 if has_zero else 0)


def w2a16_packed_bytes(n, k, has_zero, num_experts=1):
    return num_experts * (-(-n // 128)) * (k // 128) * w2a16_record_bytes(has_zero)


def w2a16_code_word_and_bit(n, k, kdim, has_zero):
    """Elementwise formula: (byte offset of the word holding code (n, k) in
    the expert blob, bit position of its low bit)."""
    n = np.asarray(n, dtype=np.int64)
    k = np.asarray(k, dtype=np.int64)
    nt, r = n // 128, n % 128
    kb, kk = k // 128, k % 128
    c, i, h = kk // 32, (kk % 32) // 2, kk % 2
    q = 2 * c + i // 8
    word = (nt * (kdim // 128) + kb) * w2a16_record_bytes(has_zero) + (q // 4 * 128 + r) * 16 + 4 * (q % 4)
    return word, 2 * (i % 8) + 16 * h


def w2a16_scale_byte(n, kb, kdim, has_zero):
    n = np.asarray(n, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    nt, r = n // 128, n % 128
    return (nt * (kdim // 128) + kb) * w2a16_record_bytes(has_zero) + 4096 + 2 * r


def w2a16_zero_byte(n, kb, kdim):
    n = np.asarray(n, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    nt, r = n // 128, n % 128
    return (nt * (kdim // 128) + kb) * w2a16_record_bytes(True) + 4096 + 256 + r


def w2a16_pack(qweight, scales, zeros, group=128):
    """Canonical (int32 [N, K/16], fp16 [N, K/128], uint8 [N, K/128] | None)
    -> packed blob of one expert, placed by the formulas above."""
    assert group == 128
    codes = F.int2_unpack_words(qweight).astype(np.uint32)
    n, k = codes.shape
    has_zero = zeros is not None
    out = np.zeros(w2a16_packed_bytes(n, k, has_zero), dtype=np.uint8)
    words = np.zeros(out.size // 4, dtype=np.uint32)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    word, bit = w2a16_code_word_and_bit(nn.ravel(), kk.ravel(), k, has_zero)
    np.bitwise_or.at(words, word // 4, codes.ravel() << bit.astype(np.uint32))
    out[:] = words.view(np.uint8)
    sb = np.asarray(scales, dtype=np.float16).view(np.uint16)
    ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
    off = w2a16_scale_byte(ng.ravel(), gg.ravel(), k, has_zero)
    out[off] = (sb.ravel() & 0xFF).astype(np.uint8)
    out[off + 1] = (sb.ravel() >> 8).astype(np.uint8)
    if has_zero:
        out[w2a16_zero_byte(ng.ravel(), gg.ravel(), k)] = np.asarray(zeros, dtype=np.uint8).ravel()
    return out


def w2a16_unpack(blob, n, k, has_zero):
    """Inverse of w2a16_pack -> (codes uint8 [N, K], scales fp16 [N, K/128],
    zeros uint8 [N, K/128] | None)."""
    blob = np.asarray(blob, dtype=np.uint8)
    words = blob.view(np.uint32)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    word, bit = w2a16_code_word_and_bit(nn.ravel(), kk.ravel(), k, has_zero)
    codes = (words[word // 4] >> bit.astype(np.uint32)) & 3
    ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
    off = w2a16_scale_byte(ng.ravel(), gg.ravel(), k, has_zero)
    sbits = blob[off].astype(np.uint16) | (blob[off + 1].astype(np.uint16) << 8)
    zeros = blob[w2a16_zero_byte(ng.ravel(), gg.ravel(), k)].reshape(n, k // 128) if has_zero else None
    return codes.reshape(n, k).astype(np.uint8), sbits.reshape(n, k // 128).view(np.float16), zeros


# ---------------------------------------------------------------------------
# Gated gate+up row order (for the GEMM with the SwiGLU epilogue), any of the
# W4A16-family layouts above.  The canonical weights have N = 2I rows, gate
# rows [0, I) and up rows [I, 2I).  Packed row p (tile j = p // 128, row
# r = p % 128 of it, quarter q = r // 32, lane l = r % 32) holds canonical
# row
#     64 j + 16 q + l            for l < 16   (gate), and
#     I + 64 j + 16 q + l - 16   for l >= 16  (up, the same feature),
# so a 128-row tile covers features [64 j, 64 j + 64) of both projections.
# The blob is the format's packed layout of the rows in this order.
# ---------------------------------------------------------------------------


def gated_source_rows(n):
    """[n] int64: canonical row of every packed row p (n % 128 == 0)."""
    assert n % 128 == 0
    p = np.arange(n, dtype=np.int64)
    j, r = p // 128, p % 128
    q, lane = r // 32, r % 32
    return np.where(lane < 16, 64 * j + 16 * q + lane, n // 2 + 64 * j + 16 * q + lane - 16)


# ---------------------------------------------------------------------------
# INT8 W8A16 (group 128), layout version 1
#   Records as for INT4: one per (tile nt of 128 rows, block kb of 128 K), in
#   (nt, kb) order, experts one after another; record size
#   16384 + 256 (+ 128 with zero points) bytes.
#   codes : code kk = k - 128*kb of row r at byte (kk // 16 * 128 + r) * 16
#           + kk % 16 (row r's 16-K chunk c is 16 contiguous bytes, the
#           chunks of 128 rows are 2 KB apart: conflict-free 16-byte reads);
#   scale : fp16 bits at byte 16384 + 2*r;  zero: uint8 at 16384 + 256 + r.
#   Rows n >= N (tile padding) hold code 0, scale 0 and zero 0.
# ---------------------------------------------------------------------------


def w8a16_record_bytes(has_zero):
    return 16384 + 256 + (128 if has_zero else 0)


def w8a16_packed_bytes(n, k, has_zero, num_experts=1):
    return num_experts * (-(-n // 128)) * (k // 128) * w8a16_record_bytes(has_zero)


def w8a16_code_byte(n, k, kdim, has_zero):
    """Elementwise formula: byte offset of code (n, k) in the expert blob."""
    n = np.asarray(n, dtype=np.int64)
    k = np.asarray(k, dtype=np.int64)
    nt, r = n // 128, n % 128
    kb, kk = k // 128, k % 128
    return (nt * (kdim // 128) + kb) * w8a16_record_bytes(has_zero) + (kk // 16 * 128 + r) * 16 + kk % 16


def w8a16_scale_byte(n, kb, kdim, has_zero):
    n = np.asarray(n, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    nt, r = n // 128, n % 128
    return (nt * (kdim // 128) + kb) * w8a16_record_bytes(has_zero) + 16384 + 2 * r


def w8a16_zero_byte(n, kb, kdim):
    n = np.asarray(n, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    nt, r = n // 128, n % 128
    return (nt * (kdim // 128) + kb) * w8a16_record_bytes(True) + 16384 + 256 + r


def w8a16_pack(qweight, scales, zeros, group=128):
    """Canonical (int32 [N, K/4], fp16 [N, K/128], uint8 [N, K/128] | None)
    -> packed blob of one expert, placed by the formulas above."""
    assert group == 128
    codes = F.int8_unpack_words(qweight)
    n, k = codes.shape
    has_zero = zeros is not None
    out = np.zeros(w8a16_packed_bytes(n, k, has_zero), dtype=np.uint8)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    out[w8a16_code_byte(nn.ravel(), kk.ravel(), k, has_zero)] = codes.ravel()
    sb = np.asarray(scales, dtype=np.float16).view(np.uint16)
    ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
    off = w8a16_scale_byte(ng.ravel(), gg.ravel(), k, has_zero)
    out[off] = (sb.ravel() & 0xFF).astype(np.uint8)
    out[off + 1] = (sb.ravel() >> 8).astype(np.uint8)
    if has_zero:
        out[w8a16_zero_byte(ng.ravel(), gg.ravel(), k)] = np.asarray(zeros, dtype=np.uint8).ravel()
    return out


def w8a16_unpack(blob, n, k, has_zero):
    """Inverse of w8a16_pack -> (codes uint8 [N, K], scales fp16 [N, K/128],
    zeros uint8 [N, K/128] | None)."""
    blob = np.asarray(blob, dtype=np.uint8)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    codes = blob[w8a16_code_byte(nn.ravel(), kk.ravel(), k, has_zero)]
    ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
    off = w8a16_scale_byte(ng.ravel(), gg.ravel(), k, has_zero)
    sbits = blob[off].astype(np.uint16) | (blob[off + 1].astype(np.uint16) << 8)
    zeros = blob[w8a16_zero_byte(ng.ravel(), gg.ravel(), k)].reshape(n, k // 128) if has_zero else None
    return codes.reshape(n, k), sbits.reshape(n, k // 128).view(np.float16), zeros


# ---------------------------------------------------------------------------
# MXINT4 for bf16 activations, layout version 1
#   Records as for MXFP4_A16: one per (tile nt, block kb), experts one after
#   another, 8192 + 512 bytes each.
#   codes : the 4-bit code (two's complement) of (n, k) where the INT4
#           layout puts its code (w4a16_code_byte_and_nibble);
#   scale : E8M0 byte of row r, 32-K block c of the record at 8192 + 4r + c.
# ---------------------------------------------------------------------------

MXI4_REC = 8192 + 512


def mxi4_packed_bytes(n, k, num_experts=1):
    return num_experts * (-(-n // 128)) * (k // 128) * MXI4_REC


def mxi4_code_byte_and_nibble(n, k, kdim):
    n = np.asarray(n, dtype=np.int64)
    k = np.asarray(k, dtype=np.int64)
    nt, r = n // 128, n % 128
    kb, kk = k // 128, k % 128
    c, w, e = kk // 32, (kk % 32) // 8, kk % 8
    p = (e % 2) * 4 + e // 2
    return (nt * (kdim // 128) + kb) * MXI4_REC + (c * 128 + r) * 16 + w * 4 + p // 2, p % 2


def mxi4_scale_byte(n, blk, kdim):
    n = np.asarray(n, dtype=np.int64)
    blk = np.asarray(blk, dtype=np.int64)
    nt, r = n // 128, n % 128
    kb, c = blk // 4, blk % 4
    return (nt * (kdim // 128) + kb) * MXI4_REC + 8192 + 4 * r + c


def mxi4_pack(codes_packed, scales):
    """Canonical (uint8 [N, K/2] even k low nibble, uint8 E8M0 [N, K/32])
    -> packed blob of one expert, placed by the formulas above."""
    codes = F.fp4_unpack_bytes(np.asarray(codes_packed, dtype=np.uint8))
    n, k = codes.shape
    out = np.zeros(mxi4_packed_bytes(n, k), dtype=np.uint8)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    byte, nib = mxi4_code_byte_and_nibble(nn.ravel(), kk.ravel(), k)
    np.bitwise_or.at(out, byte, (codes.ravel() << (4 * nib)).astype(np.uint8))
    ns, bs = np.meshgrid(np.arange(n), np.arange(k // 32), indexing="ij")
    out[mxi4_scale_byte(ns.ravel(), bs.ravel(), k)] = np.asarray(scales, dtype=np.uint8).ravel()
    return out


def mxi4_unpack(blob, n, k):
    """Inverse of mxi4_pack: blob -> (codes uint8 [N, K], scales uint8 [N, K/32])."""
    blob = np.asarray(blob, dtype=np.uint8)
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    byte, nib = mxi4_code_byte_and_nibble(nn.ravel(), kk.ravel(), k)
    codes = (blob[byte] >> (4 * nib)) & 0xF
    ns, bs = np.meshgrid(np.arange(n), np.arange(k // 32), indexing="ij")
    return codes.reshape(n, k).astype(np.uint8), blob[mxi4_scale_byte(ns.ravel(), bs.ravel(), k)].reshape(n, k // 32)
