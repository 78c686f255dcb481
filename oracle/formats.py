"""Element formats: decoders (code -> exact value) and round-to-nearest-even
quantizers, in numpy, for the oracle.  Test infrastructure only.

Formats (the pages only name them; meanings from the public standards):
  * INT4 (unsigned code 0..15) with group scale / zero point:
    "Humming: open-source kernel library for quantized inference", summary,
    second paragraph (weight, scale and zero point described separately).
  * INT3 (unsigned code 0..7, GPTQ INT3 weights: the Vietnamese edition
    of the Humming news, section "meaning for domestic deployers"), with
    the same group scale / zero point.
  * INT2 (unsigned code 0..3; INT1..INT8 weights are listed on the same
    page, section "one library, many formats"), with the same group scale
    / zero point.
  * e2m1 (FP4): OCP MX v1.0, section 5.3.3 "FP4 (E2M1)": 1 sign bit,
    2 exponent bits with bias 1, 1 mantissa bit, no inf/NaN, max 6.0.
  * E8M0 scale: OCP MX v1.0, section 5.4 "E8M0": value 2**(e-127), 0xFF NaN.
  * E4M3 "fn": OCP 8-bit Floating Point spec, E4M3 column: bias 7,
    subnormals, max normal 448, no infinities, NaN = S.1111.111.
  * bf16 and fp16 are IEEE-style; decoded exactly to fp64.

Quantizers decide integer codes, so they run in the precision the kernels
would use for the same decision (fp32 inputs, fp32 divisions), then round to
nearest, ties to even mantissa, exactly (the rounding step itself is done in
fp64 where every operation below is exact).
"""

import numpy as np

# ---------------------------------------------------------------------------
# bf16 / fp16 helpers (exact)
# ---------------------------------------------------------------------------


def bf16_bits_to_f64(bits):
    """bf16 bit patterns (uint16) -> exact fp64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f32_to_bf16_bits_rne(x):
    """fp32 -> bf16 bit pattern, round to nearest even (NaN kept quiet)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    r = np.where(nan, np.uint16(0x7FC0), r)
    return r.astype(np.uint16)


def fp16_bits_to_f64(bits):
    """fp16 bit patterns (uint16) -> exact fp64 values."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# e2m1 (FP4)
# ---------------------------------------------------------------------------


def e2m1_decode(codes):
    """4-bit e2m1 code (0..15) -> exact value.

    OCP MX v1.0, FP4 (E2M1): exponent field e (2 bits, bias 1), mantissa m
    (1 bit).  e == 0 is subnormal: value = m * 2**(1-1) * 0.5; otherwise
    value = 2**(e-1) * (1 + m/2).  Bit 3 is the sign.  Code 8 is -0.
    """
    c = np.asarray(codes).astype(np.int64) & 0xF
    s = np.where(c >> 3, -1.0, 1.0)
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return s * mag


def e2m1_quantize_rne(x):
    """fp32 values -> e2m1 codes, round to nearest, ties to even mantissa,
    saturating at +-6.  A result of zero is emitted as code 0 (never 8).

    The grid of magnitudes is {0, .5, 1, 1.5, 2, 3, 4, 6}: spacing 0.5 below
    2, 1 in [2, 4), 2 in [4, 6].  Rounding |x| / spacing to the nearest
    integer with ties to even is the same as ties-to-even-mantissa, because
    the grid index parity equals the mantissa bit inside each binade and the
    binade edges (2, 4) have mantissa 0.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.abs(x)
    q = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    mag = np.rint(a / q) * q          # np.rint: round half to even
    mag = np.minimum(mag, 6.0)
    # magnitude -> 3-bit code
    table = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    code = np.zeros(mag.shape, dtype=np.int64)
    for v, c in table.items():
        code = np.where(mag == v, c, code)
    neg = (x < 0) & (mag > 0)
    return (code | np.where(neg, 8, 0)).astype(np.uint8)


# ---------------------------------------------------------------------------
# E8M0 (MX block scale)
# ---------------------------------------------------------------------------


def e8m0_decode(codes):
    """E8M0 byte -> 2**(e-127); 0xFF -> NaN (OCP MX v1.0, E8M0)."""
    e = np.asarray(codes).astype(np.int64)
    v = np.ldexp(1.0, e - 127)
    return np.where(e == 255, np.nan, v)


# ---------------------------------------------------------------------------
# E4M3 "fn" (FP8)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """E4M3 byte -> exact value (OCP FP8, E4M3): bias 7, exponent field 0 is
    subnormal with value m * 2**-9, S.1111.111 is NaN, no infinities."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    s = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, m * 2.0 ** -9, np.ldexp(1.0 + m / 8.0, e - 7))
    out = s * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, out)


def e4m3_quantize_rne(x):
    """fp32 values -> E4M3 codes: round to nearest, ties to even, saturate
    to +-448 (finite inputs only).  Zero results are emitted as +0 (0x00).

    For |x| >= 2**-6 the spacing inside binade [2**e, 2**(e+1)) is
    2**(e-3); below that (subnormals) it is 2**-9.  |x| / spacing is exact
    in fp64 (power-of-two scaling), so np.rint gives the exact RNE choice.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # guard log2 rounding at exact powers of two
    e = np.where(np.ldexp(1.0, e.astype(np.int64)) > a, e - 1, e)
    e = np.where(np.ldexp(1.0, (e + 1).astype(np.int64)) <= a, e + 1, e)
    e = np.maximum(e, -6.0)
    q = np.ldexp(1.0, (e - 3).astype(np.int64))
    mag = np.minimum(np.rint(a / q) * q, E4M3_MAX)
    # encode the (now exactly representable) magnitude
    with np.errstate(divide="ignore"):
        ee = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    ee = np.where(np.ldexp(1.0, ee.astype(np.int64)) > mag, ee - 1, ee)
    ee = np.where(np.ldexp(1.0, (ee + 1).astype(np.int64)) <= mag, ee + 1, ee)
    normal = mag >= 2.0 ** -6
    exp_field = np.where(normal, ee + 7, 0).astype(np.int64)
    man = np.where(normal, mag / np.ldexp(1.0, ee.astype(np.int64)) * 8 - 8,
                   mag / 2.0 ** -9)
    code = (exp_field << 3) | np.rint(man).astype(np.int64)
    neg = (x < 0) & (mag > 0)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


# ---------------------------------------------------------------------------
# Activation / weight quantizers used to make block-scaled inputs
# ---------------------------------------------------------------------------


def fp8_per_token_quantize(x_f32):
    """Per-token (row) FP8 quantization of activations.

    Reading of the W4A8-MXFP4 workload: s_m = amax_m / 448 in fp32 (s_m = 1
    when the row is all zero); q = RNE-to-E4M3(fp32(x / s_m)), saturating.
    Returns (codes uint8 [M, K], scales fp32 [M]).
    """
    x = np.asarray(x_f32, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    s = np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)
    r = (x / s[:, None]).astype(np.float32)
    return e4m3_quantize_rne(r), s


def nvfp4_quantize(x_f32):
    """Two-level NVFP4 quantization of a [rows, K] tensor (K % 16 == 0).

    Reading (the pages only name NVFP4; NVIDIA's public description gives
    e2m1 codes, an E4M3 scale per 16 contiguous elements and one fp32 scale
    per tensor), every step in fp32:
      g   = amax_tensor / (448 * 6)            (g = 1 if the tensor is zero)
      sb  = RNE-E4M3(amax_block / (6 * g))     (saturating at 448)
      d   = fp32(decode(sb) * g)
      c   = RNE-e2m1(fp32(x / d)) saturating   (c = 0 when sb decodes to 0)
    Value: x_hat = e2m1(c) * decode(sb) * g.
    Returns (codes uint8 [rows, K] one code per byte, sb uint8 [rows, K/16],
    g float32).
    """
    x = np.asarray(x_f32, dtype=np.float32)
    rows, k = x.shape
    assert k % 16 == 0
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    g = np.float32(amax / np.float32(448.0 * 6.0)) if amax > 0 else np.float32(1.0)
    xb = x.reshape(rows, k // 16, 16)
    bmax = np.max(np.abs(xb), axis=2).astype(np.float32)
    ratio = (bmax / (np.float32(6.0) * g)).astype(np.float32)
    sb = e4m3_quantize_rne(ratio)
    sbv = e4m3_decode(sb).astype(np.float32)
    d = (sbv * g).astype(np.float32)
    safe = np.where(d > 0, d, np.float32(1.0)).astype(np.float32)
    r = (xb / safe[:, :, None]).astype(np.float32)
    c = e2m1_quantize_rne(r)
    c = np.where((d > 0)[:, :, None], c, np.uint8(0)).astype(np.uint8)
    return c.reshape(rows, k), sb, g


def nvfp4_dequantize(codes, sb, g):
    """x_hat[r, k] = e2m1(codes[r, k]) * E4M3(sb[r, k/16]) * g, exact fp64."""
    codes = np.asarray(codes)
    rows, k = codes.shape
    v = e2m1_decode(codes).reshape(rows, k // 16, 16)
    s = e4m3_decode(sb)[:, :, None] * float(np.float32(g))
    return (v * s).reshape(rows, k)


# ---------------------------------------------------------------------------
# Canonical (pre-pack) bit containers
# ---------------------------------------------------------------------------


def int4_unpack_words(qweight):
    """int32 [N, K/8] words -> uint8 codes [N, K].

    Canonical reading of "uint4 packed 8 per int32 along K": element k of a
    row lives in bits [4*(k%8), 4*(k%8)+4) of word k//8 (low nibble first).
    """
    w = np.asarray(qweight).astype(np.int64) & 0xFFFFFFFF
    n, kw = w.shape
    shifts = 4 * np.arange(8, dtype=np.int64)
    codes = (w[:, :, None] >> shifts[None, None, :]) & 0xF
    return codes.reshape(n, kw * 8).astype(np.uint8)


def int4_pack_words(codes):
    """uint8 codes [N, K] (0..15) -> int32 words [N, K/8] (inverse of
    int4_unpack_words)."""
    c = np.asarray(codes).astype(np.int64)
    n, k = c.shape
    assert k % 8 == 0
    c = c.reshape(n, k // 8, 8)
    w = np.zeros((n, k // 8), dtype=np.int64)
    for e in range(8):
        w |= (c[:, :, e] & 0xF) << (4 * e)
    return w.astype(np.uint32).view(np.int32)


def fp4_unpack_bytes(packed):
    """uint8 [R, K/2] -> codes [R, K]; even k in the low nibble."""
    p = np.asarray(packed, dtype=np.uint8)
    r, kh = p.shape
    out = np.empty((r, kh * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def fp4_pack_bytes(codes):
    """codes [R, K] -> uint8 [R, K/2]; even k in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return ((c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)).astype(np.uint8)


def int3_unpack_stream(qweight):
    """int32 [N, 3K/32] -> uint8 codes [N, K] (0..7).

    Canonical INT3 container (the pages name GPTQ INT3 weights and give no
    packing; the plainest reading): each row's K codes form one little-endian
    bit stream, code k in stream bits [3k, 3k+3), stream bit b being bit
    b % 32 of word b // 32 (so 32 codes fill 3 words and some codes straddle
    two words)."""
    w = np.asarray(qweight).astype(np.int64) & 0xFFFFFFFF
    n, nw = w.shape
    k = nw * 32 // 3
    bits = ((w[:, :, None] >> np.arange(32, dtype=np.int64)[None, None, :]) & 1).reshape(n, nw * 32)
    b3 = bits[:, : 3 * k].reshape(n, k, 3)
    return (b3[:, :, 0] | (b3[:, :, 1] << 1) | (b3[:, :, 2] << 2)).astype(np.uint8)


def int3_pack_stream(codes):
    """uint8 codes [N, K] (0..7), K % 32 == 0 -> int32 [N, 3K/32] (inverse
    of int3_unpack_stream)."""
    c = np.asarray(codes).astype(np.int64)
    n, k = c.shape
    assert k % 32 == 0
    bits = np.stack([(c >> i) & 1 for i in range(3)], axis=2).reshape(n, 3 * k)
    words = (bits.reshape(n, 3 * k // 32, 32) << np.arange(32, dtype=np.int64)).sum(axis=2)
    return words.astype(np.uint32).view(np.int32)


def int2_unpack_words(qweight):
    """int32 [N, K/16] words -> uint8 codes [N, K] (0..3).

    Canonical INT2 container (the pages list INT1..INT8 weights without a
    packing; the INT4 reading with 2-bit fields): element k of a row lives
    in bits [2*(k%16), 2*(k%16)+2) of word k//16 (low bits first)."""
    w = np.asarray(qweight).astype(np.int64) & 0xFFFFFFFF
    n, kw = w.shape
    shifts = 2 * np.arange(16, dtype=np.int64)
    return ((w[:, :, None] >> shifts[None, None, :]) & 3).reshape(n, kw * 16).astype(np.uint8)


def int2_pack_words(codes):
    """uint8 codes [N, K] (0..3), K % 16 == 0 -> int32 [N, K/16] (inverse of
    int2_unpack_words)."""
    c = np.asarray(codes).astype(np.int64)
    n, k = c.shape
    assert k % 16 == 0
    c = c.reshape(n, k // 16, 16)
    w = np.zeros((n, k // 16), dtype=np.int64)
    for e in range(16):
        w |= (c[:, :, e] & 3) << (2 * e)
    return w.astype(np.uint32).view(np.int32)


def int8_unpack_words(qweight):
    """int32 [N, K/4] words -> uint8 codes [N, K] (0..255).

    Canonical INT8 container (the pages list INT1..INT8 weights without a
    packing; the INT4 reading with 8-bit fields): element k of a row lives in
    bits [8*(k%4), 8*(k%4)+8) of word k//4 (low byte first)."""
    w = np.asarray(qweight).astype(np.int64) & 0xFFFFFFFF
    n, kw = w.shape
    shifts = 8 * np.arange(4, dtype=np.int64)
    return ((w[:, :, None] >> shifts[None, None, :]) & 0xFF).reshape(n, kw * 4).astype(np.uint8)


def int8_pack_words(codes):
    """uint8 codes [N, K], K % 4 == 0 -> int32 [N, K/4] (inverse of
    int8_unpack_words)."""
    c = np.asarray(codes).astype(np.int64)
    n, k = c.shape
    assert k % 4 == 0
    c = c.reshape(n, k // 4, 4)
    w = np.zeros((n, k // 4), dtype=np.int64)
    for e in range(4):
        w |= (c[:, :, e] & 0xFF) << (8 * e)
    return w.astype(np.uint32).view(np.int32)


def int4_twos_complement(codes):
    """4-bit code (0..15) -> its two's-complement integer (-8..7): the MXINT4
    element (an integer element with a shared E8M0 scale per 32 K, the MX
    integer format read at 4 bits)."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    return np.where(c >= 8, c - 16, c)
