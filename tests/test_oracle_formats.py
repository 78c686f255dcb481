"""Pins for the oracle's element formats: standard tables, torch's own
float8 dtypes (an independent implementation), tie cases and brute force."""

import math

import numpy as np
import torch

from conftest import read_golden
from oracle import formats as F


def _same(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    both_nan = np.isnan(a) & np.isnan(b)
    eq = (a == b) & (np.signbit(a) == np.signbit(b))
    return np.all(both_nan | eq)


def test_e2m1_table_matches_standard():
    rows = read_golden("e2m1_values.txt")
    codes = np.array([int(r[0]) for r in rows])
    vals = np.array([float(r[1]) for r in rows])
    assert len(codes) == 16
    assert _same(F.e2m1_decode(codes), vals)


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert _same(F.e4m3_decode(codes), ref)


def test_e4m3_special_values():
    for code, val in read_golden("e4m3_special.txt"):
        got = F.e4m3_decode(np.array([int(code, 16)]))[0]
        want = float(val)
        assert (math.isnan(got) and math.isnan(want)) or (got == want and
                                                          math.copysign(1, got) == math.copysign(1, want))


def test_e8m0_decode_matches_torch_and_standard():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = F.e8m0_decode(codes)
    # torch decodes code 0 as 2**-127 like the standard
    assert _same(got, ref)
    for code, val in read_golden("e8m0_special.txt"):
        g = F.e8m0_decode(np.array([int(code)]))[0]
        w = float(val)
        assert (math.isnan(g) and math.isnan(w)) or g == w


def test_rne_tie_cases():
    for fmt, x, want in read_golden("rne_ties.txt"):
        x, want = float(x), float(want)
        if fmt == "e2m1":
            got = F.e2m1_decode(F.e2m1_quantize_rne(np.array([x], dtype=np.float32)))[0]
        else:
            got = F.e4m3_decode(F.e4m3_quantize_rne(np.array([x], dtype=np.float32)))[0]
        assert got == want, (fmt, x, got, want)


def test_e2m1_quantizer_brute_force_nearest():
    """Every output is a nearest grid point; on exact ties the even-mantissa
    neighbour is chosen; zero is always code 0."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    even = np.array([1, 0, 1, 0, 1, 0, 1, 0], dtype=bool)   # mantissa bit 0
    xs = np.concatenate([np.linspace(-8, 8, 20001, dtype=np.float32),
                         (grid[:-1] + grid[1:]).astype(np.float32) / 2,
                         -(grid[:-1] + grid[1:]).astype(np.float32) / 2])
    codes = F.e2m1_quantize_rne(xs)
    vals = F.e2m1_decode(codes)
    for x, v, c in zip(xs.astype(np.float64), vals, codes):
        a = min(abs(x), 6.0)
        d = np.abs(grid - a)
        best = d.min()
        assert abs(abs(v) - a) == best
        cands = np.nonzero(d == best)[0]
        if len(cands) > 1:
            assert even[np.argmin(np.abs(grid - abs(v)))]
        if v == 0:
            assert c == 0
        elif x < 0:
            assert v < 0


def test_e4m3_quantizer_matches_torch_cast_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 50,
        rng.standard_normal(50000).astype(np.float32) * 0.01,
        np.linspace(-448, 448, 100001, dtype=np.float32),
    ])
    ours = F.e4m3_quantize_rne(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # both emit +0 for a zero result only when the input is non-negative;
    # torch keeps the sign of negative values that round to zero
    ref_val = F.e4m3_decode(ref)
    assert np.all(F.e4m3_decode(ours) == ref_val)      # -0 == +0 numerically
    nz = ref_val != 0
    assert np.array_equal(ours[nz], ref[nz])


def test_e4m3_quantizer_saturates():
    x = np.array([449, 500, 1e6, -1e6], dtype=np.float32)
    assert np.array_equal(F.e4m3_decode(F.e4m3_quantize_rne(x)), [448, 448, 448, -448])


def test_bf16_roundtrip_and_rne():
    x = torch.randn(10000, generator=torch.Generator().manual_seed(3))
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = F.f32_to_bf16_bits_rne(x.numpy())
    assert np.array_equal(ours, ref)
    back = F.bf16_bits_to_f64(ref)
    assert np.array_equal(back, x.to(torch.bfloat16).to(torch.float64).numpy())


def test_int4_word_pack_roundtrip_and_nibble_order():
    rng = np.random.default_rng(2)
    codes = rng.integers(0, 16, size=(7, 64), dtype=np.uint8)
    w = F.int4_pack_words(codes)
    assert np.array_equal(F.int4_unpack_words(w), codes)
    # element k sits in bits 4*(k%8): a single code 0xA at k=3 is 0xA000
    one = np.zeros((1, 8), dtype=np.uint8)
    one[0, 3] = 0xA
    assert int(F.int4_pack_words(one)[0, 0]) == 0xA000


def test_fp4_byte_pack_roundtrip_and_nibble_order():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, size=(5, 32), dtype=np.uint8)
    p = F.fp4_pack_bytes(codes)
    assert np.array_equal(F.fp4_unpack_bytes(p), codes)
    assert F.fp4_pack_bytes(np.array([[0x3, 0xC]], dtype=np.uint8))[0, 0] == 0xC3


def test_fp8_per_token_quantizer_properties():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((6, 256)).astype(np.float32)
    x[3] = 0
    q, s = F.fp8_per_token_quantize(x)
    assert s.dtype == np.float32 and s[3] == 1.0
    deq = F.e4m3_decode(q) * s[:, None]
    # the amax element lands on +-448 exactly and relative error of the
    # rest is within half an E4M3 ulp (2**-4) or the subnormal step
    amax_idx = np.argmax(np.abs(x), axis=1)
    for r in (0, 1, 2, 4, 5):
        assert abs(F.e4m3_decode(q[r, amax_idx[r]])) == 448.0
    err = np.abs(deq - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s[:, None] * 2.0 ** -10) * 1.0001
    assert np.all(err <= bound)
    # matches torch's cast of the same fp32 quotient
    r = (x / s[:, None]).astype(np.float32)
    ref = torch.from_numpy(r).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(F.e4m3_decode(q), ref + 0.0)


def test_nvfp4_quantizer_properties():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((8, 64)).astype(np.float32)
    x[2, 16:32] = 0                    # an all-zero block
    c, sb, g = F.nvfp4_quantize(x)
    assert g == np.float32(np.abs(x).max() / np.float32(2688.0))
    assert np.all(c[2, 16:32] == 0) and sb[2, 1] == 0
    xh = F.nvfp4_dequantize(c, sb, g)
    # per block the error is at most half the e2m1 spacing at the top of the
    # grid (1.0 * scale) plus the E4M3 rounding of the block scale
    blk = np.abs(x).reshape(8, 4, 16).max(axis=2)
    scale = F.e4m3_decode(sb) * float(g)
    err = np.abs(xh - x).reshape(8, 4, 16).max(axis=2)
    assert np.all(err <= scale * 1.0 + blk * 0.07 + 1e-12)
    # saturation: the largest element of a block decodes to about +-6*scale
    assert np.all(np.abs(F.e2m1_decode(c)).max(axis=1) <= 6)
    # codes follow from the stated fp32 steps (re-derived one element)
    i, j = 5, 37
    d = np.float32(F.e4m3_decode(sb[i, j // 16]) * g)
    assert c[i, j] == F.e2m1_quantize_rne(np.array([x[i, j] / d], dtype=np.float32))[0]


def test_nvfp4_quantizer_against_torch_fp32_steps():
    """Pins of the two-level NVFP4 quantizer that do not reuse its code:
    the tensor scale is torch's fp32 amax / fp32(2688); every block scale
    is torch's float8_e4m3fn cast (round to nearest even) of the fp32
    quotient amax_block / (6 g) with 6 g an fp32 product, saturated at 448;
    every code is the nearest point of the e2m1 grid {0, .5, 1, 1.5, 2, 3,
    4, 6} to the fp32 quotient x / fp32(E4M3(sb) g), ties to the even
    code, found by brute force over the grid.  Blocks span many binades, so
    a rounding step done in the wrong precision or order moves some block
    scale by one E4M3 step and fails here."""
    import torch
    rng = np.random.default_rng(11)
    rows, k = 64, 1024
    x = rng.standard_normal((rows, k)).astype(np.float32)
    x *= np.exp2(rng.integers(-12, 6, size=(rows, k // 16, 1))).repeat(16, axis=2).reshape(rows, k).astype(np.float32)
    x[3, 32:48] = 0.0                                   # an all-zero block
    c, sb, g = F.nvfp4_quantize(x)
    xt = torch.from_numpy(x)
    g_t = xt.abs().max() / torch.tensor(2688.0, dtype=torch.float32)
    assert g_t.dtype == torch.float32 and np.float32(g) == np.float32(g_t.item())
    bmax = xt.abs().reshape(rows, k // 16, 16).amax(dim=2)
    ratio = bmax / (torch.tensor(6.0, dtype=torch.float32) * g_t)
    sb_t = ratio.clamp(max=448.0).to(torch.float8_e4m3fn)
    assert np.array_equal(sb, sb_t.view(torch.uint8).numpy())
    # codes: brute force over the grid on torch's fp32 quotient
    d = (sb_t.to(torch.float32) * g_t).reshape(rows, k // 16, 1)
    safe = torch.where(d > 0, d, torch.ones_like(d))
    r = (xt.reshape(rows, k // 16, 16) / safe).reshape(rows, k).double().numpy()
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    dist = np.abs(np.abs(r)[..., None] - grid)
    best = dist.min(axis=-1, keepdims=True)
    cand = dist == best
    # ties: the even code of the two candidates
    mag = np.where(cand[..., ::2].any(axis=-1), np.argmax(cand & (np.arange(8) % 2 == 0), axis=-1),
                   np.argmax(cand, axis=-1))
    expect = np.where((r < 0) & (mag > 0), mag | 8, mag)
    zero_blk = (d.reshape(rows, k // 16) == 0).numpy().repeat(16, axis=1)
    expect = np.where(zero_blk, 0, expect)
    assert np.array_equal(c, expect.astype(np.uint8))
