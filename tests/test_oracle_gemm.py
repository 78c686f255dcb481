"""Pins for the oracle's GEMMs: integer-domain identities, special cases
that reduce to a plain matmul (torch fp64), closed forms, brute force."""

import numpy as np
import torch

from oracle import formats as F
from oracle import gemm as G
from quantized_gemm_bit_b200 import synth


def _w4(n, k, asym, seed):
    q, s, z = synth.w4a16_weights(n, k, 128, asym, seed)
    return q.numpy(), s.numpy(), (None if z is None else z.numpy())


def _a(m, k, seed):
    return synth.bf16_normal(m, k, seed).view(torch.int16).numpy().view(np.uint16)


def test_w4a16_matches_integer_domain_evaluation():
    for asym in (False, True):
        q, s, z = _w4(96, 512, asym, 11)
        a = _a(5, 512, 12)
        c1 = G.w4a16_ref(a, q, s, z, 128)
        c2 = G.w4a16_ref_integer_domain(a, q, s, z, 128)
        assert np.max(np.abs(c1 - c2)) <= 1e-12 * np.max(np.abs(c1))


def test_w4a16_unit_scale_zero_zero_is_plain_matmul():
    """s = 1, z = 0: W_hat is the integer code matrix, so C = A @ Q.T
    exactly (all sums are exact in fp64 at this size)."""
    q, _, _ = _w4(64, 256, True, 13)
    s = np.ones((64, 2), dtype=np.float16)
    z = np.zeros((64, 2), dtype=np.uint8)
    a = _a(3, 256, 14)
    got = G.w4a16_ref(a, q, s, z, 128)
    codes = torch.from_numpy(F.int4_unpack_words(q).astype(np.float64))
    at = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    ref = torch.matmul(at, codes.T).numpy()
    assert np.array_equal(got, ref)


def test_w4a16_closed_form_all_codes_and_zero_points():
    """M = N = 1, K = one group, every weight code q, zero point z, scale s,
    activations all 1: C = 128 * (q - z) * s, for all 16 x 16 (q, z)."""
    s16 = np.float16(0.0123)
    a = np.full((1, 128), 0x3F80, dtype=np.uint16)          # bf16 1.0
    for qv in range(16):
        for zv in range(16):
            codes = np.full((1, 128), qv, dtype=np.uint8)
            qw = F.int4_pack_words(codes)
            c = G.w4a16_ref(a, qw, np.array([[s16]]), np.array([[zv]], dtype=np.uint8), 128)
            assert c[0, 0] == 128.0 * (qv - zv) * float(s16)
    # symmetric form uses zero point 8
    qw = F.int4_pack_words(np.full((1, 128), 3, dtype=np.uint8))
    c = G.w4a16_ref(a, qw, np.array([[s16]]), None, 128)
    assert c[0, 0] == 128.0 * (3 - 8) * float(s16)


def test_w4a16_naive_triple_loop():
    """A separately written pure-Python loop over (m, n, k) on a tiny case."""
    q, s, z = _w4(128, 256, True, 15)
    a = _a(3, 256, 16)
    got = G.w4a16_ref(a, q, s, z, 128)
    af = F.bf16_bits_to_f64(a)
    words = q.astype(np.int64) & 0xFFFFFFFF
    for m in range(3):
        for n in (0, 1, 63, 127):
            acc = 0.0
            for k in range(256):
                code = (int(words[n, k // 8]) >> (4 * (k % 8))) & 0xF
                w = (code - int(z[n, k // 128])) * float(s[n, k // 128])
                acc += float(af[m, k]) * w
            assert abs(acc - got[m, n]) <= 1e-12 * max(1.0, abs(acc))


def test_w4a16_row_and_column_subsets():
    q, s, z = _w4(256, 384, False, 17)
    a = _a(9, 384, 18)
    full = G.w4a16_ref(a, q, s, z, 128)
    rows, cols = np.array([0, 4, 8]), np.array([1, 200, 255])
    sub = G.w4a16_ref(a, q, s, z, 128, rows=rows, cols=cols)
    assert np.array_equal(sub, full[np.ix_(rows, cols)])


def test_mxfp4_matches_exact_integer_evaluation():
    codes, e8 = synth.mxfp4_weights(64, 256, seed=21)
    aq, asc = F.fp8_per_token_quantize(synth.bf16_normal(7, 256, seed=22).float().numpy())
    c1 = G.mxfp4_a8_ref(aq, asc, codes.numpy(), e8.numpy())
    c2 = G.mxfp4_a8_ref_exact(aq, asc, codes.numpy(), e8.numpy())
    assert np.max(np.abs(c1 - c2)) <= 1e-12 * np.max(np.abs(c1))


def test_mxfp4_unit_scales_is_plain_matmul_of_decoded_values():
    """All E8M0 = 127 (scale 1) and token scale 1: C = e4m3(A) @ e2m1(W).T,
    with both decodes taken from torch's own float8 dtype / the standard's
    e2m1 table."""
    codes, _ = synth.mxfp4_weights(32, 128, seed=23)
    e8 = np.full((32, 4), 127, dtype=np.uint8)
    aq, _ = F.fp8_per_token_quantize(synth.bf16_normal(4, 128, seed=24).float().numpy())
    one = np.ones(4, dtype=np.float32)
    got = G.mxfp4_a8_ref(aq, one, codes.numpy(), e8)
    a_t = torch.from_numpy(aq).view(torch.float8_e4m3fn).to(torch.float64)
    table = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6],
                         dtype=torch.float64)
    lo = codes.to(torch.int64) & 0xF
    hi = codes.to(torch.int64) >> 4
    wv = torch.stack([table[lo], table[hi]], dim=2).reshape(32, 128)
    ref = torch.matmul(a_t, wv.T).numpy()
    assert np.array_equal(got, ref)


def test_mxfp4_closed_form_scale_exponents():
    """M = N = 1, one 32-block: activation all E4M3 1.0 (0x38), token scale
    s, weight codes all c, E8M0 exponent e: C = 32 * e2m1(c) * 2**(e-127) * s."""
    a = np.full((1, 32), 0x38, dtype=np.uint8)
    s = np.array([0.75], dtype=np.float32)
    table = [0, .5, 1, 1.5, 2, 3, 4, 6, 0, -.5, -1, -1.5, -2, -3, -4, -6]
    for c in range(16):
        for e in (119, 125, 127, 130):
            w = F.fp4_pack_bytes(np.full((1, 32), c, dtype=np.uint8))
            got = G.mxfp4_a8_ref(a, s, w, np.array([[e]], dtype=np.uint8))[0, 0]
            assert got == 32 * table[c] * 2.0 ** (e - 127) * 0.75


def test_nvfp4_matches_exact_integer_evaluation():
    rng = np.random.default_rng(31)
    xa = rng.standard_normal((9, 128)).astype(np.float32)
    xw = rng.standard_normal((40, 128)).astype(np.float32)
    ca, sa, ga = F.nvfp4_quantize(xa)
    cw, sw, gw = F.nvfp4_quantize(xw)
    pa, pw = F.fp4_pack_bytes(ca), F.fp4_pack_bytes(cw)
    c1 = G.nvfp4_ref(pa, sa, ga, pw, sw, gw)
    c2 = G.nvfp4_ref_exact(pa, sa, ga, pw, sw, gw)
    assert np.max(np.abs(c1 - c2)) <= 1e-12 * np.max(np.abs(c1))


def test_nvfp4_closed_form_one_block():
    """One 16-block: every code c_a, c_w, block scales 1.0 (0x38) and
    2.0 (0x40), globals ga, gw: C = 16 * e2m1(c_a) * e2m1(c_w) * 2 * ga * gw."""
    table = [0, .5, 1, 1.5, 2, 3, 4, 6, 0, -.5, -1, -1.5, -2, -3, -4, -6]
    ga, gw = np.float32(0.5), np.float32(0.25)
    for ca in range(16):
        for cw in range(16):
            pa = F.fp4_pack_bytes(np.full((1, 16), ca, dtype=np.uint8))
            pw = F.fp4_pack_bytes(np.full((1, 16), cw, dtype=np.uint8))
            got = G.nvfp4_ref(pa, np.array([[0x38]], np.uint8), ga, pw,
                              np.array([[0x40]], np.uint8), gw)[0, 0]
            assert got == 16 * table[ca] * table[cw] * 2.0 * 0.5 * 0.25


def test_grouped_matches_per_expert_dense():
    e, n, k = 4, 128, 256
    q, s, z = synth.w4a16_weights(n, k, 128, False, seed=41, experts=e)
    q, s = q.numpy(), s.numpy()
    off = np.array([0, 3, 3, 10, 12], dtype=np.int32)     # expert 1 empty
    a = _a(12, k, 42)
    rows, got = G.grouped_w4a16_ref(a, off, q, s, None, 128)
    for ex in range(e):
        lo, hi = off[ex], off[ex + 1]
        if hi > lo:
            ref = G.w4a16_ref(a[lo:hi], q[ex], s[ex], None, 128)
            assert np.array_equal(got[lo:hi], ref)
    rows2, sub = G.grouped_w4a16_ref(a, off, q, s, None, 128, row_subset=[11, 0, 5],
                                     cols=np.array([3, 100]))
    assert np.array_equal(sub, got[np.ix_([11, 0, 5], [3, 100])])
