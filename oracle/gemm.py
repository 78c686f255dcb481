"""Reference GEMMs with element-by-element dequantization, fp64 matmul.
Test infrastructure only.

Convention (a linear layer): C[m, n] = sum_k A_hat[m, k] * W_hat[n, k];
A is [M, K] row-major, W is logically [N, K] with K contiguous.

The method fuses dequantization into the GEMM ("Humming: open-source kernel
library for quantized inference", summary, second and fourth paragraphs:
one description with weight / scale / zero point separate; weights are
converted inside the kernel).  Fusion is an implementation choice, not an
approximation, so the oracle is the plain definition: dequantize every
weight, then multiply in fp64.  numpy's matmul serves as the one library
step; it is exact here up to fp64 rounding of the sums.
"""

import numpy as np

from . import formats as F

# ---------------------------------------------------------------------------
# W4A16: INT4 codes, fp16 group scales, uint4 zero points (or symmetric 8)
# ---------------------------------------------------------------------------


def w4a16_dequant(qweight, scales, zeros, group, rows=None):
    """W_hat[n, k] = (q[n, k] - z[n, k // G]) * s[n, k // G]   (fp64).

    qweight: int32 [N, K/8] (8 codes per word along K, low nibble first)
    scales : float16 [N, K/G]
    zeros  : uint8 [N, K/G] holding 0..15, or None for the symmetric form
             (zero point 8)
    rows   : optional subset of n to dequantize.
    The zero point is an integer code subtracted before scaling (no storage
    offset): the plainest reading of "zero point" next to "scale".
    """
    if rows is not None:
        qweight = np.asarray(qweight)[rows]
        scales = np.asarray(scales)[rows]
        zeros = None if zeros is None else np.asarray(zeros)[rows]
    q = F.int4_unpack_words(qweight).astype(np.float64)
    n, k = q.shape
    g = np.arange(k) // group
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)[:, g]
    if zeros is None:
        z = 8.0
    else:
        z = np.asarray(zeros).astype(np.float64)[:, g]
    return (q - z) * s


def w4a16_ref(a_bf16, qweight, scales, zeros, group, rows=None, cols=None):
    """C = A_hat @ W_hat.T in fp64 for W4A16.  a_bf16 holds bf16 bit
    patterns (uint16) [M, K].  rows / cols select a subset of outputs."""
    a = F.bf16_bits_to_f64(a_bf16 if rows is None else np.asarray(a_bf16)[rows])
    w = w4a16_dequant(qweight, scales, zeros, group, rows=cols)
    return a @ w.T


def w3a16_dequant(qweight, scales, zeros, group, rows=None):
    """INT3 weights: W_hat[n, k] = (q[n, k] - z[n, k // G]) * s[n, k // G]
    (fp64), the same definition as INT4 with 3-bit codes.

    qweight: int32 [N, 3K/32] (each row one little-endian bit stream of
             3-bit codes, see formats.int3_unpack_stream)
    scales : float16 [N, K/G]
    zeros  : uint8 [N, K/G] holding 0..7, or None for the symmetric form
             (zero point 4, the middle of the code range as 8 is for INT4)
    """
    if rows is not None:
        qweight = np.asarray(qweight)[rows]
        scales = np.asarray(scales)[rows]
        zeros = None if zeros is None else np.asarray(zeros)[rows]
    q = F.int3_unpack_stream(qweight).astype(np.float64)
    n, k = q.shape
    g = np.arange(k) // group
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)[:, g]
    z = 4.0 if zeros is None else np.asarray(zeros).astype(np.float64)[:, g]
    return (q - z) * s


def w3a16_ref(a_bf16, qweight, scales, zeros, group, rows=None, cols=None):
    """C = A_hat @ W_hat.T in fp64 for INT3 weights (bf16 bit patterns in)."""
    a = F.bf16_bits_to_f64(a_bf16 if rows is None else np.asarray(a_bf16)[rows])
    w = w3a16_dequant(qweight, scales, zeros, group, rows=cols)
    return a @ w.T


def w2a16_dequant(qweight, scales, zeros, group, rows=None):
    """INT2 weights: W_hat[n, k] = (q[n, k] - z[n, k // G]) * s[n, k // G]
    (fp64) with 2-bit codes (formats.int2_unpack_words); symmetric zero
    point 2, the middle of the code range."""
    if rows is not None:
        qweight = np.asarray(qweight)[rows]
        scales = np.asarray(scales)[rows]
        zeros = None if zeros is None else np.asarray(zeros)[rows]
    q = F.int2_unpack_words(qweight).astype(np.float64)
    n, k = q.shape
    g = np.arange(k) // group
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)[:, g]
    z = 2.0 if zeros is None else np.asarray(zeros).astype(np.float64)[:, g]
    return (q - z) * s


def w2a16_ref(a_bf16, qweight, scales, zeros, group, rows=None, cols=None):
    """C = A_hat @ W_hat.T in fp64 for INT2 weights (bf16 bit patterns in)."""
    a = F.bf16_bits_to_f64(a_bf16 if rows is None else np.asarray(a_bf16)[rows])
    w = w2a16_dequant(qweight, scales, zeros, group, rows=cols)
    return a @ w.T


def w8a16_dequant(qweight, scales, zeros, group, rows=None):
    """INT8 weights: W_hat[n, k] = (q[n, k] - z[n, k // G]) * s[n, k // G]
    (fp64), the INT4 definition with 8-bit codes (formats.int8_unpack_words);
    zeros uint8 [N, K/G] holding 0..255, or None for the symmetric form
    (zero point 128, the middle of the code range as 8 is for INT4)."""
    if rows is not None:
        qweight = np.asarray(qweight)[rows]
        scales = np.asarray(scales)[rows]
        zeros = None if zeros is None else np.asarray(zeros)[rows]
    q = F.int8_unpack_words(qweight).astype(np.float64)
    n, k = q.shape
    g = np.arange(k) // group
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)[:, g]
    z = 128.0 if zeros is None else np.asarray(zeros).astype(np.float64)[:, g]
    return (q - z) * s


def w8a16_ref(a_bf16, qweight, scales, zeros, group, rows=None, cols=None):
    """C = A_hat @ W_hat.T in fp64 for INT8 weights (bf16 bit patterns in)."""
    a = F.bf16_bits_to_f64(a_bf16 if rows is None else np.asarray(a_bf16)[rows])
    w = w8a16_dequant(qweight, scales, zeros, group, rows=cols)
    return a @ w.T


def w4a16_ref_integer_domain(a_bf16, qweight, scales, zeros, group):
    """The same product evaluated as sum_g s_g * sum_{k in g} a_k (q_k - z_g):
    the group sums use integer weights (q - z), the scale enters once per
    group.  Used only to pin w4a16_ref (the two must agree to fp64
    rounding)."""
    a = F.bf16_bits_to_f64(a_bf16)
    q = F.int4_unpack_words(qweight).astype(np.int64)
    n, k = q.shape
    ng = k // group
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    z = np.full((n, ng), 8, dtype=np.int64) if zeros is None else np.asarray(zeros).astype(np.int64)
    out = np.zeros((a.shape[0], n))
    for gi in range(ng):
        sl = slice(gi * group, (gi + 1) * group)
        d = (q[:, sl] - z[:, gi:gi + 1]).astype(np.float64)   # integers
        out += (a[:, sl] @ d.T) * s[None, :, gi]
    return out


# ---------------------------------------------------------------------------
# W4A8-MXFP4: e2m1 weights with E8M0 scale per 32 K, E4M3 activations with
# a per-token fp32 scale
# ---------------------------------------------------------------------------

MX_BLOCK = 32


def mxfp4_dequant(w_packed, w_e8m0, rows=None):
    """W_hat[n, k] = e2m1(c[n, k]) * 2**(e[n, k // 32] - 127)  (fp64).
    w_packed: uint8 [N, K/2] (even k low nibble); w_e8m0: uint8 [N, K/32]."""
    if rows is not None:
        w_packed = np.asarray(w_packed)[rows]
        w_e8m0 = np.asarray(w_e8m0)[rows]
    c = F.fp4_unpack_bytes(w_packed)
    n, k = c.shape
    v = F.e2m1_decode(c)
    s = F.e8m0_decode(w_e8m0)[:, np.arange(k) // MX_BLOCK]
    return v * s


def fp8_act_dequant(a_e4m3, a_scale, rows=None):
    """A_hat[m, k] = E4M3(q[m, k]) * s_m  (fp64; s_m is fp32)."""
    if rows is not None:
        a_e4m3 = np.asarray(a_e4m3)[rows]
        a_scale = np.asarray(a_scale)[rows]
    return F.e4m3_decode(a_e4m3) * np.asarray(a_scale, dtype=np.float32).astype(np.float64)[:, None]


def mxfp4_a8_ref(a_e4m3, a_scale, w_packed, w_e8m0, rows=None, cols=None):
    a = fp8_act_dequant(a_e4m3, a_scale, rows=rows)
    w = mxfp4_dequant(w_packed, w_e8m0, rows=cols)
    return a @ w.T


def mxfp4_a8_ref_exact(a_e4m3, a_scale, w_packed, w_e8m0):
    """Integer-domain evaluation used to pin mxfp4_a8_ref: every e2m1 value
    is (integer)/2 and every E4M3 value is (integer)*2**-9, so per 32-block
    the sum of products is an exact integer times 2**-10; the block scale
    and the token scale enter once.  Returns fp64 (exact up to the final
    fp64 additions)."""
    ca = np.asarray(a_e4m3)
    ia = np.rint(F.e4m3_decode(ca) * 512).astype(np.int64)      # exact
    cw = F.fp4_unpack_bytes(w_packed)
    iw = np.rint(F.e2m1_decode(cw) * 2).astype(np.int64)         # exact
    sw = F.e8m0_decode(w_e8m0)
    m, k = ia.shape
    n = iw.shape[0]
    out = np.zeros((m, n))
    for b in range(k // MX_BLOCK):
        sl = slice(b * MX_BLOCK, (b + 1) * MX_BLOCK)
        blk = ia[:, sl] @ iw[:, sl].T                              # exact int64
        out += blk.astype(np.float64) * 2.0 ** -10 * sw[None, :, b]
    return out * np.asarray(a_scale, dtype=np.float32).astype(np.float64)[:, None]


# ---------------------------------------------------------------------------
# W4A4 NVFP4: e2m1 codes, E4M3 scale per 16 K, fp32 global per tensor
# ---------------------------------------------------------------------------

NV_BLOCK = 16


def nvfp4_dequant(packed, sf_e4m3, g, rows=None):
    """X_hat[r, k] = e2m1(c[r, k]) * E4M3(sf[r, k // 16]) * g  (fp64)."""
    if rows is not None:
        packed = np.asarray(packed)[rows]
        sf_e4m3 = np.asarray(sf_e4m3)[rows]
    c = F.fp4_unpack_bytes(packed)
    r, k = c.shape
    v = F.e2m1_decode(c)
    s = F.e4m3_decode(sf_e4m3)[:, np.arange(k) // NV_BLOCK]
    return v * s * float(np.float32(g))


def nvfp4_ref(a_packed, a_sf, a_g, w_packed, w_sf, w_g, rows=None, cols=None):
    a = nvfp4_dequant(a_packed, a_sf, a_g, rows=rows)
    w = nvfp4_dequant(w_packed, w_sf, w_g, rows=cols)
    return a @ w.T


def nvfp4_ref_exact(a_packed, a_sf, a_g, w_packed, w_sf, w_g):
    """Integer-domain evaluation used to pin nvfp4_ref: per 16-block the
    sum of (2*e2m1)*(2*e2m1) is an exact integer in [-144*16, 144*16]; the
    two E4M3 block scales and the two globals enter once per block."""
    ia = np.rint(F.e2m1_decode(F.fp4_unpack_bytes(a_packed)) * 2).astype(np.int64)
    iw = np.rint(F.e2m1_decode(F.fp4_unpack_bytes(w_packed)) * 2).astype(np.int64)
    sa = F.e4m3_decode(a_sf)
    sw = F.e4m3_decode(w_sf)
    m, k = ia.shape
    n = iw.shape[0]
    out = np.zeros((m, n))
    for b in range(k // NV_BLOCK):
        sl = slice(b * NV_BLOCK, (b + 1) * NV_BLOCK)
        blk = (ia[:, sl] @ iw[:, sl].T).astype(np.float64) * 0.25
        out += blk * sa[:, b][:, None] * sw[:, b][None, :]
    return out * float(np.float32(a_g)) * float(np.float32(w_g))


# ---------------------------------------------------------------------------
# Grouped MoE W4A16 over expert-sorted rows
# ---------------------------------------------------------------------------


def _grouped(a_sorted_bf16, expert_offsets, dequant, row_subset, ncols):
    """Rows of C_sorted: row i uses the weights of the expert e whose range
    [offsets[e], offsets[e+1]) holds i; dequant(e) gives W_hat_e (fp64,
    ncols rows)."""
    off = np.asarray(expert_offsets, dtype=np.int64)
    e_count = off.shape[0] - 1
    assert e_count >= 1
    total = int(off[-1])
    rows = np.arange(total) if row_subset is None else np.asarray(row_subset, dtype=np.int64)
    expert_of = np.searchsorted(off, rows, side="right") - 1
    out = np.zeros((len(rows), ncols))
    for e in np.unique(expert_of):
        sel = np.nonzero(expert_of == e)[0]
        w = dequant(int(e))
        a = F.bf16_bits_to_f64(np.asarray(a_sorted_bf16)[rows[sel]])
        out[sel] = a @ w.T
    return rows, out


def grouped_w4a16_ref(a_sorted_bf16, expert_offsets, qweights, scales, zeros, group,
                      row_subset=None, cols=None):
    """C_sorted[i, :] = A_sorted_hat[i, :] @ W_hat_e.T for the expert e whose
    row range [offsets[e], offsets[e+1]) holds i.

    qweights: int32 [E, N, K/8]; scales: float16 [E, N, K/G]; zeros: uint8
    [E, N, K/G] or None.  row_subset restricts the rows computed (returned
    in the given order); cols restricts the output columns.
    Returns (rows, C) with C fp64 [len(rows), len(cols) or N].
    """
    def dequant(e):
        z = None if zeros is None else zeros[e]
        return w4a16_dequant(qweights[e], scales[e], z, group, rows=cols)
    ncols = np.asarray(qweights).shape[1] if cols is None else len(cols)
    return _grouped(a_sorted_bf16, expert_offsets, dequant, row_subset, ncols)


# ---------------------------------------------------------------------------
# MXFP4 weights x bf16 activations (the W4A16 kernels with MXFP4 weights)
# ---------------------------------------------------------------------------


def mxfp4_a16_ref(a_bf16, w_packed, w_e8m0, rows=None, cols=None):
    """C = A_hat @ W_hat.T in fp64 with A_hat the bf16 activations widened
    exactly and W_hat[n, k] = e2m1(c[n, k]) * 2**(e[n, k // 32] - 127), the
    MXFP4 weight of the OCP MX definition (the pages list MXFP4 among the
    weight types and bf16 among the activation types, "Humming: open-source
    kernel library for quantized inference", summary, second paragraph)."""
    a = F.bf16_bits_to_f64(a_bf16 if rows is None else np.asarray(a_bf16)[rows])
    w = mxfp4_dequant(w_packed, w_e8m0, rows=cols)
    return a @ w.T


def grouped_mxfp4_a16_ref(a_sorted_bf16, expert_offsets, w_packed, w_e8m0, row_subset=None, cols=None):
    """Grouped form of mxfp4_a16_ref over expert-sorted rows: w_packed uint8
    [E, N, K/2], w_e8m0 uint8 [E, N, K/32].  Returns (rows, C)."""
    def dequant(e):
        return mxfp4_dequant(w_packed[e], w_e8m0[e], rows=cols)
    ncols = np.asarray(w_packed).shape[1] if cols is None else len(cols)
    return _grouped(a_sorted_bf16, expert_offsets, dequant, row_subset, ncols)


def grouped_w3a16_ref(a_sorted_bf16, expert_offsets, qweights, scales, zeros, group, row_subset=None, cols=None):
    """Grouped form of w3a16_ref: qweights int32 [E, N, 3K/32], scales
    float16 [E, N, K/G], zeros uint8 [E, N, K/G] or None.  Returns (rows, C)."""
    def dequant(e):
        z = None if zeros is None else zeros[e]
        return w3a16_dequant(qweights[e], scales[e], z, group, rows=cols)
    ncols = np.asarray(qweights).shape[1] if cols is None else len(cols)
    return _grouped(a_sorted_bf16, expert_offsets, dequant, row_subset, ncols)


def grouped_w2a16_ref(a_sorted_bf16, expert_offsets, qweights, scales, zeros, group, row_subset=None, cols=None):
    """Grouped form of w2a16_ref: qweights int32 [E, N, K/16], scales
    float16 [E, N, K/G], zeros uint8 [E, N, K/G] or None.  Returns (rows, C)."""
    def dequant(e):
        z = None if zeros is None else zeros[e]
        return w2a16_dequant(qweights[e], scales[e], z, group, rows=cols)
    ncols = np.asarray(qweights).shape[1] if cols is None else len(cols)
    return _grouped(a_sorted_bf16, expert_offsets, dequant, row_subset, ncols)


def grouped_w8a16_ref(a_sorted_bf16, expert_offsets, qweights, scales, zeros, group, row_subset=None, cols=None):
    """Grouped form of w8a16_ref: qweights int32 [E, N, K/4], scales
    float16 [E, N, K/G], zeros uint8 [E, N, K/G] or None.  Returns (rows, C)."""
    def dequant(e):
        z = None if zeros is None else zeros[e]
        return w8a16_dequant(qweights[e], scales[e], z, group, rows=cols)
    ncols = np.asarray(qweights).shape[1] if cols is None else len(cols)
    return _grouped(a_sorted_bf16, expert_offsets, dequant, row_subset, ncols)


# ---------------------------------------------------------------------------
# MXINT4 weights x bf16 activations
# ---------------------------------------------------------------------------


def mxint4_dequant(w_packed, w_e8m0, rows=None):
    """W_hat[n, k] = c[n, k] * 2**(e[n, k // 32] - 127) (fp64, exact): c the
    two's-complement integer of the 4-bit code (formats.int4_twos_complement),
    e the E8M0 scale byte of its 32-K block.  w_packed uint8 [N, K/2] (even
    k in the low nibble), w_e8m0 uint8 [N, K/32]."""
    if rows is not None:
        w_packed = np.asarray(w_packed)[rows]
        w_e8m0 = np.asarray(w_e8m0)[rows]
    c = F.int4_twos_complement(F.fp4_unpack_bytes(w_packed)).astype(np.float64)
    n, k = c.shape
    e = np.asarray(w_e8m0).astype(np.int64)[:, np.arange(k) // MX_BLOCK]
    return c * np.ldexp(1.0, e - 127)


def mxint4_a16_ref(a_bf16, w_packed, w_e8m0, rows=None, cols=None):
    """C = A_hat @ W_hat.T in fp64 for MXINT4 weights (the pages list MXINT4
    among the weight types; Humming news page, section "one library, many
    formats") and bf16 activations."""
    a = F.bf16_bits_to_f64(a_bf16 if rows is None else np.asarray(a_bf16)[rows])
    w = mxint4_dequant(w_packed, w_e8m0, rows=cols)
    return a @ w.T


def grouped_mxint4_a16_ref(a_sorted_bf16, expert_offsets, w_packed, w_e8m0, row_subset=None, cols=None):
    """Grouped form of mxint4_a16_ref: w_packed uint8 [E, N, K/2], w_e8m0
    uint8 [E, N, K/32].  Returns (rows, C)."""
    def dequant(e):
        return mxint4_dequant(w_packed[e], w_e8m0[e], rows=cols)
    ncols = np.asarray(w_packed).shape[1] if cols is None else len(cols)
    return _grouped(a_sorted_bf16, expert_offsets, dequant, row_subset, ncols)
