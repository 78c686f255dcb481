"""Seeded synthetic inputs shaped like the method's workloads.

This module only draws random numbers (torch CPU generator, fixed seeds) and
puts them in the canonical containers the library and the oracle both read.
It holds none of the method's arithmetic: no quantization, no
dequantization, no GEMM, no routing.

Recipes (one per workload; seed = workload index * 1000 + shape index):
  * W4A16: qweight int32 [N, K/8] with every bit uniform (= eight uniform
    uint4 codes per word, packed along K, low nibble first); fp16 scales
    0.002 + 0.01*|N(0,1)| per (row, group of 128 along K); zero points
    uniform in [0, 15] (asymmetric) or none (symmetric, zero point 8);
    activations bf16 N(0,1).
  * W3A16 (INT3): as W4A16 with 3 K/32 int32 words per row (every bit
    uniform = uniform 3-bit codes in a little-endian bit stream) and zero
    points uniform in [0, 7] (symmetric: zero point 4).
  * W2A16 (INT2): as W4A16 with K/16 int32 words per row (16 uniform
    2-bit codes each) and zero points uniform in [0, 3] (symmetric: 2).
  * W8A16 (INT8): as W4A16 with K/4 int32 words per row (4 uniform 8-bit
    codes each) and zero points uniform in [0, 255] (symmetric: 128).
  * MXINT4 weights: 4-bit codes uniform over the 16 codes (two's
    complement -8..7), two per byte (even k low nibble); one E8M0 scale per
    32 K with exponent uniform in [-8, -2], as for MXFP4.
  * W4A8-MXFP4 (and MXFP4 weights with bf16 activations): FP4 codes
    uniform over the 16 codes, two per byte (even k low nibble); one E8M0
    scale per 32 K with exponent uniform in [-8, -2];
    activations bf16 N(0,1) draws; their per-token FP8 quantization
    (scale amax/448) is the method's arithmetic and is not done here (the
    GPU path runs the library's quantizer, the tests the oracle's).
  * NVFP4: bf16 N(0,1) draws for both operands; the two-level quantization
    that turns them into codes is the method's arithmetic and is not done
    here.
  * MoE: router logits fp32 N(0,1) [T, E]; activations bf16 N(0,1).
"""

import torch


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def bf16_normal(rows, cols, seed):
    """bf16 N(0,1) [rows, cols] (torch tensor, CPU)."""
    g = _gen(seed)
    return torch.randn(rows, cols, generator=g, dtype=torch.float32).to(torch.bfloat16)


def w4a16_weights(n, k, group=128, asym=False, seed=0, experts=None):
    """Canonical W4A16 weights.  Returns (qweight int32 [.., N, K/8],
    scales fp16 [.., N, K/G], zeros uint8 [.., N, K/G] or None).  With
    `experts` set, a leading expert dimension is added."""
    assert k % group == 0 and k % 8 == 0
    g = _gen(seed)
    lead = () if experts is None else (experts,)
    qweight = torch.randint(-(2 ** 31), 2 ** 31, lead + (n, k // 8), generator=g, dtype=torch.int32)
    scales = (0.002 + 0.01 * torch.randn(lead + (n, k // group), generator=g).abs()).to(torch.float16)
    zeros = None
    if asym:
        zeros = torch.randint(0, 16, lead + (n, k // group), generator=g, dtype=torch.uint8)
    return qweight, scales, zeros


def w2a16_weights(n, k, group=128, asym=False, seed=0, experts=None):
    """Canonical INT2 weights: qweight int32 [.., N, K/16] with every bit
    uniform (= 16 uniform 2-bit codes per word along K, low bits first), fp16
    scales as for W4A16, zero points uniform in [0, 3] (asymmetric) or none
    (symmetric, zero point 2)."""
    assert k % group == 0 and k % 16 == 0
    g = _gen(seed)
    lead = () if experts is None else (experts,)
    qweight = torch.randint(-(2 ** 31), 2 ** 31, lead + (n, k // 16), generator=g, dtype=torch.int32)
    scales = (0.002 + 0.01 * torch.randn(lead + (n, k // group), generator=g).abs()).to(torch.float16)
    zeros = None
    if asym:
        zeros = torch.randint(0, 4, lead + (n, k // group), generator=g, dtype=torch.uint8)
    return qweight, scales, zeros


def w3a16_weights(n, k, group=128, asym=False, seed=0, experts=None):
    """Canonical INT3 weights: qweight int32 [.., N, 3K/32] with every bit
    uniform (= uniform 3-bit codes in each row's little-endian bit stream),
    fp16 scales as for W4A16, zero points uniform in [0, 7] (asymmetric) or
    none (symmetric, zero point 4)."""
    assert k % group == 0 and k % 32 == 0
    g = _gen(seed)
    lead = () if experts is None else (experts,)
    qweight = torch.randint(-(2 ** 31), 2 ** 31, lead + (n, 3 * k // 32), generator=g, dtype=torch.int32)
    scales = (0.002 + 0.01 * torch.randn(lead + (n, k // group), generator=g).abs()).to(torch.float16)
    zeros = None
    if asym:
        zeros = torch.randint(0, 8, lead + (n, k // group), generator=g, dtype=torch.uint8)
    return qweight, scales, zeros


def w8a16_weights(n, k, group=128, asym=False, seed=0, experts=None):
    """Canonical INT8 weights: qweight int32 [.., N, K/4] with every bit
    uniform (= 4 uniform 8-bit codes per word along K, low byte first), fp16
    scales as for W4A16, zero points uniform in [0, 255] (asymmetric) or none
    (symmetric, zero point 128)."""
    assert k % group == 0 and k % 4 == 0
    g = _gen(seed)
    lead = () if experts is None else (experts,)
    qweight = torch.randint(-(2 ** 31), 2 ** 31, lead + (n, k // 4), generator=g, dtype=torch.int32)
    scales = (0.002 + 0.01 * torch.randn(lead + (n, k // group), generator=g).abs()).to(torch.float16)
    zeros = None
    if asym:
        zeros = torch.randint(0, 256, lead + (n, k // group), generator=g, dtype=torch.uint8)
    return qweight, scales, zeros


def mxint4_weights(n, k, seed=0, experts=None):
    """MXINT4 weights: codes uint8 [.., N, K/2] (two uniform 4-bit codes per
    byte, even k low nibble), E8M0 scales uint8 [.., N, K/32] with exponent
    uniform in [-8, -2] (the MXFP4 recipe's draws)."""
    return mxfp4_weights(n, k, seed=seed, experts=experts)


def mxfp4_weights(n, k, seed=0, experts=None):
    """MXFP4 weights: codes uint8 [.., N, K/2] (two uniform FP4 codes per
    byte), E8M0 scales uint8 [.., N, K/32] with exponent uniform in [-8, -2].
    With `experts` set, a leading expert dimension is added."""
    assert k % 32 == 0
    g = _gen(seed)
    lead = () if experts is None else (experts,)
    codes = torch.randint(0, 256, lead + (n, k // 2), generator=g, dtype=torch.uint8)
    e8m0 = (127 + torch.randint(-8, -1, lead + (n, k // 32), generator=g, dtype=torch.int32)).to(torch.uint8)
    return codes, e8m0


def router_logits(t, e, seed=0):
    g = _gen(seed)
    return torch.randn(t, e, generator=g, dtype=torch.float32)
