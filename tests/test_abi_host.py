"""Host-side checks of the C ABI (no GPU needed): the library loads and
exports every declared symbol, descriptors validate, the packer matches the
oracle's layout formulas bit for bit, and invalid calls fail before any
launch."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import layout as L
from quantized_gemm_bit_b200 import hq, synth
from quantized_gemm_bit_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()


def test_exports_every_declared_symbol():
    header = open(os.path.join(ROOT, "include", "hq.h")).read()
    declared = set(re.findall(r"\b(hq_[a-z0-9_]+)\s*\(", header))
    assert declared == set(hq.EXPORTS)
    raw = ctypes.CDLL(hq.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name
    assert hq.hq_layout_version() == hq.HQ_LAYOUT_VERSION == 1


def test_desc_validation():
    hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 1024, 1024, 128, 1, 1)
    for args, code in [((hq.HQ_FMT_INT4, 1024, 1000, 128, 0, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_INT4, 1024, 1024, 64, 0, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_INT4, 0, 1024, 128, 0, 1), hq.HQ_ERR_INVALID_ARG),
                       ((hq.HQ_FMT_MXFP4, 128, 128, 32, 1, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_NVFP4, 128, 128, 16, 0, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_MXFP4_A16, 128, 128, 16, 0, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_MXFP4_A16, 128, 96, 32, 0, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_MXFP4_A16, 128, 128, 32, 1, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_MXFP4_A16, 128, 128, 32, 0, 1025), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_INT3, 128, 128, 64, 0, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_INT3, 128, 160, 128, 0, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_INT3, 128, 128, 128, 2, 1), hq.HQ_ERR_INVALID_ARG),
                       ((hq.HQ_FMT_INT2, 128, 128, 32, 0, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_INT2, 128, 128, 128, 0, 1025), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_INT8, 128, 128, 128, 2, 1), hq.HQ_ERR_INVALID_ARG),
                       ((9, 128, 128, 16, 0, 1), hq.HQ_ERR_INVALID_ARG)]:
        with pytest.raises(hq.HQError) as e:
            hq.hq_quant_desc_init(*args)
        assert e.value.status == code
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 128, 128, 128, 0, 1)
    d.layout_version = 0
    assert hq.hq_packed_size(d) == 0


@pytest.mark.parametrize("n,k,asym,experts", [(256, 384, False, 1), (200, 256, True, 1), (128, 256, False, 3)])
def test_int4_pack_matches_oracle_layout(n, k, asym, experts):
    q, s, z = synth.w4a16_weights(n, k, 128, asym, seed=7, experts=experts if experts > 1 else None)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, int(asym), experts)
    blob = hq.hq_pack_weights(d, q, s, z)
    assert blob.size == L.w4a16_packed_bytes(n, k, asym, experts)
    qn, sn = q.numpy(), s.numpy()
    zn = None if z is None else z.numpy()
    if experts == 1:
        ref = L.w4a16_pack(qn, sn, zn)
    else:
        ref = np.concatenate([L.w4a16_pack(qn[e], sn[e], None if zn is None else zn[e]) for e in range(experts)])
    assert np.array_equal(blob, ref)


@pytest.mark.parametrize("fmt,block", [(hq.HQ_FMT_MXFP4, 32), (hq.HQ_FMT_NVFP4, 16)])
@pytest.mark.parametrize("n", [128, 300])
def test_fp4_pack_matches_oracle_layout(fmt, block, n):
    k = 512
    rng = np.random.default_rng(n)
    codes = rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    scales = rng.integers(0, 255, size=(n, k // block), dtype=np.uint8)
    d = hq.hq_quant_desc_init(fmt, n, k, block, 0, 1)
    g = 0.125 if fmt == hq.HQ_FMT_NVFP4 else 0.0
    blob = hq.hq_pack_weights(d, codes, scales, None, g)
    ref = L.fp4_pack(codes, scales, block, g if fmt == hq.HQ_FMT_NVFP4 else None)
    assert np.array_equal(blob, ref)


@pytest.mark.parametrize("n,k,asym,experts", [(256, 384, False, 1), (200, 256, True, 1), (136, 256, True, 3)])
def test_int3_pack_matches_oracle_layout(n, k, asym, experts):
    q, s, z = synth.w3a16_weights(n, k, 128, asym, seed=n + 3, experts=experts if experts > 1 else None)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT3, n, k, 128, int(asym), experts)
    blob = hq.hq_pack_weights(d, q, s, z)
    assert blob.size == L.w3a16_packed_bytes(n, k, asym, experts)
    qn, sn = q.numpy(), s.numpy()
    zn = None if z is None else z.numpy()
    if experts == 1:
        ref = L.w3a16_pack(qn, sn, zn)
    else:
        ref = np.concatenate([L.w3a16_pack(qn[e], sn[e], None if zn is None else zn[e]) for e in range(experts)])
    assert np.array_equal(blob, ref)


@pytest.mark.parametrize("n,k,asym,experts", [(256, 384, False, 1), (200, 256, True, 1), (136, 256, True, 3)])
def test_int2_pack_matches_oracle_layout(n, k, asym, experts):
    q, s, z = synth.w2a16_weights(n, k, 128, asym, seed=n + 2, experts=experts if experts > 1 else None)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT2, n, k, 128, int(asym), experts)
    blob = hq.hq_pack_weights(d, q, s, z)
    assert blob.size == L.w2a16_packed_bytes(n, k, asym, experts)
    qn, sn = q.numpy(), s.numpy()
    zn = None if z is None else z.numpy()
    if experts == 1:
        ref = L.w2a16_pack(qn, sn, zn)
    else:
        ref = np.concatenate([L.w2a16_pack(qn[e], sn[e], None if zn is None else zn[e]) for e in range(experts)])
    assert np.array_equal(blob, ref)


def test_int2_pack_rejects_bad_zero_points():
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT2, 128, 128, 128, 1, 1)
    q, s, z = synth.w2a16_weights(128, 128, 128, True, seed=4)
    zb = z.clone()
    zb[9, 0] = 4
    with pytest.raises(hq.HQError) as e:
        hq.hq_pack_weights(d, q, s, zb)
    assert e.value.status == hq.HQ_ERR_INVALID_ARG


def test_int3_pack_rejects_bad_zero_points():
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT3, 128, 128, 128, 1, 1)
    q, s, z = synth.w3a16_weights(128, 128, 128, True, seed=4)
    zb = z.clone()
    zb[5, 0] = 8
    with pytest.raises(hq.HQError) as e:
        hq.hq_pack_weights(d, q, s, zb)
    assert e.value.status == hq.HQ_ERR_INVALID_ARG
    with pytest.raises(hq.HQError) as e:                 # zeros missing for an asymmetric descriptor
        hq.hq_pack_weights(d, q, s, None)
    assert e.value.status == hq.HQ_ERR_INVALID_ARG


@pytest.mark.parametrize("n,k,experts", [(128, 128, 1), (300, 384, 1), (136, 256, 3)])
def test_mxfp4_a16_pack_matches_oracle_layout(n, k, experts):
    codes, e8 = synth.mxfp4_weights(n, k, seed=n + k, experts=experts if experts > 1 else None)
    if experts == 1:
        # the whole scale range the packer accepts
        e8 = torch.from_numpy(np.random.default_rng(n).integers(0, 253, size=(n, k // 32), dtype=np.uint8))
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4_A16, n, k, 32, 0, experts)
    blob = hq.hq_pack_weights(d, codes, e8)
    assert blob.size == L.mxa16_packed_bytes(n, k, experts)
    cn, en = codes.numpy(), e8.numpy()
    if experts == 1:
        ref = L.mxa16_pack(cn, en)
    else:
        ref = np.concatenate([L.mxa16_pack(cn[e], en[e]) for e in range(experts)])
    assert np.array_equal(blob, ref)


def test_mxfp4_a16_pack_rejects_scales_that_overflow_bf16():
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4_A16, 128, 128, 32, 0, 1)
    codes, e8 = synth.mxfp4_weights(128, 128, seed=5)
    for bad in (253, 255):
        eb = e8.clone()
        eb[3, 1] = bad
        with pytest.raises(hq.HQError) as e:
            hq.hq_pack_weights(d, codes, eb)
        assert e.value.status == hq.HQ_ERR_INVALID_ARG
    with pytest.raises(hq.HQError) as e:                 # no zero points for this format
        hq.hq_pack_weights(d, codes, e8, torch.zeros(128, 4, dtype=torch.uint8))
    assert e.value.status == hq.HQ_ERR_INVALID_ARG


def test_mxfp4_a16_pack_accepts_the_largest_finite_scale():
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4_A16, 128, 128, 32, 0, 1)
    codes, e8 = synth.mxfp4_weights(128, 128, seed=6)
    e8[:] = 252
    blob = hq.hq_pack_weights(d, codes, e8)
    assert np.array_equal(blob, L.mxa16_pack(codes.numpy(), e8.numpy()))


def test_w4a16_family_formats_share_one_launch_plan():
    """INT3, INT2 and MXFP4 weights run the INT4 kernels' plan: the same
    workspace for the same shape, token count and tuning (no device needed;
    the size is computed for a 148-SM part), except where INT4 runs its
    register-path kernel (plan kernel 4), which the other formats do not
    have."""
    for m, t in ((1, None), (16, None), (300, None), (4096, None), (40, hq.Tuning(split_k=3)),
                 (200, hq.Tuning(tile_m=128))):
        d4 = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 18432, 7168, 128, 0, 1)
        d3 = hq.hq_quant_desc_init(hq.HQ_FMT_INT3, 18432, 7168, 128, 1, 1)
        dx = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4_A16, 18432, 7168, 32, 0, 1)
        d2 = hq.hq_quant_desc_init(hq.HQ_FMT_INT2, 18432, 7168, 128, 0, 1)
        w = hq.hq_workspace_size(d3, m, t)
        assert w >= 256 and hq.hq_workspace_size(dx, m, t) == w == hq.hq_workspace_size(d2, m, t)
        if hq.hq_plan_describe(d4, m, t).kernel != 4:
            assert hq.hq_workspace_size(d4, m, t) == w
        else:
            assert m <= 16 and hq.hq_plan_describe(d3, m, t).kernel != 4


def test_fp4_scale_layout_is_a_bijection():
    n, k, block = 256, 512, 16
    nn, bb = np.meshgrid(np.arange(n), np.arange(k // block), indexing="ij")
    off = L.fp4_scale_byte_np(nn.ravel(), bb.ravel(), k, block, 256)
    assert len(np.unique(off)) == off.size
    assert off.min() == 256 * k // 2 and off.max() == 256 * k // 2 + off.size - 1


def test_pack_rejects_bad_arguments():
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 128, 128, 128, 1, 1)
    q, s, z = synth.w4a16_weights(128, 128, 128, True, seed=1)
    with pytest.raises(hq.HQError) as e:          # zeros missing for an asymmetric descriptor
        hq.hq_pack_weights(d, q, s, None)
    assert e.value.status == hq.HQ_ERR_INVALID_ARG
    zb = z.clone()
    zb[0, 0] = 16
    with pytest.raises(hq.HQError) as e:          # zero point out of range
        hq.hq_pack_weights(d, q, s, zb)
    assert e.value.status == hq.HQ_ERR_INVALID_ARG
    out = np.empty(10, dtype=np.uint8)
    st = hq.lib().hq_pack_weights(ctypes.byref(d), q.numpy().ctypes.data, s.numpy().ctypes.data,
                                  z.numpy().ctypes.data, 0.0, out.ctypes.data, out.nbytes)
    assert st == hq.HQ_ERR_WORKSPACE_TOO_SMALL


def test_gemm_argument_errors_need_no_gpu():
    L_ = hq.lib()
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 256, 256, 128, 0, 1)
    # m == 0: nothing to do
    assert L_.hq_gemm_w4a16(ctypes.byref(d), None, None, 0, None, None, None, 0, None) == hq.HQ_OK
    # NULL pointers
    assert L_.hq_gemm_w4a16(ctypes.byref(d), None, None, 4, None, None, None, 0, None) == hq.HQ_ERR_INVALID_ARG
    # misaligned pointers
    assert L_.hq_gemm_w4a16(ctypes.byref(d), 16, 18, 4, 32, None, 256, 1 << 20, None) == hq.HQ_ERR_ALIGNMENT
    # wrong format for the entry point
    d2 = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, 256, 256, 32, 0, 1)
    assert L_.hq_gemm_w4a16(ctypes.byref(d2), 16, 16, 4, 32, None, 256, 1 << 20, None) == hq.HQ_ERR_INVALID_ARG
    # stale descriptor
    d.layout_version = 99
    assert L_.hq_gemm_w4a16(ctypes.byref(d), 16, 16, 4, 32, None, 256, 1 << 20, None) == hq.HQ_ERR_LAYOUT_VERSION
    # unsupported tuning
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 256, 256, 128, 0, 1)
    t = hq.Tuning(tile_m=48)
    assert L_.hq_gemm_w4a16(ctypes.byref(d), 16, 16, 4, 32, ctypes.byref(t), 256, 1 << 20,
                            None) == hq.HQ_ERR_UNSUPPORTED
    for bad in (hq.Tuning(variant=4), hq.Tuning(variant=-1), hq.Tuning(stages=-1), hq.Tuning(cta_group=3),
                hq.Tuning(cta_group=2, tile_m=128), hq.Tuning(cta_group=2, split_k=2), hq.Tuning(flags=2)):
        assert L_.hq_gemm_w4a16(ctypes.byref(d), 16, 16, 4, 32, ctypes.byref(bad), 256, 1 << 20,
                                None) == hq.HQ_ERR_UNSUPPORTED
    # grouped: no K split, no 512-token tile; block-scaled: no variants
    dg = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 256, 256, 128, 0, 8)
    for bad in (hq.Tuning(tile_m=512), hq.Tuning(split_k=2), hq.Tuning(cta_group=2)):
        assert L_.hq_grouped_gemm_moe(ctypes.byref(dg), 16, 16, 16, 40, 32, ctypes.byref(bad), 256, 1 << 20,
                                      None) == hq.HQ_ERR_UNSUPPORTED
    # CTA pairs need 256-row weight tiles: N a multiple of 256
    d384 = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 384, 256, 128, 0, 1)
    t2 = hq.Tuning(cta_group=2)
    assert L_.hq_gemm_w4a16(ctypes.byref(d384), 16, 16, 4, 32, ctypes.byref(t2), 256, 1 << 20,
                            None) == hq.HQ_ERR_UNSUPPORTED
    # MXFP4 weights with bf16 activations: no exact-integer variant (INT3 and
    # INT2 weights have one); the block-scaled entry points do not take them
    dx = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4_A16, 256, 256, 32, 0, 1)
    t = hq.Tuning(variant=2)
    assert L_.hq_gemm_w4a16(ctypes.byref(dx), 16, 16, 4, 32, ctypes.byref(t), 256, 1 << 20,
                            None) == hq.HQ_ERR_UNSUPPORTED
    assert L_.hq_gemm_w4a16_static(ctypes.byref(dx), 16, 16, 4, 32, ctypes.byref(t), None) == hq.HQ_ERR_UNSUPPORTED
    assert L_.hq_gemm_mxfp4_a8(ctypes.byref(dx), 4096, 16, 16, 4, 32, None, 256, 1 << 20,
                               None) == hq.HQ_ERR_INVALID_ARG
    dxg = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4_A16, 256, 256, 32, 0, 8)
    assert L_.hq_grouped_gemm_moe(ctypes.byref(dxg), 16, 16, 16, 40, 32, ctypes.byref(t), 256, 1 << 20,
                                  None) == hq.HQ_ERR_UNSUPPORTED
    assert L_.hq_gemm_w4a16(ctypes.byref(dxg), 16, 16, 4, 32, None, 256, 1 << 20, None) == hq.HQ_ERR_INVALID_ARG
    dm = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, 256, 256, 32, 0, 1)
    t = hq.Tuning(variant=1)
    assert L_.hq_gemm_mxfp4_a8(ctypes.byref(dm), 4096, 16, 16, 4, 32, ctypes.byref(t), 256, 1 << 20,
                               None) == hq.HQ_ERR_UNSUPPORTED
    # CTA pairs (cta_group 2): 256-row weight tiles (N a multiple of 256),
    # 128- or 256-token tiles, whole tiles (no K split); no third group
    dm2 = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, 384, 256, 32, 0, 1)
    dn2 = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, 256, 256, 16, 0, 1)
    for dd, bad in ((dm2, hq.Tuning(cta_group=2)), (dm, hq.Tuning(cta_group=2, tile_m=64)),
                    (dm, hq.Tuning(cta_group=2, split_k=2)), (dm, hq.Tuning(cta_group=3))):
        assert L_.hq_gemm_mxfp4_a8(ctypes.byref(dd), 4096, 16, 16, 4, 32, ctypes.byref(bad), 256, 1 << 20,
                                   None) == hq.HQ_ERR_UNSUPPORTED
    bad = hq.Tuning(cta_group=2, tile_m=32)
    assert L_.hq_gemm_nvfp4(ctypes.byref(dn2), 4096, 16, 16, ctypes.c_float(1.0), 4, 32, ctypes.byref(bad), 256,
                            1 << 20, None) == hq.HQ_ERR_UNSUPPORTED
    # routing arguments
    assert L_.hq_moe_topk(None, 4, 8, 0, None, None) == hq.HQ_ERR_INVALID_ARG
    assert L_.hq_moe_topk(None, 4, 4, 8, None, None) == hq.HQ_ERR_INVALID_ARG
    assert L_.hq_debug_timeout_probe(256, 10 ** 9, None) == hq.HQ_ERR_INVALID_ARG


def test_moe_layer_argument_errors_need_no_gpu():
    L_ = hq.lib()
    # routing with weights
    assert L_.hq_moe_topk_softmax(None, 0, 8, 2, None, None, None) == hq.HQ_OK
    assert L_.hq_moe_topk_softmax(None, 4, 8, 0, None, None, None) == hq.HQ_ERR_INVALID_ARG
    assert L_.hq_moe_topk_softmax(16, 4, 8, 2, 16, None, None) == hq.HQ_ERR_INVALID_ARG
    assert L_.hq_moe_topk_softmax(16, 4, 8, 2, 16, 18, None) == hq.HQ_ERR_ALIGNMENT
    # SwiGLU
    assert L_.hq_moe_swiglu(None, 0, 64, None, None) == hq.HQ_OK
    assert L_.hq_moe_swiglu(16, 4, 60, 16, None) == hq.HQ_ERR_INVALID_ARG
    assert L_.hq_moe_swiglu(None, 4, 64, 16, None) == hq.HQ_ERR_INVALID_ARG
    assert L_.hq_moe_swiglu(16, 4, 64, 24, None) == hq.HQ_ERR_ALIGNMENT
    # combine
    need = hq.hq_moe_combine_workspace_size(10, 8)
    assert need >= 256 + 4 * 10 * 8
    assert L_.hq_moe_combine(None, None, None, 0, 8, 64, None, None, 0, None) == hq.HQ_OK
    assert L_.hq_moe_combine(16, 16, 16, 10, 17, 64, 16, 256, need, None) == hq.HQ_ERR_INVALID_ARG
    assert L_.hq_moe_combine(16, 16, 16, 10, 8, 60, 16, 256, need, None) == hq.HQ_ERR_INVALID_ARG
    assert L_.hq_moe_combine(16, 16, 16, 10, 8, 64, 24, 256, need, None) == hq.HQ_ERR_ALIGNMENT
    assert L_.hq_moe_combine(16, 16, 16, 10, 8, 64, 16, 256, need - 1, None) == hq.HQ_ERR_WORKSPACE_TOO_SMALL


def test_workspace_size_is_deterministic_and_covers_header():
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 7168, 18432, 128, 0, 1)
    a = hq.hq_workspace_size(d, 16)
    assert a == hq.hq_workspace_size(d, 16) and a >= 256
    assert hq.hq_workspace_size(d, 4096) >= 256


def test_status_strings():
    for s in range(10):
        assert hq.status_string(s)


def test_autotune_candidates_need_no_gpu():
    from quantized_gemm_bit_b200 import autotune
    c = autotune.candidates("w4a16", 16)
    assert c[0] is None and all(t.tile_m in (16, 32) for t in c[1:])
    assert not any(t.variant == 2 and t.tile_m > 64 for t in autotune.candidates("w4a16", 4096)[1:])
    assert all(t.variant == 0 for t in autotune.candidates("nvfp4", 256)[1:])
    assert all(t.variant == 1 for t in autotune.candidates("mxfp4_a16", 16)[1:])
    assert {t.variant for t in autotune.candidates("w3a16", 64)[1:]} == {1, 2}
    assert {t.stages for t in autotune.candidates("w4a16", 16)[1:]} == set(autotune.STAGES)
    assert {t.variant for t in autotune.candidates("w2a16", 16)[1:]} == {1, 2}
    assert all(t.split_k == 0 for t in autotune.candidates("moe", 64)[1:])


@pytest.mark.parametrize("fmt", [hq.HQ_FMT_INT4, hq.HQ_FMT_INT3, hq.HQ_FMT_INT2, hq.HQ_FMT_MXFP4_A16])
@pytest.mark.parametrize("experts", [1, 3])
def test_gated_pack_matches_oracle_row_order(fmt, experts):
    """hq_pack_weights_gated equals the format's oracle layout of the rows
    taken in the gated gate+up order, bit for bit."""
    n, k = 256, 256
    ex = experts if experts > 1 else None
    perm = L.gated_source_rows(n)
    if fmt == hq.HQ_FMT_MXFP4_A16:
        codes, e8 = synth.mxfp4_weights(n, k, seed=31, experts=ex)
        d = hq.hq_quant_desc_init(fmt, n, k, 32, 0, experts)
        blob = hq.hq_pack_weights_gated(d, codes, e8)
        cn, en = codes.numpy().reshape(experts, n, -1), e8.numpy().reshape(experts, n, -1)
        ref = np.concatenate([L.mxa16_pack(cn[e][perm], en[e][perm]) for e in range(experts)])
    else:
        make, pack = {hq.HQ_FMT_INT4: (synth.w4a16_weights, L.w4a16_pack),
                      hq.HQ_FMT_INT3: (synth.w3a16_weights, L.w3a16_pack),
                      hq.HQ_FMT_INT2: (synth.w2a16_weights, L.w2a16_pack)}[fmt]
        q, s, z = make(n, k, 128, True, seed=32, experts=ex)
        d = hq.hq_quant_desc_init(fmt, n, k, 128, 1, experts)
        blob = hq.hq_pack_weights_gated(d, q, s, z)
        qn, sn, zn = (x.numpy().reshape(experts, n, -1) for x in (q, s, z))
        ref = np.concatenate([pack(qn[e][perm], sn[e][perm], zn[e][perm]) for e in range(experts)])
    assert np.array_equal(blob, ref)


def test_gated_pack_and_fused_swiglu_argument_errors():
    L_ = hq.lib()
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 192, 256, 128, 0, 4)       # n % 128 != 0
    assert L_.hq_pack_weights_gated(ctypes.byref(d), 16, 16, None, 16, 1 << 30) == hq.HQ_ERR_UNSUPPORTED
    assert L_.hq_grouped_gemm_moe_swiglu(ctypes.byref(d), 16, 16, 16, 40, 16, None, 256, 1 << 20,
                                         None) == hq.HQ_ERR_UNSUPPORTED
    dn = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, 256, 256, 16, 0, 1)
    assert L_.hq_pack_weights_gated(ctypes.byref(dn), 16, 16, None, 16, 1 << 30) == hq.HQ_ERR_UNSUPPORTED
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 256, 256, 128, 0, 4)
    assert L_.hq_grouped_gemm_moe_swiglu(ctypes.byref(d), 16, 16, 16, 0, 16, None, 256, 1 << 20, None) == hq.HQ_OK
    assert L_.hq_grouped_gemm_moe_swiglu(ctypes.byref(d), 16, 16, 16, 40, 24, None, 256, 1 << 20,
                                         None) == hq.HQ_ERR_ALIGNMENT
    d1 = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 256, 256, 128, 0, 1)     # dense: not grouped
    assert L_.hq_grouped_gemm_moe_swiglu(ctypes.byref(d1), 16, 16, 16, 40, 16, None, 256, 1 << 20,
                                         None) == hq.HQ_ERR_INVALID_ARG


@pytest.mark.parametrize("n,k,asym,experts", [(256, 384, False, 1), (200, 256, True, 1), (136, 256, True, 3)])
def test_int8_pack_matches_oracle_layout(n, k, asym, experts):
    q, s, z = synth.w8a16_weights(n, k, 128, asym, seed=n + 8, experts=experts if experts > 1 else None)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT8, n, k, 128, int(asym), experts)
    blob = hq.hq_pack_weights(d, q, s, z)
    assert blob.size == L.w8a16_packed_bytes(n, k, asym, experts)
    qn, sn = q.numpy(), s.numpy()
    zn = None if z is None else z.numpy()
    if experts == 1:
        ref = L.w8a16_pack(qn, sn, zn)
    else:
        ref = np.concatenate([L.w8a16_pack(qn[e], sn[e], None if zn is None else zn[e]) for e in range(experts)])
    assert np.array_equal(blob, ref)


@pytest.mark.parametrize("n,k,experts", [(128, 128, 1), (300, 384, 1), (136, 256, 3)])
def test_mxint4_pack_matches_oracle_layout(n, k, experts):
    codes, e8 = synth.mxint4_weights(n, k, seed=n + k + 4, experts=experts if experts > 1 else None)
    if experts == 1:
        # the whole scale range the packer accepts
        e8 = torch.from_numpy(np.random.default_rng(n).integers(0, 252, size=(n, k // 32), dtype=np.uint8))
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXINT4, n, k, 32, 0, experts)
    blob = hq.hq_pack_weights(d, codes, e8)
    assert blob.size == L.mxi4_packed_bytes(n, k, experts)
    cn, en = codes.numpy(), e8.numpy()
    if experts == 1:
        ref = L.mxi4_pack(cn, en)
    else:
        ref = np.concatenate([L.mxi4_pack(cn[e], en[e]) for e in range(experts)])
    assert np.array_equal(blob, ref)


def test_mxint4_pack_rejects_scales_that_overflow_bf16_and_descriptor_rules():
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXINT4, 128, 128, 32, 0, 1)
    codes, e8 = synth.mxint4_weights(128, 128, seed=9)
    e8 = e8.clone()
    e8[3, 1] = 252
    with pytest.raises(hq.HQError) as e:
        hq.hq_pack_weights(d, codes, e8)
    assert e.value.status == hq.HQ_ERR_INVALID_ARG
    for args, code in (((hq.HQ_FMT_MXINT4, 128, 128, 16, 0, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_MXINT4, 128, 128, 32, 1, 1), hq.HQ_ERR_UNSUPPORTED),
                       ((hq.HQ_FMT_INT8, 128, 100, 128, 0, 1), hq.HQ_ERR_UNSUPPORTED)):
        with pytest.raises(hq.HQError) as e:
            hq.hq_quant_desc_init(*args)
        assert e.value.status == code
    # MXINT4 has no exact-integer variant (one scale per 32 K)
    L_ = hq.lib()
    t = hq.Tuning(variant=2)
    assert L_.hq_gemm_w4a16(ctypes.byref(d), 16, 16, 4, 32, ctypes.byref(t), 256, 1 << 20,
                            None) == hq.HQ_ERR_UNSUPPORTED


def test_split_plans_fit_the_workspace_counter_region():
    """Stream-K tile counters live in a fixed 256 KiB region after the
    256-byte header (4 per tile for W4A16, 8 for the block-scaled GEMMs):
    a split request on more tiles than that holds runs as whole tiles, and
    every scratch area starts past the region."""
    header, region = 256, 256 << 10
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 18432, 7168, 128, 0, 1)
    t = hq.Tuning(tile_m=16, split_k=2, variant=2)
    p = hq.hq_plan_describe(d, 16, t)
    assert p.split == 2 and p.workspace_bytes == header + region + p.grid * 2 * 16 * 128 * 4
    # the register path (M <= 16): one 8 KiB fp32 partial tile per CTA
    pr = hq.hq_plan_describe(d, 16, hq.Tuning(split_k=2, variant=3))
    assert (pr.kernel, pr.split, pr.grid) == (4, 2, 2 * 144)
    assert pr.workspace_bytes == header + region + pr.grid * 8192
    assert hq.hq_plan_describe(d, 16 * 113, t).split == 2          # 16272 tiles
    big = hq.hq_plan_describe(d, 16 * 114, t)                      # 16416 tiles
    assert (big.split, big.workspace_bytes) == (0, header)
    dm = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, 18432, 7168, 32, 0, 1)
    tb = hq.Tuning(tile_m=16, split_k=2)
    assert hq.hq_plan_describe(dm, 16 * 56, tb).split == 2         # 8064 tiles
    assert hq.hq_plan_describe(dm, 16 * 57, tb).split == 0         # 8208 tiles
    dn = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, 8192, 8192, 16, 0, 1)
    pn = hq.hq_plan_describe(dn, 8192)
    assert pn.split == 0 and pn.workspace_bytes > header + region  # re-laid scales past the region
    assert hq.hq_moe_combine_workspace_size(10, 8) >= header + region + 4 * 10 * 8
    assert hq.hq_moe_permute_workspace_size(64, 8, 256) > header + region
    assert hq.hq_quantize_nvfp4_workspace_size(64, 1024) > header + region


def test_grouped_token_tile_rule():
    """Grouped GEMMs: the token tile covers a typical expert's rows (avg +
    2 sd of Poisson(avg) rows per expert); above 128 it is 256 only for K of
    at least 4096 and at most 511 experts (the 256-token tile's output
    transposes sit beside the expert tables), else 128.  INT4 experts whose
    typical rows fit 8 tokens run on the register path (8-token units)."""
    def plan(n, k, e, rows, fmt=hq.HQ_FMT_INT4):
        d = hq.hq_quant_desc_init(fmt, n, k, 128, 0, e)
        return hq.hq_plan_describe(d, rows)
    def tile(n, k, e, rows):
        return plan(n, k, e, rows).tile_m
    p64 = plan(4096, 7168, 256, 64 * 8)                 # T=64, top-8 of 256: 2 rows per expert
    assert (p64.kernel, p64.tile_m, p64.grid) == (4, 8, 148 * 3)
    p64i3 = plan(4096, 7168, 256, 64 * 8, hq.HQ_FMT_INT3)   # INT3: no register path, 16-token tiles
    assert (p64i3.kernel, p64i3.tile_m) == (2, 16)
    assert tile(4096, 7168, 256, 1024 * 8) == 64        # 32 rows per expert
    assert tile(4096, 7168, 256, 8192 * 8) == 256       # 256 rows per expert, long K
    assert tile(7168, 2048, 256, 8192 * 8) == 128       # short K
    assert tile(4096, 7168, 600, 600 * 256) == 128      # tables too large for the transposes
    assert tile(4096, 7168, 256, 256 * 150) == 128      # 150 + 2 sd <= 192


def test_tuning_table_entry_changes_the_plan():
    """A table entry replaces the library's rules for calls without a tuning
    of its shape and m range; an explicit tuning still wins; clearing the
    table restores the rules.  The workspace size follows the plan."""
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 18432, 7168, 128, 0, 1)
    base16 = hq.hq_plan_describe(d, 16)
    assert (base16.tile_m, base16.kernel, base16.from_table) == (16, 4, 0)      # the register path
    assert base16.stages == base16.ring_stages >= 2
    base64 = hq.hq_plan_describe(d, 64)
    entry = {"fmt": hq.HQ_FMT_INT4, "n": 18432, "k": 7168, "num_experts": 1, "m_min": 1, "m_max": 32,
             "tuning": {"tile_m": 32, "variant": 1, "stages": 3, "split_k": 2}}
    try:
        hq.hq_tuning_table_set([entry])
        p = hq.hq_plan_describe(d, 16)
        assert (p.tile_m, p.kernel, p.stages, p.from_table) == (32, 1, 3, 1)
        assert p.split == 2 and p.grid == 2 * 144
        assert hq.hq_workspace_size(d, 16) == p.workspace_bytes != base16.workspace_bytes
        p64 = hq.hq_plan_describe(d, 64)                    # outside the entry's m range
        assert (p64.tile_m, p64.kernel, p64.from_table) == (base64.tile_m, base64.kernel, 0)
        pe = hq.hq_plan_describe(d, 16, hq.Tuning(tile_m=16))   # an explicit tuning wins
        assert (pe.tile_m, pe.from_table) == (16, 0)
        d2 = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 18432, 7168, 128, 1, 1)   # zero points: same shape key
        assert hq.hq_plan_describe(d2, 16).from_table == 1
        d3 = hq.hq_quant_desc_init(hq.HQ_FMT_INT3, 18432, 7168, 128, 0, 1)   # another format: not matched
        assert hq.hq_plan_describe(d3, 16).from_table == 0
        # a bad entry is refused and leaves the table as it was
        bad = dict(entry, tuning={"tile_m": 48})
        with pytest.raises(hq.HQError) as e:
            hq.hq_tuning_table_set([bad])
        assert e.value.status == hq.HQ_ERR_UNSUPPORTED
        assert hq.hq_plan_describe(d, 16).from_table == 1
        # block-scaled entries go to that planner
        dm = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, 7168, 7168, 32, 0, 1)
        hq.hq_tuning_table_set([entry, {"fmt": hq.HQ_FMT_MXFP4, "n": 7168, "k": 7168, "m_min": 200, "m_max": 300,
                                        "tuning": {"tile_m": 256, "stages": 2}}])
        pm = hq.hq_plan_describe(dm, 256)
        assert (pm.kernel, pm.tile_m, pm.stages, pm.from_table) == (3, 256, 2, 1)
    finally:
        hq.hq_tuning_table_set([])
    assert hq.hq_plan_describe(d, 16).from_table == 0


def test_stages_above_the_ring_mean_the_whole_ring():
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 4096, 4096, 128, 0, 1)
    p = hq.hq_plan_describe(d, 256, hq.Tuning(stages=99))
    assert p.stages == p.ring_stages
    p = hq.hq_plan_describe(d, 256, hq.Tuning(stages=2))
    assert p.stages == 2 < p.ring_stages or p.ring_stages == 2
