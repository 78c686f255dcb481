"""Back-to-back GEMM calls on one stream, each consuming what the kernel just
before it wrote (the GEMM kernels start early as programmatic dependents of
that kernel and must still read its results): a torch kernel rewrites the
activations, GEMM 1 reads them, GEMM 2 reads GEMM 1's output.  Every result
is checked against the fp64 oracle's own chain (GEMM 2's reference takes the
oracle's GEMM 1 result rounded to bf16) at the GEMM tolerance."""

import numpy as np
import pytest
import torch

from gpu_helpers import check_gemm, workspace
from oracle import formats as F
from oracle import gemm as G
from quantized_gemm_bit_b200 import hq, synth
from quantized_gemm_bit_b200.build import build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    build()
    torch.cuda.init()


def _bits(a):
    return a.view(torch.int16).cpu().numpy().view(np.uint16)


def _w4(n, k, seed):
    q, s, z = synth.w4a16_weights(n, k, 128, True, seed)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 1, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
    return d, blob, (q.numpy(), s.numpy(), z.numpy())


@pytest.mark.parametrize("m,variant", [(16, 0), (16, 2), (48, 0), (48, 2), (300, 0)])
def test_chained_w4a16_calls_read_fresh_inputs(m, variant):
    k1, n1, n2 = 512, 1024, 384
    d1, b1, w1 = _w4(n1, k1, 700 + m)
    d2, b2, w2 = _w4(n2, n1, 710 + m)
    t = hq.Tuning(variant=variant) if variant else None
    reps = 6
    xs = [synth.bf16_normal(m, k1, 720 + m + r).to(DEV) for r in range(reps)]
    x = torch.empty(m, k1, dtype=torch.bfloat16, device=DEV)
    y1 = torch.empty(m, n1, dtype=torch.bfloat16, device=DEV)
    y2 = torch.empty(m, n2, dtype=torch.bfloat16, device=DEV)
    ws1 = workspace(hq.hq_workspace_size(d1, m, t))
    ws2 = workspace(hq.hq_workspace_size(d2, m, t))
    outs = []
    for r in range(reps):
        torch.add(xs[r], 0.0, out=x)                       # a kernel writes the activations
        hq.hq_gemm_w4a16(d1, b1, x, m, y1, ws1, t)         # reads them
        hq.hq_gemm_w4a16(d2, b2, y1, m, y2, ws2, t)        # reads GEMM 1's output
        outs.append((y1.clone(), y2.clone()))
    torch.cuda.synchronize()
    assert hq.hq_check_device_status(ws1) == hq.HQ_OK
    assert hq.hq_check_device_status(ws2) == hq.HQ_OK
    for r, (o1, o2) in enumerate(outs):
        ref1 = G.w4a16_ref(_bits(xs[r]), *w1, 128)
        check_gemm(o1, ref1, k1, f"chain m={m} rep={r} gemm1")
        ref2 = G.w4a16_ref(F.f32_to_bf16_bits_rne(ref1.astype(np.float32)), *w2, 128)
        check_gemm(o2, ref2, n1, f"chain m={m} rep={r} gemm2")


def test_chained_nvfp4_quantize_then_gemm():
    """The activation quantizer writes codes and scales, the scale re-layout
    and the GEMM read them right after."""
    m, n, k = 64, 256, 1024
    x = synth.bf16_normal(n, k, 730).float().numpy()
    wc, wsf, wg = F.nvfp4_quantize(x)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, n, k, 16, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, F.fp4_pack_bytes(wc), wsf, None, float(wg))).to(DEV)
    c = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m))
    codes = torch.empty(m, k // 2, dtype=torch.uint8, device=DEV)
    sf = torch.empty(m, k // 16, dtype=torch.uint8, device=DEV)
    g = torch.empty(1, dtype=torch.float32, device=DEV)
    wsq = workspace(hq.hq_quantize_nvfp4_workspace_size(m, k))
    for r in range(3):
        a_host = synth.bf16_normal(m, k, 740 + r)
        a = a_host.to(DEV)
        hq.hq_quantize_nvfp4(a, m, k, codes, sf, g, wsq)
        # the tensor scale stays on the device: pass it through the host once
        # per call, as a caller would
        torch.cuda.synchronize()
        hq.hq_gemm_nvfp4(d, blob, codes, sf, float(g.item()), m, c, ws)
        got = c.clone()
        torch.cuda.synchronize()
        assert hq.hq_check_device_status(ws) == hq.HQ_OK
        # the oracle's quantizer on the same activations; the GPU's codes,
        # scales and tensor scale equal it bit for bit
        ac, asb, ag = F.nvfp4_quantize(a_host.float().numpy())
        assert np.array_equal(codes.cpu().numpy(), F.fp4_pack_bytes(ac))
        assert np.array_equal(sf.cpu().numpy(), asb) and np.float32(g.item()) == np.float32(ag)
        ref = G.nvfp4_ref(F.fp4_pack_bytes(ac), asb, ag, F.fp4_pack_bytes(wc), wsf, float(wg))
        check_gemm(got, ref, k, f"nvfp4 chain rep={r}")


@pytest.mark.parametrize("m", [16, 300])
def test_weight_writing_kernel_before_gemm_with_no_early_weights(m):
    """A kernel that rewrites the packed weights right before each GEMM call
    (an in-place weight update): with HQ_TUNE_NO_EARLY_WEIGHTS the GEMM reads
    the new weights, every time, for both kernels of the W4A16 family."""
    n, k = 640, 1024
    reps = 4
    packs = []
    for r in range(reps):
        d, blob, w = _w4(n, k, 760 + r)
        packs.append((blob, w))
    blob = torch.empty_like(packs[0][0])
    a = synth.bf16_normal(m, k, 770 + m).to(DEV)
    t = hq.Tuning(flags=hq.HQ_TUNE_NO_EARLY_WEIGHTS)
    ws = workspace(hq.hq_workspace_size(d, m, t))
    outs = []
    for r in range(reps):
        torch.add(packs[r][0], 0, out=blob)                  # a kernel writes the packed weights
        c = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
        hq.hq_gemm_w4a16(d, blob, a, m, c, ws, t)            # reads them
        outs.append(c)
    torch.cuda.synchronize()
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    for r, c in enumerate(outs):
        ref = G.w4a16_ref(_bits(a), *packs[r][1], 128)
        check_gemm(c, ref, k, f"weights rewritten before the call m={m} rep={r}")


def test_weight_writing_kernel_before_block_scaled_gemm_with_no_early_weights():
    """The same for the MXFP4 x FP8 GEMM."""
    m, n, k = 64, 512, 1024
    reps = 3
    packs = []
    for r in range(reps):
        codes, e8 = synth.mxfp4_weights(n, k, seed=780 + r)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, n, k, 32, 0, 1)
        packs.append((torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(DEV), codes.numpy(), e8.numpy()))
    blob = torch.empty_like(packs[0][0])
    aq, asc = F.fp8_per_token_quantize(synth.bf16_normal(m, k, 790).float().numpy())
    aq_d, asc_d = torch.from_numpy(aq).to(DEV), torch.from_numpy(asc).to(DEV)
    t = hq.Tuning(flags=hq.HQ_TUNE_NO_EARLY_WEIGHTS)
    ws = workspace(hq.hq_workspace_size(d, m, t))
    outs = []
    for r in range(reps):
        torch.add(packs[r][0], 0, out=blob)
        c = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
        hq.hq_gemm_mxfp4_a8(d, blob, aq_d, asc_d, m, c, ws, t)
        outs.append(c)
    torch.cuda.synchronize()
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    for r, c in enumerate(outs):
        check_gemm(c, G.mxfp4_a8_ref(aq, asc, packs[r][1], packs[r][2]), k, f"mxfp4 weights rewritten rep={r}")
