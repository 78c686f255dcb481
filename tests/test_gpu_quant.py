"""GPU activation quantizers (through the C ABI) against the oracle's
quantizers: codes, block scales and tensor/row scales must match bit for
bit (both sides decide every code in fp32 with round-to-nearest-even)."""

import numpy as np
import pytest
import torch

from gpu_helpers import workspace
from oracle import formats as F
from quantized_gemm_bit_b200 import hq, synth
from quantized_gemm_bit_b200.build import build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    build()
    torch.cuda.init()


def _inputs(rows, k, seed, special=False):
    x = synth.bf16_normal(rows, k, seed)
    if special:
        x[0] = 0                                    # an all-zero row / blocks
        x[1, :16] = torch.tensor([0.25, -0.25, 3.0, -5.0] * 4, dtype=torch.bfloat16) * 2 ** -3
        x[2] = x[2] * 1e4                           # a row with large values
        x[3, 5] = -0.0
    return x


@pytest.mark.parametrize("rows,k,special", [(1, 64, False), (16, 7168, False), (37, 1024, True), (4096, 7168, False)])
def test_fp8_rows_bit_exact(rows, k, special):
    x = _inputs(rows, k, 7000 + rows, special)
    q = torch.empty(rows, k, dtype=torch.uint8, device=DEV)
    s = torch.empty(rows, dtype=torch.float32, device=DEV)
    hq.hq_quantize_fp8_rows(x.to(DEV), rows, k, q, s)
    q_ref, s_ref = F.fp8_per_token_quantize(x.float().numpy())
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("rows,k,special", [(1, 16, False), (16, 512, True), (200, 1024, False),
                                            (8192, 8192, False)])
def test_nvfp4_bit_exact(rows, k, special):
    x = _inputs(rows, k, 7100 + rows, special)
    codes = torch.empty(rows, k // 2, dtype=torch.uint8, device=DEV)
    sf = torch.empty(rows, k // 16, dtype=torch.uint8, device=DEV)
    g = torch.empty(1, dtype=torch.float32, device=DEV)
    ws = workspace(hq.hq_quantize_nvfp4_workspace_size(rows, k))
    hq.hq_quantize_nvfp4(x.to(DEV), rows, k, codes, sf, g, ws)
    c_ref, sb_ref, g_ref = F.nvfp4_quantize(x.float().numpy())
    assert g.cpu().numpy().view(np.uint32)[0] == np.float32(g_ref).view(np.uint32)
    assert np.array_equal(sf.cpu().numpy(), sb_ref)
    assert np.array_equal(codes.cpu().numpy(), F.fp4_pack_bytes(c_ref))


def test_quantized_activations_feed_the_nvfp4_gemm():
    """GPU-quantized activations through the NVFP4 GEMM equal the oracle's
    GEMM on the oracle-quantized activations (identical codes)."""
    from gpu_helpers import check_gemm
    from oracle import gemm as G
    m, n, k = 48, 256, 1024
    x = _inputs(m, k, 7200)
    codes = torch.empty(m, k // 2, dtype=torch.uint8, device=DEV)
    sf = torch.empty(m, k // 16, dtype=torch.uint8, device=DEV)
    g = torch.empty(1, dtype=torch.float32, device=DEV)
    hq.hq_quantize_nvfp4(x.to(DEV), m, k, codes, sf, g, workspace(hq.hq_quantize_nvfp4_workspace_size(m, k)))
    wx = synth.bf16_normal(n, k, 7201).float().numpy()
    wc, wsb, wg = F.nvfp4_quantize(wx)
    wp = F.fp4_pack_bytes(wc)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, n, k, 16, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, wp, wsb, None, float(wg))).to(DEV)
    c = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m))
    hq.hq_gemm_nvfp4(d, blob, codes, sf, float(g.item()), m, c, ws)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    ac, asb, ag = F.nvfp4_quantize(x.float().numpy())
    ref = G.nvfp4_ref(F.fp4_pack_bytes(ac), asb, ag, wp, wsb, wg)
    check_gemm(c, ref, k, "quantize -> nvfp4 gemm")
