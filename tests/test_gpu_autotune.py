"""The offline autotuner through the C ABI: it times valid plans, skips the
ones the library refuses, and its pick computes the same GEMM (checked
against the fp64 oracle)."""

import numpy as np
import pytest
import torch

from gpu_helpers import check_gemm, workspace
from oracle import gemm as G
from quantized_gemm_bit_b200 import autotune, hq, synth
from quantized_gemm_bit_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    build()
    torch.cuda.init()


def test_autotune_w4a16_pick_is_valid_and_correct():
    m, n, k = 16, 512, 512
    tunings = [None, hq.Tuning(tile_m=16, split_k=1, variant=1), hq.Tuning(tile_m=16, split_k=2, variant=1),
               hq.Tuning(tile_m=32, variant=2), hq.Tuning(tile_m=48)]          # 48: refused, skipped
    results, best, library = autotune.autotune("w4a16", m, n, k, tunings=tunings)
    assert len(results) == 4 and library["tuning"] is None
    assert all(r["us"] > 0 for r in results) and best["us"] == min(r["us"] for r in results)
    # the same inputs the autotuner used, through the picked plan
    q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=1000)
    a = synth.bf16_normal(m, k, seed=1001)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).cuda()
    c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ws = workspace(hq.hq_workspace_size(d, m, best["tuning"]))
    hq.hq_gemm_w4a16(d, blob, a.cuda(), m, c, ws, best["tuning"])
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    ref = G.w4a16_ref(a.view(torch.int16).numpy().view(np.uint16), q.numpy(), s.numpy(), None, 128)
    check_gemm(c, ref, k, f"autotuned {best['desc']}")


@pytest.mark.parametrize("kind", ["mxfp4", "moe"])
def test_autotune_other_kinds_run(kind):
    m, n, k = (64, 256, 512) if kind == "mxfp4" else (32, 256, 256)
    results, best, library = autotune.autotune(kind, m, n, k, experts=8, topk=2)
    assert library in results and best["us"] <= library["us"]
