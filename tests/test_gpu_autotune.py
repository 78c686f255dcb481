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
    results, best, library, _, _ = autotune.autotune("w4a16", m, n, k, tunings=tunings)
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
    results, best, library, _, _ = autotune.autotune(kind, m, n, k, experts=8, topk=2)
    assert library in results and best["us"] <= library["us"]


@pytest.mark.parametrize("stages", [1, 2, 3])
@pytest.mark.parametrize("tile_m,variant", [(16, 2), (16, 1), (128, 1)])
def test_stages_in_flight_give_the_same_result(tile_m, variant, stages):
    """The pipeline-depth knob (stages in flight) only throttles the
    producer: every depth gives the oracle's result, and the same bits as
    the whole ring."""
    m, n, k = 2 * tile_m - 5, 384, 2048
    q, s, z = synth.w4a16_weights(n, k, 128, True, seed=1100 + tile_m)
    a = synth.bf16_normal(m, k, seed=1101)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 1, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).cuda()
    outs = []
    for st in (0, stages):
        t = hq.Tuning(tile_m=tile_m, variant=variant, stages=st)
        c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        ws = workspace(hq.hq_workspace_size(d, m, t))
        hq.hq_gemm_w4a16(d, blob, a.cuda(), m, c, ws, t)
        assert hq.hq_check_device_status(ws) == hq.HQ_OK
        outs.append(c)
    ref = G.w4a16_ref(a.view(torch.int16).numpy().view(np.uint16), q.numpy(), s.numpy(), z.numpy(), 128)
    check_gemm(outs[1], ref, k, f"stages={stages} tile_m={tile_m} variant={variant}")
    assert torch.equal(outs[0], outs[1])


def test_block_scaled_stages_in_flight():
    m, n, k = 100, 256, 2048
    codes, e8 = synth.mxfp4_weights(n, k, seed=1200)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, n, k, 32, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).cuda()
    from oracle import formats as F
    aq, asc = F.fp8_per_token_quantize(synth.bf16_normal(m, k, 1201).float().numpy())
    outs = []
    for st in (0, 1, 2):
        t = hq.Tuning(stages=st)
        c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        ws = workspace(hq.hq_workspace_size(d, m, t))
        hq.hq_gemm_mxfp4_a8(d, blob, torch.from_numpy(aq).cuda(), torch.from_numpy(asc).cuda(), m, c, ws, t)
        assert hq.hq_check_device_status(ws) == hq.HQ_OK
        outs.append(c)
    check_gemm(outs[1], G.mxfp4_a8_ref(aq, asc, codes.numpy(), e8.numpy()), k, "mxfp4 stages=1")
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_autotuned_table_entry_drives_calls_without_a_tuning(tmp_path):
    """The autotuner's table, installed in the library, changes the plan of
    calls that pass no tuning, and the result is still the oracle's."""
    m, n, k = 16, 512, 1024
    tunings = [None, hq.Tuning(tile_m=32, variant=1, stages=2)]
    results, best, library, d, rows = autotune.autotune("w4a16", m, n, k, tunings=tunings)
    pick = hq.Tuning(tile_m=32, variant=1, stages=2)
    path = str(tmp_path / "table.json")
    autotune.merge_table(path, autotune.table_entry(d, 1, 16, pick))
    try:
        autotune.load_table(path)
        plan = hq.hq_plan_describe(d, m)
        assert (plan.tile_m, plan.kernel, plan.stages, plan.from_table) == (32, 1, 2, 1)
        q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=1000)
        a = synth.bf16_normal(m, k, seed=1001)
        blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).cuda()
        c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        ws = workspace(hq.hq_workspace_size(d, m))
        hq.hq_gemm_w4a16(d, blob, a.cuda(), m, c, ws)
        assert hq.hq_check_device_status(ws) == hq.HQ_OK
        ref = G.w4a16_ref(a.view(torch.int16).numpy().view(np.uint16), q.numpy(), s.numpy(), None, 128)
        check_gemm(c, ref, k, "plan from the tuning table")
    finally:
        hq.hq_tuning_table_set([])
