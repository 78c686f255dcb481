"""GPU parity of the block-scaled 4-bit GEMMs (through the C ABI) against
the fp64 oracle: W4A8-MXFP4 (E2M1 weights, E8M0 per 32 K, E4M3 activations
with per-token scale) and W4A4 NVFP4 (E2M1, E4M3 per 16 K, fp32 tensor
scales).  Full outputs on small shapes spanning tiles and ragged tails;
sampled rows and columns at the full workload sizes."""

import numpy as np
import pytest
import torch

from gpu_helpers import check_gemm, tile_rows, workspace
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


# ---------------------------------------------------------------- MXFP4 x FP8

def mx_case(m, n, k, seed):
    codes, e8 = synth.mxfp4_weights(n, k, seed=seed)
    # E4M3 activations from the oracle's per-token quantizer (amax / 448)
    aq, asc = (torch.from_numpy(v) for v in F.fp8_per_token_quantize(
        synth.bf16_normal(m, k, seed=seed + 1).float().numpy()))
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, n, k, 32, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(DEV)
    return d, blob, aq, asc, codes.numpy(), e8.numpy()


def mx_run(d, blob, aq, asc, m, tuning=None):
    c = torch.empty(m, d.n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m, tuning))
    hq.hq_gemm_mxfp4_a8(d, blob, aq.to(DEV), asc.to(DEV), m, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    return c


@pytest.mark.parametrize("m,n,k", [(16, 256, 512), (5, 200, 384), (70, 384, 1024), (300, 256, 640), (33, 130, 512)])
def test_mxfp4_full_output(m, n, k):
    d, blob, aq, asc, codes, e8 = mx_case(m, n, k, 200 + m)
    c = mx_run(d, blob, aq, asc, m)
    ref = G.mxfp4_a8_ref(aq.numpy(), asc.numpy(), codes, e8)
    check_gemm(c, ref, k, f"mxfp4 m={m} n={n} k={k}")


@pytest.mark.parametrize("tile_m", [16, 32, 64, 128, 256])
def test_mxfp4_every_token_tile(tile_m):
    m, n, k = 90, 256, 1024
    d, blob, aq, asc, codes, e8 = mx_case(m, n, k, 300)
    c = mx_run(d, blob, aq, asc, m, hq.Tuning(tile_m=tile_m))
    check_gemm(c, G.mxfp4_a8_ref(aq.numpy(), asc.numpy(), codes, e8), k, f"mxfp4 tile_m={tile_m}")


@pytest.mark.parametrize("tile_m,splits", [(16, 3), (64, 2), (256, 2)])
def test_mxfp4_split_k_repeats_bit_for_bit(tile_m, splits):
    m, n, k = 200, 384, 1024
    d, blob, aq, asc, codes, e8 = mx_case(m, n, k, 310)
    t = hq.Tuning(tile_m=tile_m, split_k=splits)
    c1 = mx_run(d, blob, aq, asc, m, t)
    c2 = mx_run(d, blob, aq, asc, m, t)
    assert torch.equal(c1, c2)
    check_gemm(c1, G.mxfp4_a8_ref(aq.numpy(), asc.numpy(), codes, e8), k, f"mxfp4 split {tile_m}x{splits}")


@pytest.mark.parametrize("m", [16, 256, 4096])
def test_mxfp4_full_size(m):
    """W4A8-MXFP4 workload: K = N = 7168, seeds per shape."""
    n = k = 7168
    d, blob, aq, asc, codes, e8 = mx_case(m, n, k, 2000 + m)
    c = mx_run(d, blob, aq, asc, m)
    rows = tile_rows(m, 128, np.random.default_rng(m))
    ref = G.mxfp4_a8_ref(aq.numpy(), asc.numpy(), codes, e8, rows=rows)
    check_gemm(c[torch.from_numpy(rows).to(DEV)], ref, k, f"mxfp4 full m={m}")


# ---------------------------------------------------------------- NVFP4 W4A4

def nv_quant(rows, k, seed):
    x = synth.bf16_normal(rows, k, seed).float().numpy()
    codes, sf, g = F.nvfp4_quantize(x)
    return F.fp4_pack_bytes(codes), sf, g


def nv_case(m, n, k, seed):
    wp, wsf, wg = nv_quant(n, k, seed)
    ap, asf, ag = nv_quant(m, k, seed + 1)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, n, k, 16, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, wp, wsf, None, float(wg))).to(DEV)
    return d, blob, (ap, asf, ag), (wp, wsf, wg)


def nv_run(d, blob, act, m, tuning=None):
    ap, asf, ag = act
    c = torch.empty(m, d.n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m, tuning))
    hq.hq_gemm_nvfp4(d, blob, torch.from_numpy(ap).to(DEV), torch.from_numpy(asf).to(DEV), float(ag), m, c, ws,
                     tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    return c


@pytest.mark.parametrize("m,n,k", [(16, 256, 512), (7, 200, 768), (130, 384, 1024), (300, 128, 256),
                                   (33, 130, 512)])
def test_nvfp4_full_output(m, n, k):
    d, blob, act, w = nv_case(m, n, k, 400 + m)
    c = nv_run(d, blob, act, m)
    ref = G.nvfp4_ref(*act, *w)
    check_gemm(c, ref, k, f"nvfp4 m={m} n={n} k={k}")


@pytest.mark.parametrize("tile_m", [16, 32, 64, 128, 256])
def test_nvfp4_every_token_tile(tile_m):
    m, n, k = 200, 256, 1024
    d, blob, act, w = nv_case(m, n, k, 500)
    c = nv_run(d, blob, act, m, hq.Tuning(tile_m=tile_m))
    check_gemm(c, G.nvfp4_ref(*act, *w), k, f"nvfp4 tile_m={tile_m}")


@pytest.mark.parametrize("tile_m,splits", [(16, 3), (128, 2), (256, 2)])
def test_nvfp4_split_k_repeats_bit_for_bit(tile_m, splits):
    m, n, k = 300, 256, 1536
    d, blob, act, w = nv_case(m, n, k, 510)
    t = hq.Tuning(tile_m=tile_m, split_k=splits)
    c1 = nv_run(d, blob, act, m, t)
    c2 = nv_run(d, blob, act, m, t)
    assert torch.equal(c1, c2)
    check_gemm(c1, G.nvfp4_ref(*act, *w), k, f"nvfp4 split {tile_m}x{splits}")


@pytest.mark.parametrize("m,n,k", [(8192, 8192, 8192), (16384, 18432, 7168)])
def test_nvfp4_full_size(m, n, k):
    """NVFP4 W4A4 large-batch workload, sampled rows and columns."""
    d, blob, act, w = nv_case(m, n, k, 4000 + (0 if m == 8192 else 1))
    c = nv_run(d, blob, act, m)
    rng = np.random.default_rng(m)
    rows = tile_rows(m, 256, rng, per_tile=1)
    cols = np.array(sorted({c0 for nt in range(n // 128)
                            for c0 in (nt * 128, nt * 128 + 127, nt * 128 + int(rng.integers(0, 128)))}))
    ref = G.nvfp4_ref(*act, *w, rows=rows, cols=cols)
    got = c[torch.from_numpy(rows).to(DEV)][:, torch.from_numpy(cols).to(DEV)]
    check_gemm(got, ref, k, f"nvfp4 full m={m} n={n} k={k}")


# ---------------------------------------------------------------- CTA pairs (cta_group::2)

@pytest.mark.parametrize("tile_m", [128, 256])
@pytest.mark.parametrize("m,n,k", [(300, 512, 1024), (129, 768, 640)])
def test_mxfp4_cta_pairs(m, n, k, tile_m):
    """256-row weight tiles on CTA pairs (cta_group::2 MMAs, each CTA
    staging its 128 weight rows and half of the token tile): every output
    against the oracle, a ragged last token tile, and the same call twice
    gives the same bits."""
    d, blob, aq, asc, codes, e8 = mx_case(m, n, k, 600 + m)
    t = hq.Tuning(tile_m=tile_m, cta_group=2)
    c1 = mx_run(d, blob, aq, asc, m, t)
    c2 = mx_run(d, blob, aq, asc, m, t)
    assert torch.equal(c1, c2)
    check_gemm(c1, G.mxfp4_a8_ref(aq.numpy(), asc.numpy(), codes, e8), k, f"mxfp4 pairs {tile_m} m={m} n={n}")


@pytest.mark.parametrize("tile_m", [128, 256])
@pytest.mark.parametrize("m,n,k", [(300, 512, 1024), (129, 768, 1536)])
def test_nvfp4_cta_pairs(m, n, k, tile_m):
    d, blob, act, w = nv_case(m, n, k, 700 + m)
    t = hq.Tuning(tile_m=tile_m, cta_group=2)
    c1 = nv_run(d, blob, act, m, t)
    c2 = nv_run(d, blob, act, m, t)
    assert torch.equal(c1, c2)
    check_gemm(c1, G.nvfp4_ref(*act, *w), k, f"nvfp4 pairs {tile_m} m={m} n={n}")


def test_cta_pairs_more_tiles_than_clusters():
    """More (token tile, 256-row weight tile) units than resident clusters:
    every cluster runs several units, accumulators alternating."""
    m, n, k = 1100, 4096, 512
    d, blob, act, w = nv_case(m, n, k, 720)
    c = nv_run(d, blob, act, m, hq.Tuning(tile_m=128, cta_group=2))
    rows = tile_rows(m, 128, np.random.default_rng(5))
    ref = G.nvfp4_ref(*act, *w, rows=rows)
    check_gemm(c[torch.from_numpy(rows).to(DEV)], ref, k, "nvfp4 pairs, many units")


@pytest.mark.parametrize("m,n,k", [(8192, 8192, 8192)])
def test_nvfp4_one_cta_per_tile_full_size(m, n, k):
    """The library runs this size on CTA pairs; one CTA per 128-row weight
    tile (cta_group 1) must give the same results."""
    d, blob, act, w = nv_case(m, n, k, 4000)
    plan = hq.hq_plan_describe(d, m, hq.Tuning(cta_group=1))
    assert plan.tile_m == 256 and plan.split == 0 and plan.cta_group == 1
    c = nv_run(d, blob, act, m, hq.Tuning(cta_group=1))
    rng = np.random.default_rng(m + 1)
    rows = tile_rows(m, 256, rng, per_tile=1)
    cols = np.array(sorted({c0 for nt in range(n // 128)
                            for c0 in (nt * 128, nt * 128 + 127, nt * 128 + int(rng.integers(0, 128)))}))
    ref = G.nvfp4_ref(*act, *w, rows=rows, cols=cols)
    got = c[torch.from_numpy(rows).to(DEV)][:, torch.from_numpy(cols).to(DEV)]
    check_gemm(got, ref, k, f"nvfp4 one CTA per tile, full m={m} n={n} k={k}")


def test_mxfp4_one_cta_per_tile_full_size():
    m = 4096
    n = k = 7168
    d, blob, aq, asc, codes, e8 = mx_case(m, n, k, 2000 + m)
    c = mx_run(d, blob, aq, asc, m, hq.Tuning(cta_group=1))
    rows = tile_rows(m, 128, np.random.default_rng(m + 1))
    ref = G.mxfp4_a8_ref(aq.numpy(), asc.numpy(), codes, e8, rows=rows)
    check_gemm(c[torch.from_numpy(rows).to(DEV)], ref, k, f"mxfp4 one CTA per tile, full m={m}")


def test_large_tiles_default_to_cta_pairs():
    """The plan the full-size workloads run: 256-token whole tiles on CTA
    pairs (grid = two CTAs per resident cluster)."""
    d = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, 8192, 8192, 16, 0, 1)
    plan = hq.hq_plan_describe(d, 8192)
    assert (plan.tile_m, plan.split, plan.cta_group, plan.grid % 2) == (256, 0, 2, 0)
    assert hq.hq_plan_describe(d, 8192, hq.Tuning(cta_group=1)).cta_group == 1


def test_workspace_shared_across_entry_points_and_plans():
    """One workspace serves, in turn, NVFP4 calls (whose re-laid activation
    scales stay behind as scratch, split or not) and MXFP4 split-K calls of
    different plans: the tile counters sit in the fixed region after the
    256-byte header, which every completed call leaves at zero, and no
    call keeps data there."""
    n, k = 512, 2048
    codes, e8 = synth.mxfp4_weights(n, k, seed=740)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, n, k, 32, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(DEV)
    dn, nblob, nact, nw = nv_case(300, 256, 1536, 745)
    ws = workspace(1 << 24)
    counter_region = ws[:256 + (256 << 10)]
    for step, (m, t) in enumerate([(None, None), (16, hq.Tuning(tile_m=16, split_k=3)),
                                   (None, hq.Tuning(tile_m=16, split_k=3)), (200, hq.Tuning(tile_m=16, split_k=3)),
                                   (16, hq.Tuning(tile_m=64, split_k=2))]):
        if m is None:
            ap, asf, ag = nact
            c = torch.empty(300, dn.n, dtype=torch.bfloat16, device=DEV)
            assert hq.hq_workspace_size(dn, 300, t) <= ws.numel()
            hq.hq_gemm_nvfp4(dn, nblob, torch.from_numpy(ap).to(DEV), torch.from_numpy(asf).to(DEV), float(ag), 300,
                             c, ws, t)
            assert hq.hq_check_device_status(ws) == hq.HQ_OK
            check_gemm(c, G.nvfp4_ref(*nact, *nw), 1536, f"nvfp4 shared workspace step {step}")
        else:
            aq, asc = F.fp8_per_token_quantize(synth.bf16_normal(m, k, 741 + m).float().numpy())
            c = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
            assert hq.hq_workspace_size(d, m, t) <= ws.numel()
            hq.hq_gemm_mxfp4_a8(d, blob, torch.from_numpy(aq).to(DEV), torch.from_numpy(asc).to(DEV), m, c, ws, t)
            assert hq.hq_check_device_status(ws) == hq.HQ_OK
            check_gemm(c, G.mxfp4_a8_ref(aq, asc, codes.numpy(), e8.numpy()), k, f"mxfp4 shared workspace step {step}")
        assert torch.count_nonzero(counter_region) == 0
    assert torch.count_nonzero(ws) > 0      # scratch stays behind, past the counters
