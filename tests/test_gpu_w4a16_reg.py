"""GPU parity of the register-path W4A16 kernel (tuning variant 3: dense
INT4 at 1..16 tokens, codes dequantized straight into mma.sync fragments)
against the fp64 oracle, through the C ABI: full outputs on shapes with
ragged token counts, ragged N and several K splits, the bench's full-size
M-sweep shapes (every row), bitwise repeats, counters left at zero,
guard bands, exact zeros, and the plan it reports; the grouped MoE GEMM on
the same path (8- and 16-token units, experts of many tokens, empty
experts, the fused SwiGLU epilogue)."""

import numpy as np
import pytest
import torch

from gpu_helpers import check_gemm, check_swiglu, workspace
from oracle import formats as F
from oracle import gemm as G
from oracle import moe as R
from quantized_gemm_bit_b200 import hq, synth
from quantized_gemm_bit_b200.build import build

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    build()
    torch.cuda.init()


def _bits(a):
    return a.view(torch.int16).numpy().view(np.uint16)


def make_case(m, n, k, asym, seed):
    q, s, z = synth.w4a16_weights(n, k, 128, asym, seed)
    a = synth.bf16_normal(m, k, seed + 1)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, int(asym), 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
    return d, blob, a, (q.numpy(), s.numpy(), None if z is None else z.numpy())


def run(d, blob, a, m, tuning, c=None):
    a_d = a.to(DEV)
    if c is None:
        c = torch.empty(m, d.n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m, tuning))
    hq.hq_gemm_w4a16(d, blob, a_d, m, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    return c, ws


REG = hq.Tuning(variant=3)


@pytest.mark.parametrize("m,n,k,asym", [
    (1, 128, 128, False), (1, 256, 1024, True), (4, 200, 384, False), (5, 640, 384, True),
    (8, 384, 1152, False), (9, 1000, 640, True), (13, 1152, 2560, False), (16, 1024, 1024, True),
    (16, 136, 256, False), (3, 9, 512, True), (7, 4096, 2048, True), (16, 4096, 2048, False),
])
def test_register_path_full_output(m, n, k, asym):
    """One and two 8-token tiles, N not a multiple of 128 (down to one
    partial tile), K from one record to 20, the library's K split; grids
    below one CTA per SM (eight warps of 16 rows per CTA) and above it (the
    N=4096 cases: four warps of 32 rows)."""
    d, blob, a, (q, s, z) = make_case(m, n, k, asym, 500 + m + n)
    assert hq.hq_plan_describe(d, m, REG).kernel == 4
    c, _ = run(d, blob, a, m, REG)
    check_gemm(c, G.w4a16_ref(_bits(a), q, s, z, 128), k, f"reg m={m} n={n} k={k} asym={asym}")


@pytest.mark.parametrize("m", [2, 16])
@pytest.mark.parametrize("splits", [1, 2, 3, 7, 20])
def test_register_path_splits_repeat_and_reset(m, splits):
    """Every K split (7 and 20 leave uneven slices, 20 slices of one record)
    gives the oracle's result, the same bits twice, and leaves the tile
    counters at zero."""
    n, k = 384, 2560
    d, blob, a, (q, s, z) = make_case(m, n, k, splits % 2 == 1, 600 + splits)
    t = hq.Tuning(variant=3, split_k=splits)
    c1, ws = run(d, blob, a, m, t)
    c2, _ = run(d, blob, a, m, t)
    assert torch.equal(c1, c2)
    check_gemm(c1, G.w4a16_ref(_bits(a), q, s, z, 128), k, f"reg splits={splits} m={m}")
    counters = ws[256:256 + 4 * 4 * 3].view(torch.int32)
    assert int(counters.abs().sum()) == 0


_SWEEP = {}


def _sweep_case(k, n):
    if (k, n) not in _SWEEP:
        seed = 1000 + (0 if k == 7168 else 1)
        q, s, z = synth.w4a16_weights(n, k, 128, False, seed)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
        w = G.w4a16_dequant(q.numpy(), s.numpy(), None, 128)
        _SWEEP[(k, n)] = (d, blob, w)
    return _SWEEP[(k, n)]


@pytest.mark.parametrize("k,n", [(7168, 18432), (18432, 7168)])
@pytest.mark.parametrize("m", [1, 4, 16])
def test_register_path_full_size(m, k, n):
    """The bench's M-sweep shapes at M <= 16 in the register path's own
    launch plan; every output row against the oracle."""
    d, blob, w = _sweep_case(k, n)
    a = synth.bf16_normal(m, k, 1000 + m)
    c, _ = run(d, blob, a, m, REG)
    ref = F.bf16_bits_to_f64(_bits(a)) @ w.T
    check_gemm(c, ref, k, f"reg sweep m={m} k={k} n={n}")


def test_register_path_guard_bands():
    m, n, k = 11, 200, 768
    d, blob, a, (q, s, z) = make_case(m, n, k, True, 71)
    flat = torch.full((m * n + 64,), 7.0, dtype=torch.bfloat16, device=DEV)
    c = flat[32:32 + m * n].view(m, n)
    c, _ = run(d, blob, a, m, hq.Tuning(variant=3, split_k=3), c=c)
    assert torch.all(flat[:32] == 7.0) and torch.all(flat[32 + m * n:] == 7.0)
    check_gemm(c, G.w4a16_ref(_bits(a), q, s, z, 128), k, "reg guard")


def test_register_path_zero_weights_give_exact_zeros():
    m, n, k = 16, 384, 1024
    q = torch.full((n, k // 8), 0x55555555, dtype=torch.int32)          # every nibble 5
    s = torch.full((n, k // 128), 0.01, dtype=torch.float16)
    z = torch.full((n, k // 128), 5, dtype=torch.uint8)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 1, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
    a = synth.bf16_normal(m, k, 333)
    c, _ = run(d, blob, a, m, hq.Tuning(variant=3, split_k=4))
    assert torch.count_nonzero(c) == 0


def test_register_path_request_that_does_not_apply():
    """Variant 3 with more than 16 tokens, or another format, runs the
    library's choice instead (and still matches the oracle)."""
    m, n, k = 17, 256, 512
    d, blob, a, (q, s, z) = make_case(m, n, k, False, 81)
    assert hq.hq_plan_describe(d, m, REG).kernel != 4
    c, _ = run(d, blob, a, m, REG)
    check_gemm(c, G.w4a16_ref(_bits(a), q, s, z, 128), k, "reg request m=17")
    d3 = hq.hq_quant_desc_init(hq.HQ_FMT_INT3, n, k, 128, 0, 1)
    assert hq.hq_plan_describe(d3, 8, REG).kernel != 4


def _moe_case(e, t, topk, n, k, asym, seed, heavy=None, gated=False):
    q, s, z = synth.w4a16_weights(n, k, 128, asym, seed, experts=e)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, int(asym), e)
    pack = hq.hq_pack_weights_gated if gated else hq.hq_pack_weights
    blob = torch.from_numpy(pack(d, q, s, z)).to(DEV)
    logits = synth.router_logits(t, e, seed=seed + 1)
    logits[:, 1] = -100.0                      # expert 1 never chosen: an empty group
    if heavy is not None:
        logits[:heavy, 2] = 100.0              # expert 2 takes `heavy` rows: several token tiles
    ids = R.topk_by_logit(logits.numpy(), topk)
    _, off, src = R.permute(ids, e)
    a = synth.bf16_normal(t, k, seed=seed + 2)
    a_sorted = R.gather_rows(_bits(a), src, topk)
    a_dev = torch.from_numpy(a_sorted.view(np.int16)).view(torch.bfloat16).to(DEV)
    off_dev = torch.from_numpy(off.astype(np.int32)).to(DEV)
    zn = None if z is None else z.numpy()
    return d, blob, a_sorted, a_dev, off, off_dev, (q.numpy(), s.numpy(), zn)


@pytest.mark.parametrize("e,t,topk,tile_m,asym,heavy", [
    (16, 24, 2, 0, False, None), (16, 24, 2, 0, True, 21), (16, 24, 2, 16, True, 40), (64, 7, 4, 0, False, None),
])
def test_register_path_grouped_full_output(e, t, topk, tile_m, asym, heavy):
    """Grouped MoE on the register path: 8-token units (a few rows per
    expert) and 16-token units (tile_m=16), an expert whose rows span
    several units, an empty expert, ragged N."""
    n, k = 384, 1024
    d, blob, a_sorted, a_dev, off, off_dev, (q, s, z) = _moe_case(e, t, topk, n, k, asym, 7000 + e + t,
                                                                  None if heavy is None else min(heavy, t))
    tuning = hq.Tuning(tile_m=tile_m, variant=3)
    plan = hq.hq_plan_describe(d, t * topk, tuning)
    assert plan.kernel == 4 and plan.tile_m == (16 if tile_m == 16 else 8)
    rows = t * topk
    c = torch.full((rows, n), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, rows, tuning))
    hq.hq_grouped_gemm_moe(d, blob, a_dev, off_dev, rows, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    _, ref = G.grouped_w4a16_ref(a_sorted, off, q, s, z, 128)
    check_gemm(c, ref, k, f"reg grouped e={e} t={t} tile_m={tile_m} asym={asym} heavy={heavy}")


@pytest.mark.parametrize("tile_m,heavy", [(0, None), (0, 12), (16, 20)])
def test_register_path_grouped_swiglu(tile_m, heavy):
    """Gate+up on the register path with the SwiGLU epilogue (gated row
    order: each warp's gate and up rows of the same features)."""
    e, t, topk, inter, k = 16, 24, 2, 192, 1024
    n = 2 * inter
    d, blob, a_sorted, a_dev, off, off_dev, (q, s, z) = _moe_case(e, t, topk, n, k, True, 7100, heavy, gated=True)
    tuning = hq.Tuning(tile_m=tile_m, variant=3)
    assert hq.hq_plan_describe(d, t * topk, tuning).kernel == 4
    rows = t * topk
    h = torch.full((rows, inter), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, rows, tuning))
    hq.hq_grouped_gemm_moe_swiglu(d, blob, a_dev, off_dev, rows, h, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    _, gu = G.grouped_w4a16_ref(a_sorted, off, q, s, z, 128)
    check_swiglu(h, gu, inter, k, f"reg grouped swiglu tile_m={tile_m} heavy={heavy}")
