"""GPU parity of the W4A16 kernels with MXINT4 weights (two's-complement
4-bit integers, E8M0 scale per 32 K) and bf16 activations, through the C
ABI, against the fp64 oracle: full outputs on shapes that span several tiles
with ragged tails, every token tile and explicit K splits, the whole range
of scale bytes the format keeps finite in bf16, sampled outputs at full
layer sizes, the grouped MoE form and the allocation-free entry point."""

import ctypes

import numpy as np
import pytest
import torch

from gpu_helpers import check_gemm, tile_rows, workspace
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


def make(n, k, seed, e8=None):
    codes, scales = synth.mxint4_weights(n, k, seed)
    if e8 is not None:
        scales = torch.from_numpy(e8)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXINT4, n, k, 32, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, codes, scales)).to(DEV)
    return d, blob, codes.numpy(), scales.numpy()


def run(d, blob, a, m, tuning=None):
    c = torch.empty(m, d.n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m, tuning))
    hq.hq_gemm_w4a16(d, blob, a.to(DEV), m, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    return c


@pytest.mark.parametrize("m,n,k,tile_m,split_k", [
    (1, 256, 256, 0, 0), (16, 1000, 512, 0, 0), (48, 384, 1152, 0, 0), (100, 640, 384, 0, 0),
    (300, 256, 768, 0, 0), (700, 384, 256, 0, 0), (64, 512, 512, 64, 0), (33, 256, 1024, 32, 0),
    (600, 256, 512, 256, 0), (200, 384, 384, 128, 0), (16, 384, 2048, 16, 0), (40, 256, 1024, 0, 3),
    (130, 128, 640, 128, 2),
])
def test_dense_full_output(m, n, k, tile_m, split_k):
    d, blob, codes, e8 = make(n, k, 11000 + m)
    a = synth.bf16_normal(m, k, 11100 + m)
    t = hq.Tuning(tile_m=tile_m, split_k=split_k) if (tile_m or split_k) else None
    c = run(d, blob, a, m, t)
    ref = G.mxint4_a16_ref(_bits(a), codes, e8)
    check_gemm(c, ref, k, f"mxint4-a16 m={m} n={n} k={k} tile={tile_m} split={split_k}")


def test_scale_range():
    """Scale bytes from 0 (weights down to 2^-127) to 251 (up to 8 * 2^124),
    three regimes on interleaved columns, each checked on its own columns:
    tiny (0..6) with activations carrying 2^100, ordinary (118..135) with
    plain activations, large (240..251) with activations carrying 2^-120
    (exact scalings of bf16 N(0,1), so every product stays a normal fp32
    number)."""
    m, n, k = 24, 384, 512
    rng = np.random.default_rng(11200)
    regime = np.arange(n) % 3
    lo = np.array([0, 118, 240])[regime]
    hi = np.array([7, 136, 252])[regime]
    e8 = rng.integers(lo[:, None], hi[:, None], size=(n, k // 32)).astype(np.uint8)
    d, blob, codes, e8 = make(n, k, 11201, e8)
    base = synth.bf16_normal(m, k, 11202).float()
    for r, f in ((0, 2.0 ** 100), (1, 1.0), (2, 2.0 ** -120)):
        a = (base * f).to(torch.bfloat16)
        c = run(d, blob, a, m)
        cols = np.nonzero(regime == r)[0]
        ref = G.mxint4_a16_ref(_bits(a), codes, e8, cols=cols)
        check_gemm(c[:, cols], ref, k, f"mxint4 scale regime {r}")


@pytest.mark.parametrize("m,n,k", [(16, 18432, 7168), (4096, 7168, 7168)])
def test_full_size_sampled(m, n, k):
    """Layer sizes in the library's own launch plan: every row of a sample
    of columns covering each 128-row weight tile (first, last, random)."""
    d, blob, codes, e8 = make(n, k, 11300 + m)
    a = synth.bf16_normal(m, k, 11301 + m)
    c = run(d, blob, a, m).cpu()
    rng = np.random.default_rng(11302)
    cols = tile_rows(n, 128, rng, per_tile=1)
    rows = np.arange(m) if m <= 64 else tile_rows(m, 256, rng, per_tile=1)
    ref = G.mxint4_a16_ref(_bits(a), codes, e8, rows=rows, cols=cols)
    check_gemm(c[rows][:, cols], ref, k, f"mxint4-a16 full size m={m}")


def test_runs_are_bit_identical():
    m, n, k = 40, 768, 2048                            # stream-K with partial sums
    d, blob, _, _ = make(n, k, 11400)
    a = synth.bf16_normal(m, k, 11401)
    c1 = run(d, blob, a, m)
    c2 = run(d, blob, a, m)
    assert torch.equal(c1, c2)


def test_allocation_free_entry_point():
    m, n, k = 20, 384, 1024
    d, blob, codes, e8 = make(n, k, 11500)
    a = synth.bf16_normal(m, k, 11501)
    c = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
    st = hq.lib().hq_gemm_w4a16_static(ctypes.byref(d), blob.data_ptr(), a.to(DEV).data_ptr(), m, c.data_ptr(),
                                       None, torch.cuda.current_stream().cuda_stream)
    assert st == hq.HQ_OK
    torch.cuda.synchronize()
    check_gemm(c, G.mxint4_a16_ref(_bits(a), codes, e8), k, "mxint4-a16 static")


@pytest.mark.parametrize("tile_m", [0, 16, 32, 64, 128, 256])
def test_grouped_full_output(tile_m):
    """8 experts, 40 tokens top-2, one expert never chosen; expert-sorted
    rows and offsets from the oracle's routing."""
    e, n, k, t, topk = 8, 256, 512, 40, 2
    codes, e8 = synth.mxint4_weights(n, k, seed=11600, experts=e)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXINT4, n, k, 32, 0, e)
    blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(DEV)
    logits = synth.router_logits(t, e, seed=11601)
    logits[:, 5] = -100.0
    ids = R.topk_by_logit(logits.numpy(), topk)
    _, off, src = R.permute(ids, e)
    a = synth.bf16_normal(t, k, seed=11602)
    a_sorted = R.gather_rows(_bits(a), src, topk)
    rows = t * topk
    tuning = hq.Tuning(tile_m=tile_m) if tile_m else None
    c = torch.empty(rows, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, rows, tuning))
    a_dev = torch.from_numpy(a_sorted.view(np.int16)).view(torch.bfloat16).to(DEV)
    off_dev = torch.from_numpy(off.astype(np.int32)).to(DEV)
    hq.hq_grouped_gemm_moe(d, blob, a_dev, off_dev, rows, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    _, ref = G.grouped_mxint4_a16_ref(a_sorted, off, codes.numpy(), e8.numpy())
    check_gemm(c, ref, k, f"grouped mxint4-a16 tile={tile_m}")
