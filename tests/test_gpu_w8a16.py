"""GPU parity of the W4A16 kernels with INT8 weights (8-bit codes, fp16
scale and optional uint8 zero point per 128 K) and bf16 activations,
through the C ABI, against the fp64 oracle: full outputs on shapes that
span several tiles with ragged tails, every token tile and explicit K
splits, both zero-point forms, sampled outputs at full layer sizes, run to
run determinism, the grouped MoE form and the allocation-free entry
point."""

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


def make(n, k, asym, seed):
    q, s, z = synth.w8a16_weights(n, k, 128, asym, seed)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT8, n, k, 128, int(asym), 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
    return d, blob, (q.numpy(), s.numpy(), None if z is None else z.numpy())


def run(d, blob, a, m, tuning=None):
    c = torch.empty(m, d.n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m, tuning))
    hq.hq_gemm_w4a16(d, blob, a.to(DEV), m, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    return c


@pytest.mark.parametrize("m,n,k,asym,tile_m,split_k", [
    (1, 256, 256, False, 0, 0), (16, 1000, 512, True, 0, 0), (48, 384, 1152, False, 0, 0),
    (100, 640, 384, True, 0, 0), (300, 256, 768, False, 0, 0), (700, 384, 256, True, 0, 0),
    (64, 512, 512, True, 64, 0), (33, 256, 1024, False, 32, 0), (600, 256, 512, True, 256, 0),
    (200, 384, 384, False, 128, 0), (16, 384, 2048, True, 16, 0), (40, 256, 1024, False, 0, 3),
    (130, 128, 640, True, 128, 2),
])
def test_dense_full_output(m, n, k, asym, tile_m, split_k):
    d, blob, w = make(n, k, asym, 10700 + m)
    a = synth.bf16_normal(m, k, 10800 + m)
    t = hq.Tuning(tile_m=tile_m, split_k=split_k) if (tile_m or split_k) else None
    c = run(d, blob, a, m, t)
    ref = G.w8a16_ref(_bits(a), *w, 128)
    check_gemm(c, ref, k, f"w8a16 m={m} n={n} k={k} asym={asym} tile={tile_m} split={split_k}")


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("tile_m", [16, 32, 64])
def test_small_tiles_both_variants(tile_m, variant):
    """Tiles of up to 64 tokens: variant 1 (weights correctly rounded to
    bf16, the rescaling kernel) and 2 (exact (q - z), per-group fp32 scale,
    the library's default there), with zero points and a ragged tail."""
    m, n, k = 2 * tile_m - 3, 384, 1408
    d, blob, w = make(n, k, True, 10950 + tile_m + variant)
    a = synth.bf16_normal(m, k, 10951 + tile_m)
    c = run(d, blob, a, m, hq.Tuning(tile_m=tile_m, variant=variant))
    check_gemm(c, G.w8a16_ref(_bits(a), *w, 128), k, f"w8a16 tile={tile_m} variant={variant}")


@pytest.mark.parametrize("m,n,k", [(16, 18432, 7168), (4096, 7168, 7168)])
def test_full_size_sampled(m, n, k):
    d, blob, w = make(n, k, False, 10900 + m)
    a = synth.bf16_normal(m, k, 10901 + m)
    c = run(d, blob, a, m).cpu()
    rng = np.random.default_rng(10902)
    cols = tile_rows(n, 128, rng, per_tile=1)
    rows = np.arange(m) if m <= 64 else tile_rows(m, 256, rng, per_tile=1)
    ref = G.w8a16_ref(_bits(a), *w, 128, rows=rows, cols=cols)
    check_gemm(c[rows][:, cols], ref, k, f"w8a16 full size m={m}")


def test_runs_are_bit_identical():
    m, n, k = 40, 768, 2048
    d, blob, _ = make(n, k, True, 10910)
    a = synth.bf16_normal(m, k, 10911)
    assert torch.equal(run(d, blob, a, m), run(d, blob, a, m))


def test_allocation_free_entry_point():
    m, n, k = 20, 384, 1024
    d, blob, w = make(n, k, True, 10920)
    a = synth.bf16_normal(m, k, 10921)
    c = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
    st = hq.lib().hq_gemm_w4a16_static(ctypes.byref(d), blob.data_ptr(), a.to(DEV).data_ptr(), m, c.data_ptr(),
                                       None, torch.cuda.current_stream().cuda_stream)
    assert st == hq.HQ_OK
    torch.cuda.synchronize()
    check_gemm(c, G.w8a16_ref(_bits(a), *w, 128), k, "w8a16 static")


@pytest.mark.parametrize("tile_m", [0, 16, 64, 128, 256])
def test_grouped_full_output(tile_m):
    """8 experts, 40 tokens top-2, one expert never chosen, asymmetric;
    expert-sorted rows and offsets from the oracle's routing."""
    e, n, k, t, topk = 8, 256, 512, 40, 2
    q, s, z = synth.w8a16_weights(n, k, 128, True, seed=10930, experts=e)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT8, n, k, 128, 1, e)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
    logits = synth.router_logits(t, e, seed=10931)
    logits[:, 2] = -100.0
    ids = R.topk_by_logit(logits.numpy(), topk)
    _, off, src = R.permute(ids, e)
    a = synth.bf16_normal(t, k, seed=10932)
    a_sorted = R.gather_rows(_bits(a), src, topk)
    rows = t * topk
    tuning = hq.Tuning(tile_m=tile_m) if tile_m else None
    c = torch.empty(rows, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, rows, tuning))
    a_dev = torch.from_numpy(a_sorted.view(np.int16)).view(torch.bfloat16).to(DEV)
    off_dev = torch.from_numpy(off.astype(np.int32)).to(DEV)
    hq.hq_grouped_gemm_moe(d, blob, a_dev, off_dev, rows, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    _, ref = G.grouped_w8a16_ref(a_sorted, off, q.numpy(), s.numpy(), z.numpy(), 128)
    check_gemm(c, ref, k, f"grouped w8a16 tile={tile_m}")
