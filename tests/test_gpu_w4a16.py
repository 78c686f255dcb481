"""GPU parity of the dense W4A16 GEMM (through the C ABI) against the fp64
oracle: full outputs on small shapes that span several tiles and ragged
tails, sampled rows at the full M-sweep sizes in the bench's launch
configuration, determinism, guard bands and workspace hygiene."""

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


def _bits(a):
    return a.view(torch.int16).numpy().view(np.uint16)


def make_case(m, n, k, asym, seed):
    q, s, z = synth.w4a16_weights(n, k, 128, asym, seed)
    a = synth.bf16_normal(m, k, seed + 1)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, int(asym), 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
    return d, blob, a, (q.numpy(), s.numpy(), None if z is None else z.numpy())


def run(d, blob, a, m, tuning=None, c=None):
    a_d = a.to(DEV)
    if c is None:
        c = torch.empty(m, d.n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m, tuning))
    hq.hq_gemm_w4a16(d, blob, a_d, m, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    return c, ws


def test_tiny_config_full_output():
    """W4A16 tiny: M=16, K=N=1024, asymmetric, seed 0."""
    m, n, k = 16, 1024, 1024
    d, blob, a, (q, s, z) = make_case(m, n, k, True, 0)
    c, _ = run(d, blob, a, m)
    ref = G.w4a16_ref(_bits(a), q, s, z, 128)
    check_gemm(c, ref, k, "tiny")


@pytest.mark.parametrize("m,n,k,asym", [
    (1, 256, 256, False), (7, 200, 384, True), (17, 384, 1152, False), (100, 128, 512, True),
    (129, 640, 640, False), (300, 256, 768, True), (513, 384, 256, False), (5, 640, 384, True),
    (40, 1152, 2560, False),
])
def test_ragged_shapes_full_output(m, n, k, asym):
    d, blob, a, (q, s, z) = make_case(m, n, k, asym, 100 + m)
    c, _ = run(d, blob, a, m)
    ref = G.w4a16_ref(_bits(a), q, s, z, 128)
    check_gemm(c, ref, k, f"m={m} n={n} k={k}")


@pytest.mark.parametrize("m,n,k,variant", [(1, 1, 128, 1), (3, 7, 128, 2), (16, 8, 256, 1), (64, 9, 128, 2),
                                           (300, 1, 128, 1), (33, 136, 128, 0)])
def test_narrow_and_single_block_shapes(m, n, k, variant):
    """Degenerate shapes: N below one 32-row slice (the scalar store path
    when N % 8 != 0), a single 128-K block, single-row outputs."""
    d, blob, a, (q, s, z) = make_case(m, n, k, True, 300 + m + n)
    c, _ = run(d, blob, a, m, hq.Tuning(variant=variant) if variant else None)
    check_gemm(c, G.w4a16_ref(_bits(a), q, s, z, 128), k, f"narrow m={m} n={n} k={k}")


@pytest.mark.parametrize("variant", [1, 2])
def test_zero_weights_give_exact_zeros(variant):
    """Every code equal to its zero point: w = (q - z) s = 0 exactly, so the
    output is exactly zero (both kernels, and the stream-K partial sums)."""
    m, n, k = 16, 384, 1024
    q = torch.full((n, k // 8), 0x55555555, dtype=torch.int32)          # every nibble 5
    s = torch.full((n, k // 128), 0.01, dtype=torch.float16)
    z = torch.full((n, k // 128), 5, dtype=torch.uint8)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 1, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
    a = synth.bf16_normal(m, k, 333)
    c, _ = run(d, blob, a, m, hq.Tuning(variant=variant))
    assert torch.count_nonzero(c) == 0
    assert np.all(G.w4a16_ref(_bits(a), q.numpy(), s.numpy(), z.numpy(), 128) == 0.0)


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("tile_m", [16, 32, 64, 128, 256])
def test_every_token_tile(tile_m, variant):
    """Every token tile of both kernels: variant 1 rescales weights to bf16
    for every tile; variant 2 feeds exact (q - z) and scales per group in
    fp32 for tiles <= 64."""
    m, n, k = 70, 384, 1024
    d, blob, a, (q, s, z) = make_case(m, n, k, True, 7)
    c, _ = run(d, blob, a, m, hq.Tuning(tile_m=tile_m, variant=variant))
    check_gemm(c, G.w4a16_ref(_bits(a), q, s, z, 128), k, f"tile_m={tile_m} variant={variant}")


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("splits", [2, 3, 7])
def test_split_k_and_determinism(splits, variant):
    m, n, k = 20, 256, 1792
    d, blob, a, (q, s, z) = make_case(m, n, k, False, 9)
    t = hq.Tuning(tile_m=32, split_k=splits, variant=variant)
    c1, ws = run(d, blob, a, m, t)
    c2, _ = run(d, blob, a, m, t)
    assert torch.equal(c1, c2)
    check_gemm(c1, G.w4a16_ref(_bits(a), q, s, z, 128), k, f"splits={splits}")
    # the workspace is left zero-filled (counters reset by the last split)
    counters = ws[256:256 + 4 * 4 * 2].view(torch.int32)
    assert int(counters.abs().sum()) == 0


@pytest.mark.parametrize("m", [1, 16, 48])
def test_stream_k_repeats_bit_for_bit(m):
    """Default plan at a stream-K size (K=N=2048 spread over every SM): two
    runs give identical bits and match the oracle."""
    n = k = 2048
    d, blob, a, (q, s, z) = make_case(m, n, k, True, 13 + m)
    c1, _ = run(d, blob, a, m)
    c2, _ = run(d, blob, a, m)
    assert torch.equal(c1, c2)
    check_gemm(c1, G.w4a16_ref(_bits(a), q, s, z, 128), k, f"stream-K m={m}")


@pytest.mark.parametrize("m,n,k", [(512, 25600, 256), (700, 14080, 384)])
def test_whole_waves_then_stream_k_tail(m, n, k):
    """Default plans whose whole-tile waves would leave the last wave part
    empty on 148 SMs (400 and 330 tiles of 256 tokens, the second with a
    ragged last token tile): whole tiles first, then the remaining tiles'
    K range shared stream-K style.  Full output, repeated bit for bit."""
    d, blob, a, (q, s, z) = make_case(m, n, k, False, 17 + n)
    assert hq.hq_workspace_size(d, m) > (1 << 20)     # partial sums: not a whole-tile plan
    c1, _ = run(d, blob, a, m)
    c2, _ = run(d, blob, a, m)
    assert torch.equal(c1, c2)
    check_gemm(c1, G.w4a16_ref(_bits(a), q, s, z, 128), k, f"stream-K tail m={m} n={n} k={k}")


def test_guard_bands_untouched():
    m, n, k = 33, 200, 512
    d, blob, a, (q, s, z) = make_case(m, n, k, True, 11)
    # sentinels before and after C in one flat buffer
    flat = torch.full((m * n + 64,), 7.0, dtype=torch.bfloat16, device=DEV)
    c = flat[32:32 + m * n].view(m, n)
    c, _ = run(d, blob, a, m, c=c)
    assert torch.all(flat[:32] == 7.0) and torch.all(flat[32 + m * n:] == 7.0)
    check_gemm(c, G.w4a16_ref(_bits(a), q, s, z, 128), k, "guard")


def test_timeout_probe_reports_instead_of_hanging():
    ws = workspace(256)
    hq.hq_debug_timeout_probe(ws, 2_000_000)      # 2 ms limit, nobody arrives
    assert hq.hq_check_device_status(ws) == hq.HQ_ERR_DEVICE_TIMEOUT
    assert hq.hq_check_device_status(ws) == hq.HQ_OK   # cleared


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
@pytest.mark.parametrize("m", [1, 4, 16, 64, 256, 1024, 4096])
def test_m_sweep_full_size_sampled_rows(m, k, n):
    """Full-size M-sweep shapes in the default (heuristic) launch
    configuration; the oracle evaluates tile-covering sampled rows."""
    d, blob, w = _sweep_case(k, n)
    a = synth.bf16_normal(m, k, 1000 + m)
    c, _ = run(d, blob, a, m)
    rows = tile_rows(m, 128, np.random.default_rng(m))
    ref = F.bf16_bits_to_f64(_bits(a)[rows]) @ w.T
    check_gemm(c[torch.from_numpy(rows).to(DEV)], ref, k, f"sweep m={m} k={k} n={n}")


@pytest.mark.parametrize("variant", [1, 2])
def test_workspace_reused_across_split_plans(variant):
    """One workspace serves split-K calls of different plans in turn (few
    tiles, then many, then few again): the tile counters sit in a fixed
    region after the 256-byte header, every call that completes leaves them
    at zero, and the partial sums lie past that region."""
    n, k = 1024, 2048
    d, blob, _, (q, s, z) = make_case(8, n, k, True, 1500)
    ws = workspace(1 << 22)
    for m in (16, 100, 16, 100):
        t = hq.Tuning(tile_m=16, split_k=3, variant=variant)
        assert hq.hq_workspace_size(d, m, t) <= ws.numel()
        a = synth.bf16_normal(m, k, 1501 + m)
        c = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
        hq.hq_gemm_w4a16(d, blob, a.to(DEV), m, c, ws, t)
        assert hq.hq_check_device_status(ws) == hq.HQ_OK
        check_gemm(c, G.w4a16_ref(_bits(a), q, s, z, 128), k, f"reused workspace m={m} variant={variant}")
        assert torch.count_nonzero(ws[:256 + (256 << 10)]) == 0
