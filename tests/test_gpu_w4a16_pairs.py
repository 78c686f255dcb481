"""GPU parity of the W4A16-family GEMM on CTA pairs (cta_group::2: a
cluster of two CTAs runs a 256-row weight tile, each CTA dequantizing its
own 128 rows into its TMEM and staging half of the 256-token tile) against
the fp64 oracle, for every weight format; the plan the library picks; and
one CTA per tile at the same sizes."""

import numpy as np
import pytest
import torch

from gpu_helpers import check_gemm, tile_rows, workspace
from oracle import gemm as G
from quantized_gemm_bit_b200 import hq, synth
from quantized_gemm_bit_b200.build import build

pytestmark = pytest.mark.gpu
DEV = "cuda"
PAIRS = hq.Tuning(cta_group=2)


@pytest.fixture(scope="module", autouse=True)
def _setup():
    build()
    torch.cuda.init()


def _bits(a):
    return a.view(torch.int16).numpy().view(np.uint16)


def case(fmt, n, k, asym, seed):
    """(descriptor, device blob, oracle function of (a_bits, rows, cols))."""
    if fmt in ("int4", "int3", "int2", "int8"):
        gen, code, ref = {"int4": (synth.w4a16_weights, hq.HQ_FMT_INT4, G.w4a16_ref),
                          "int3": (synth.w3a16_weights, hq.HQ_FMT_INT3, G.w3a16_ref),
                          "int2": (synth.w2a16_weights, hq.HQ_FMT_INT2, G.w2a16_ref),
                          "int8": (synth.w8a16_weights, hq.HQ_FMT_INT8, G.w8a16_ref)}[fmt]
        q, s, z = gen(n, k, 128, asym, seed)
        d = hq.hq_quant_desc_init(code, n, k, 128, int(asym), 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
        qn, sn, zn = q.numpy(), s.numpy(), None if z is None else z.numpy()
        return d, blob, lambda a, rows=None, cols=None: ref(a, qn, sn, zn, 128, rows=rows, cols=cols)
    gen, code, ref = {"mxfp4": (synth.mxfp4_weights, hq.HQ_FMT_MXFP4_A16, G.mxfp4_a16_ref),
                      "mxint4": (synth.mxint4_weights, hq.HQ_FMT_MXINT4, G.mxint4_a16_ref)}[fmt]
    codes, e8 = gen(n, k, seed=seed)
    d = hq.hq_quant_desc_init(code, n, k, 32, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(DEV)
    cn, en = codes.numpy(), e8.numpy()
    return d, blob, lambda a, rows=None, cols=None: ref(a, cn, en, rows=rows, cols=cols)


def run(d, blob, a, m, tuning=None):
    c = torch.empty(m, d.n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m, tuning))
    hq.hq_gemm_w4a16(d, blob, a.to(DEV), m, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    return c


@pytest.mark.parametrize("fmt,asym", [("int4", False), ("int4", True), ("int3", True), ("int2", False),
                                      ("int8", True), ("mxfp4", False), ("mxint4", False)])
def test_every_format_on_pairs(fmt, asym):
    """Two 256-row weight tiles x two token tiles (the second ragged: its
    upper half lies past M), every output against the oracle; the same call
    twice gives the same bits."""
    m, n, k = 300, 512, 1024
    d, blob, ref = case(fmt, n, k, asym, 900 + len(fmt))
    a = synth.bf16_normal(m, k, 901)
    plan = hq.hq_plan_describe(d, m, PAIRS)
    assert (plan.cta_group, plan.tile_m, plan.split) == (2, 256, 0)
    c1 = run(d, blob, a, m, PAIRS)
    c2 = run(d, blob, a, m, PAIRS)
    assert torch.equal(c1, c2)
    check_gemm(c1, ref(_bits(a)), k, f"w4a16 pairs fmt={fmt} asym={asym}")


def test_pairs_more_units_than_clusters():
    """More (token tile, 256-row weight tile) units than resident clusters,
    with a last token tile of 80 rows (its second half empty)."""
    m, n, k = 1104, 4096, 512
    d, blob, ref = case("int4", n, k, True, 910)
    a = synth.bf16_normal(m, k, 911)
    c = run(d, blob, a, m, PAIRS)
    rows = tile_rows(m, 128, np.random.default_rng(7))
    check_gemm(c[torch.from_numpy(rows).to(DEV)], ref(_bits(a), rows=rows), k, "w4a16 pairs, many units")


@pytest.mark.parametrize("k,n", [(7168, 18432), (18432, 7168)])
def test_full_size_library_plan_and_one_cta(k, n):
    """The M = 4096 sweep shapes: the library's plan (one CTA per tile),
    CTA pairs on request, and one CTA per tile by name (cta_group 1) agree
    with the oracle on sampled rows."""
    m = 4096
    d, blob, ref = case("int4", n, k, False, 920)
    a = synth.bf16_normal(m, k, 921)
    rows = tile_rows(m, 256, np.random.default_rng(k), per_tile=1)
    want = ref(_bits(a), rows=rows)
    for name, t in (("lib", None), ("pairs", PAIRS), ("one CTA", hq.Tuning(cta_group=1))):
        c = run(d, blob, a, m, t)
        check_gemm(c[torch.from_numpy(rows).to(DEV)], want, k, f"w4a16 m=4096 k={k} plan={name}")
    assert hq.hq_plan_describe(d, m).cta_group == 1
    assert hq.hq_plan_describe(d, m, PAIRS).cta_group == 2


def test_pairs_refused_where_they_do_not_apply():
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 384, 512, 128, 0, 1)      # N not a multiple of 256
    ws = workspace(1 << 20)
    c = torch.empty(256, 384, dtype=torch.bfloat16, device=DEV)
    a = synth.bf16_normal(256, 512, 1).to(DEV)
    blob = torch.zeros(hq.hq_packed_size(d), dtype=torch.uint8, device=DEV)
    with pytest.raises(hq.HQError):
        hq.hq_gemm_w4a16(d, blob, a, 256, c, ws, PAIRS)
    d2 = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 512, 512, 128, 0, 1)
    blob2 = torch.zeros(hq.hq_packed_size(d2), dtype=torch.uint8, device=DEV)
    c2 = torch.empty(256, 512, dtype=torch.bfloat16, device=DEV)
    for bad in (hq.Tuning(cta_group=2, tile_m=128), hq.Tuning(cta_group=2, split_k=2)):
        with pytest.raises(hq.HQError):
            hq.hq_gemm_w4a16(d2, blob2, a, 256, c2, ws, bad)


def test_int8_large_tiles_default_to_pairs():
    """INT8 records leave room for only two 256-token stages on one CTA; the
    library runs such whole tiles on CTA pairs (four stages), and the result
    is the oracle's."""
    m, n, k = 1024, 4608, 1024            # 18 x 4 256-row x 256-token tiles: whole tiles
    d, blob, ref = case("int8", n, k, True, 930)
    plan = hq.hq_plan_describe(d, m)
    assert (plan.cta_group, plan.tile_m, plan.split) == (2, 256, 0)
    assert plan.ring_stages > hq.hq_plan_describe(d, m, hq.Tuning(cta_group=1)).ring_stages
    a = synth.bf16_normal(m, k, 931)
    c = run(d, blob, a, m)
    rows = tile_rows(m, 256, np.random.default_rng(9))
    check_gemm(c[torch.from_numpy(rows).to(DEV)], ref(_bits(a), rows=rows), k, "w4a16 int8 default pairs")
