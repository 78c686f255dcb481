"""GPU parity of the MoE path through the C ABI: top-k routing and the
expert-sorted permutation are bit-exact against the oracle; the grouped
W4A16 GEMM matches the fp64 oracle within the GEMM tolerance, in full on a
reduced configuration and on sampled rows/columns at the full workload
(256 experts, top-8, hidden 7168, gate+up N=4096, down K=2048).  The layer
around the grouped GEMMs: routing weights, SwiGLU and the weighted combine
against their oracle functions with bounds derived from their fp32
arithmetic, and the whole layer end to end."""

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


def gpu_route(logits, k):
    t, e = logits.shape
    ids = torch.empty(t, k, dtype=torch.int32, device=DEV)
    hq.hq_moe_topk(logits.to(DEV), t, e, k, ids)
    return ids


def gpu_permute(ids, e, a=None):
    t, k = ids.shape
    src = torch.full((t * k,), -1, dtype=torch.int32, device=DEV)
    off = torch.full((e + 1,), -1, dtype=torch.int32, device=DEV)
    ws = workspace(hq.hq_moe_permute_workspace_size(t, k, e))
    a_sorted = None
    if a is not None:
        a_sorted = torch.empty(t * k, a.shape[1], dtype=torch.bfloat16, device=DEV)
    hq.hq_moe_permute(ids, t, k, e, src, off, ws, a=None if a is None else a.to(DEV),
                      hidden=0 if a is None else a.shape[1], a_sorted=a_sorted)
    st = hq.hq_check_device_status(ws)
    return src, off, a_sorted, st


@pytest.mark.parametrize("t", [1, 64, 1024, 8192])
def test_topk_bit_exact(t):
    logits = synth.router_logits(t, 256, seed=3001 + t)
    ids = gpu_route(logits, 8).cpu().numpy()
    assert np.array_equal(ids, R.topk_by_logit(logits.numpy(), 8))


def test_topk_ties_go_to_lower_index():
    logits = torch.zeros(5, 40)
    logits[1, 7] = 1.0
    logits[2, ::3] = -1.0
    logits[3] = torch.arange(40).float() % 4
    ids = gpu_route(logits, 6).cpu().numpy()
    assert np.array_equal(ids, R.topk_by_logit(logits.numpy(), 6))


@pytest.mark.parametrize("t,e,k", [(1, 256, 8), (64, 256, 8), (1000, 256, 8), (8192, 256, 8), (37, 5, 3)])
def test_permute_and_gather_bit_exact(t, e, k):
    logits = synth.router_logits(t, e, seed=4000 + t)
    ids = R.topk_by_logit(logits.numpy(), k)
    hidden = 64
    a = synth.bf16_normal(t, hidden, seed=4100 + t)
    src, off, a_sorted, st = gpu_permute(torch.from_numpy(ids).to(DEV), e, a)
    assert st == hq.HQ_OK
    counts, off_ref, src_ref = R.permute(ids, e)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(src.cpu().numpy(), src_ref)
    ref_rows = R.gather_rows(_bits(a), src_ref, k)
    assert np.array_equal(_bits(a_sorted.cpu()), ref_rows)


def test_permute_duplicates_empty_experts_and_bad_ids():
    ids = torch.tensor([[3, 3], [0, 3], [1, 1]], dtype=torch.int32)
    src, off, _, st = gpu_permute(ids.to(DEV), 6)
    assert st == hq.HQ_OK
    _, off_ref, src_ref = R.permute(ids.numpy(), 6)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(src.cpu().numpy(), src_ref)
    bad = torch.tensor([[0, 9]], dtype=torch.int32)
    _, _, _, st = gpu_permute(bad.to(DEV), 6)
    assert st == hq.HQ_ERR_DEVICE_BAD_OFFSETS


def _grouped(desc, blob, a_sorted, off, rows, n, tuning=None):
    c = torch.empty(rows, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(desc, rows, tuning))
    hq.hq_grouped_gemm_moe(desc, blob, a_sorted, off, rows, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    return c


@pytest.mark.parametrize("tile_m,variant", [(0, 0), (16, 0), (32, 0), (64, 0), (128, 0), (256, 0), (16, 2), (32, 2),
                                            (64, 2), (0, 3), (16, 3)])
def test_grouped_reduced_config_full_output(tile_m, variant):
    e, n, k, t, topk = 8, 256, 512, 40, 2
    q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=5000, experts=e)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, e)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(DEV)
    logits = synth.router_logits(t, e, seed=5001)
    logits[:, 5] = -100.0                      # expert 5 never chosen: an empty group
    ids = R.topk_by_logit(logits.numpy(), topk)
    a = synth.bf16_normal(t, k, seed=5002)
    src, off, a_sorted, st = gpu_permute(torch.from_numpy(ids).to(DEV), e, a)
    assert st == hq.HQ_OK
    # the reference runs on the oracle's own permutation (the GPU's is bit-equal)
    _, off_ref, src_ref = R.permute(ids, e)
    a_sorted_ref = R.gather_rows(_bits(a), src_ref, topk)
    assert np.array_equal(off.cpu().numpy(), off_ref) and np.array_equal(src.cpu().numpy(), src_ref)
    assert np.array_equal(_bits(a_sorted.cpu()), a_sorted_ref)
    tuning = hq.Tuning(tile_m=tile_m, variant=variant) if (tile_m or variant) else None
    c = _grouped(d, blob, a_sorted, off, t * topk, n, tuning)
    _, ref = G.grouped_w4a16_ref(a_sorted_ref, off_ref, q.numpy(), s.numpy(), None, 128)
    check_gemm(c, ref, k, f"grouped tile_m={tile_m} variant={variant}")


def test_grouped_maximum_expert_count():
    """1024 experts (the device tile table's limit), 600 tokens top-2: most
    experts hold one or two rows, many none; full output."""
    e, n, k, t, topk = 1024, 128, 128, 600, 2
    q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=5200, experts=e)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, e)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(DEV)
    logits = synth.router_logits(t, e, seed=5201)
    ids = R.topk_by_logit(logits.numpy(), topk)
    a = synth.bf16_normal(t, k, seed=5202)
    src, off, a_sorted, st = gpu_permute(torch.from_numpy(ids).to(DEV), e, a)
    assert st == hq.HQ_OK
    _, off_ref, src_ref = R.permute(ids, e)
    assert np.array_equal(off.cpu().numpy(), off_ref) and np.array_equal(src.cpu().numpy(), src_ref)
    a_sorted_ref = R.gather_rows(_bits(a), src_ref, topk)
    c = _grouped(d, blob, a_sorted, off, t * topk, n)
    _, ref = G.grouped_w4a16_ref(a_sorted_ref, off_ref, q.numpy(), s.numpy(), None, 128)
    check_gemm(c, ref, k, "grouped 1024 experts")


def test_grouped_bad_offsets_are_reported():
    e, n, k = 4, 128, 256
    q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=5100, experts=e)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, e)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(DEV)
    a = synth.bf16_normal(10, k, seed=5101).to(DEV)
    off = torch.tensor([0, 6, 3, 8, 10], dtype=torch.int32, device=DEV)   # not monotone
    c = torch.zeros(10, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, 10))
    hq.hq_grouped_gemm_moe(d, blob, a, off, 10, c, ws)
    assert hq.hq_check_device_status(ws) == hq.HQ_ERR_DEVICE_BAD_OFFSETS
    assert int(c.float().abs().sum()) == 0                               # nothing written


_FULL = {}


def _full_weights(which):
    """256 experts; gate+up: N=4096, K=7168; down: N=7168, K=2048."""
    if which not in _FULL:
        n, k, seed = (4096, 7168, 3000) if which == "gate_up" else (7168, 2048, 3010)
        q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=seed, experts=256)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, 256)
        blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(DEV)
        _FULL[which] = (d, blob, q.numpy(), s.numpy(), n, k)
    return _FULL[which]


@pytest.mark.parametrize("t", [64, 1024, 8192])
@pytest.mark.parametrize("which", ["gate_up", "down"])
def test_grouped_full_size_sampled(t, which):
    d, blob, q, s, n, k = _full_weights(which)
    logits = synth.router_logits(t, 256, seed=3001)
    ids = gpu_route(logits, 8)
    # the oracle's routing and permutation, which the GPU's must equal bit for bit
    ids_ref = R.topk_by_logit(logits.numpy(), 8)
    _, off_ref, src_ref = R.permute(ids_ref, 256)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    if which == "gate_up":
        a = synth.bf16_normal(t, k, seed=3002)
        src, off, a_sorted, st = gpu_permute(ids, 256, a)
        assert st == hq.HQ_OK
        a_sorted_ref = R.gather_rows(_bits(a), src_ref, 8)
    else:
        src, off, _, st = gpu_permute(ids, 256)
        assert st == hq.HQ_OK
        a_in = synth.bf16_normal(t * 8, k, seed=3003)
        a_sorted, a_sorted_ref = a_in.to(DEV), _bits(a_in)
    assert np.array_equal(off.cpu().numpy(), off_ref) and np.array_equal(src.cpu().numpy(), src_ref)
    rows_total = t * 8
    c = _grouped(d, blob, a_sorted, off, rows_total, n)
    offs = off_ref
    rng = np.random.default_rng(t)
    rows = []
    for ex in range(256):
        lo, hi = offs[ex], offs[ex + 1]
        if hi > lo:
            rows.extend({lo, hi - 1, int(rng.integers(lo, hi))})
    rows = np.array(sorted(set(rows)))
    cols = np.array(sorted({c0 for nt in range(n // 128) for c0 in (nt * 128, nt * 128 + 127,
                                                                     nt * 128 + int(rng.integers(0, 128)))}))
    a_rows = a_sorted_ref[rows]
    expert_of = np.searchsorted(offs, rows, side="right") - 1
    ref = np.zeros((len(rows), len(cols)))
    for ex in np.unique(expert_of):
        sel = np.nonzero(expert_of == ex)[0]
        w = G.w4a16_dequant(q[ex], s[ex], None, 128, rows=cols)
        ref[sel] = F.bf16_bits_to_f64(a_rows[sel]) @ w.T
    got = c[torch.from_numpy(rows).to(DEV)][:, torch.from_numpy(cols).to(DEV)]
    check_gemm(got, ref, k, f"moe {which} t={t}")


# ---------------------------------------------------------------- the MoE layer around the grouped GEMMs

@pytest.mark.parametrize("t", [1, 64, 1024])
def test_topk_softmax_ids_and_weights(t):
    """Ids bit-exact (and equal to hq_moe_topk's); weights = the oracle's
    softmax probabilities within fp32 rounding: E exps, a 256-term sum and
    a division, each a few fp32 ulps, so |w - ref| <= 1e-5 * ref."""
    logits = synth.router_logits(t, 256, seed=3300 + t)
    ids = torch.empty(t, 8, dtype=torch.int32, device=DEV)
    w = torch.empty(t, 8, dtype=torch.float32, device=DEV)
    hq.hq_moe_topk_softmax(logits.to(DEV), t, 256, 8, ids, w)
    ids_ref = R.topk_by_logit(logits.numpy(), 8)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.array_equal(gpu_route(logits, 8).cpu().numpy(), ids_ref)
    w_ref = R.softmax_topk_weights(logits.numpy(), ids_ref)
    assert np.all(np.abs(w.cpu().numpy() - w_ref) <= 1e-5 * w_ref)


def _bf16_bits(x):
    return F.f32_to_bf16_bits_rne(np.asarray(x, dtype=np.float32))


@pytest.mark.parametrize("rows,inter", [(1, 8), (37, 24), (512, 2048)])
def test_swiglu_elementwise(rows, inter):
    """h = silu(g) * u in fp32, rounded to bf16: |h - ref| <= 2^-8 |ref|
    plus the smallest bf16 subnormal (fp32 arithmetic adds ~1e-6 relative
    to the half-ulp of the bf16 rounding)."""
    rng = np.random.default_rng(rows + inter)
    x = rng.normal(0.0, 3.0, (rows, 2 * inter))
    x[0, :4] = [0.0, -100.0, 100.0, -0.5]                 # zero, both tails
    bits = _bf16_bits(x)
    gu = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(DEV)
    h = torch.empty(rows, inter, dtype=torch.bfloat16, device=DEV)
    hq.hq_moe_swiglu(gu, rows, inter, h)
    got = h.float().double().cpu().numpy()
    ref = R.silu_mul(bits, inter)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -133)


def _combine_case(t, k, e, hidden, seed):
    logits = synth.router_logits(t, e, seed=seed)
    ids = R.topk_by_logit(logits.numpy(), k)
    _, _, src = R.permute(ids, e)
    w = R.softmax_topk_weights(logits.numpy(), ids).astype(np.float32)
    y = _bf16_bits(np.random.default_rng(seed).normal(size=(t * k, hidden)))
    return src, w, y


def _gpu_combine(y, src, w, t, k, hidden):
    out = torch.empty(t, hidden, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_moe_combine_workspace_size(t, k))
    yd = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).to(DEV)
    hq.hq_moe_combine(yd, torch.from_numpy(src).to(DEV), torch.from_numpy(w).to(DEV), t, k, hidden, out, ws)
    return out, hq.hq_check_device_status(ws)


@pytest.mark.parametrize("t,hidden", [(1, 8), (50, 264), (1024, 7168)])
def test_combine_against_oracle(t, hidden):
    """fp32 fused multiply-adds in slot order then one bf16 rounding:
    |out - ref| <= 2^-8 |ref| + 2^-20 sum_j |w_j y_j|."""
    k, e = 8, 256
    src, w, y = _combine_case(t, k, e, hidden, 3400 + t)
    out, st = _gpu_combine(y, src, w, t, k, hidden)
    assert st == hq.HQ_OK
    got = out.float().double().cpu().numpy()
    ref = R.combine(y, src, w, k)
    mag = R.combine(y & np.uint16(0x7FFF), src, np.abs(w), k)    # sum_j |w_j y_j|
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -20 * mag)
    out2, _ = _gpu_combine(y, src, w, t, k, hidden)
    assert torch.equal(out, out2)                                   # no atomics: same bits


@pytest.mark.parametrize("bad", ["duplicate", "out_of_range"])
def test_combine_reports_a_sorted_list_that_is_not_a_permutation(bad):
    t, k, e, hidden = 20, 4, 16, 64
    src, w, y = _combine_case(t, k, e, hidden, 3500)
    src = src.copy()
    if bad == "duplicate":
        src[3] = src[5]
    else:
        src[7] = t * k + 3
    _, st = _gpu_combine(y, src, w, t, k, hidden)
    assert st == hq.HQ_ERR_DEVICE_BAD_OFFSETS


def _layer_oracle(x_bits, logits, q1, s1, q2, s2, k, e, inter, fused=False):
    """The layer from oracle pieces only, rounding to bf16 wherever the GPU
    path stores bf16 (after each GEMM and after SwiGLU; with the SwiGLU fused
    into the gate+up GEMM, gate and up are not rounded)."""
    ids = R.topk_by_logit(logits, k)
    w = R.softmax_topk_weights(logits, ids)
    _, off, src = R.permute(ids, e)
    xs = R.gather_rows(x_bits, src, k)
    _, c1 = G.grouped_w4a16_ref(xs, off, q1, s1, None, 128)
    h = R.silu_mul_f64(c1, inter) if fused else R.silu_mul(_bf16_bits(c1), inter)
    _, c2 = G.grouped_w4a16_ref(_bf16_bits(h), off, q2, s2, None, 128)
    return R.combine(_bf16_bits(c2), src, w, k), ids, off, src


@pytest.mark.parametrize("tile_m,variant,fmt", [(0, 0, hq.HQ_FMT_INT4), (16, 0, hq.HQ_FMT_INT4),
                                                (64, 0, hq.HQ_FMT_INT4), (128, 0, hq.HQ_FMT_INT4),
                                                (256, 0, hq.HQ_FMT_INT4), (32, 1, hq.HQ_FMT_INT4),
                                                (0, 0, hq.HQ_FMT_INT3), (0, 0, hq.HQ_FMT_MXFP4_A16),
                                                (0, 3, hq.HQ_FMT_INT4), (16, 3, hq.HQ_FMT_INT4)])
def test_grouped_swiglu_fused_reduced_config(tile_m, variant, fmt):
    """Gate+up grouped GEMM with the SwiGLU epilogue (weights packed in the
    gated row order) against the oracle's fp64 gate and up values: 8
    experts, 40 tokens top-2, one expert never chosen, I = 192 (three
    128-row gated tiles), every token tile and both weight variants."""
    e, inter, k, t, topk = 8, 192, 512, 40, 2
    n = 2 * inter
    if fmt == hq.HQ_FMT_MXFP4_A16:
        codes, e8 = synth.mxfp4_weights(n, k, seed=5400, experts=e)
        d = hq.hq_quant_desc_init(fmt, n, k, 32, 0, e)
        blob = torch.from_numpy(hq.hq_pack_weights_gated(d, codes, e8)).to(DEV)
        ref_fn = lambda xs, off: G.grouped_mxfp4_a16_ref(xs, off, codes.numpy(), e8.numpy())[1]
    else:
        make, ref = ((synth.w4a16_weights, G.grouped_w4a16_ref) if fmt == hq.HQ_FMT_INT4
                     else (synth.w3a16_weights, G.grouped_w3a16_ref))
        q, s, z = make(n, k, 128, True, seed=5400, experts=e)
        d = hq.hq_quant_desc_init(fmt, n, k, 128, 1, e)
        blob = torch.from_numpy(hq.hq_pack_weights_gated(d, q, s, z)).to(DEV)
        ref_fn = lambda xs, off: ref(xs, off, q.numpy(), s.numpy(), z.numpy(), 128)[1]
    logits = synth.router_logits(t, e, seed=5401)
    logits[:, 3] = -100.0
    ids = R.topk_by_logit(logits.numpy(), topk)
    _, off, src = R.permute(ids, e)
    a = synth.bf16_normal(t, k, seed=5402)
    a_sorted = R.gather_rows(_bits(a), src, topk)
    rows = t * topk
    tuning = hq.Tuning(tile_m=tile_m, variant=variant) if (tile_m or variant) else None
    h = torch.full((rows, inter), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, rows, tuning))
    a_dev = torch.from_numpy(a_sorted.view(np.int16)).view(torch.bfloat16).to(DEV)
    hq.hq_grouped_gemm_moe_swiglu(d, blob, a_dev, torch.from_numpy(off.astype(np.int32)).to(DEV), rows, h, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    check_swiglu(h, ref_fn(a_sorted, off), inter, k, f"swiglu fused fmt={fmt} tile_m={tile_m} variant={variant}")


@pytest.mark.parametrize("t", [64, 8192])
def test_grouped_swiglu_fused_full_size_sampled(t):
    """The layer's gate+up GEMM with the fused SwiGLU at the full workload
    (256 experts, top-8, hidden 7168, I = 2048), in the bench's launch
    configuration; sampled rows (at least two per non-empty expert), every
    output feature."""
    e, topk, hid, inter = 256, 8, 7168, 2048
    n = 2 * inter
    q, s, _ = synth.w4a16_weights(n, hid, 128, False, seed=5500, experts=e)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, hid, 128, 0, e)
    blob = torch.from_numpy(hq.hq_pack_weights_gated(d, q, s, None)).to(DEV)
    logits = synth.router_logits(t, e, seed=5501 + t)
    ids = R.topk_by_logit(logits.numpy(), topk)
    _, off, src = R.permute(ids, e)
    x = synth.bf16_normal(t, hid, seed=5502 + t)
    a_sorted = R.gather_rows(_bits(x), src, topk)
    rows = t * topk
    h = torch.empty(rows, inter, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, rows))
    a_dev = torch.from_numpy(a_sorted.view(np.int16)).view(torch.bfloat16).to(DEV)
    hq.hq_grouped_gemm_moe_swiglu(d, blob, a_dev, torch.from_numpy(off.astype(np.int32)).to(DEV), rows, h, ws)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    rng = np.random.default_rng(5503)
    sample = []
    for ex in range(e):
        lo, hi = int(off[ex]), int(off[ex + 1])
        if hi > lo:
            sample += sorted(set(rng.integers(lo, hi, size=2).tolist()))
    sample = np.array(sorted(set(sample)))
    # output features: first, last and one random of every 64-feature tile;
    # the oracle computes their gate rows f and up rows I + f only
    feats = np.array(sorted({f for j in range(inter // 64)
                             for f in (64 * j, 64 * j + 63, 64 * j + int(rng.integers(0, 64)))}))
    _, ref = G.grouped_w4a16_ref(a_sorted, off, q.numpy(), s.numpy(), None, 128, row_subset=sample,
                                 cols=np.concatenate([feats, inter + feats]))
    check_swiglu(h.cpu()[sample][:, feats], ref, len(feats), hid, f"swiglu fused full size T={t}")


@pytest.mark.parametrize("variant,fused", [(0, False), (2, False), (0, True), (2, True)])
def test_moe_layer_end_to_end(variant, fused):
    """Route (top-k + weights) -> permute + gather -> gate+up grouped GEMM ->
    SwiGLU -> down grouped GEMM -> weighted combine, all through the C ABI
    on one stream, against the oracle's layer (32 experts, top-4, T=64,
    hidden 1024, intermediate 256).  Routing and permutation bit-exact; the
    layer output at the GEMM tolerance, with the down GEMM's K."""
    t, e, k, hid, inter = 64, 32, 4, 1024, 256
    q1, s1, _ = synth.w4a16_weights(2 * inter, hid, 128, False, seed=3600, experts=e)
    q2, s2, _ = synth.w4a16_weights(hid, inter, 128, False, seed=3601, experts=e)
    d1 = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, 2 * inter, hid, 128, 0, e)
    d2 = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, hid, inter, 128, 0, e)
    b1 = torch.from_numpy(hq.hq_pack_weights(d1, q1, s1, None)).to(DEV)
    b2 = torch.from_numpy(hq.hq_pack_weights(d2, q2, s2, None)).to(DEV)
    logits = synth.router_logits(t, e, seed=3602)
    x = synth.bf16_normal(t, hid, seed=3603)
    tun = hq.Tuning(variant=variant) if variant else None
    # GPU layer
    ids = torch.empty(t, k, dtype=torch.int32, device=DEV)
    wts = torch.empty(t, k, dtype=torch.float32, device=DEV)
    hq.hq_moe_topk_softmax(logits.to(DEV), t, e, k, ids, wts)
    src, off, xs, st = gpu_permute(ids, e, x)
    assert st == hq.HQ_OK
    h = torch.empty(t * k, inter, dtype=torch.bfloat16, device=DEV)
    if fused:
        # gate+up weights in the gated row order, SwiGLU in the GEMM's epilogue
        b1g = torch.from_numpy(hq.hq_pack_weights_gated(d1, q1, s1, None)).to(DEV)
        ws1 = workspace(hq.hq_workspace_size(d1, t * k, tun))
        hq.hq_grouped_gemm_moe_swiglu(d1, b1g, xs, off, t * k, h, ws1, tun)
        assert hq.hq_check_device_status(ws1) == hq.HQ_OK
    else:
        c1 = _grouped(d1, b1, xs, off, t * k, 2 * inter, tun)
        hq.hq_moe_swiglu(c1, t * k, inter, h)
    c2 = _grouped(d2, b2, h, off, t * k, hid, tun)
    out = torch.empty(t, hid, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_moe_combine_workspace_size(t, k))
    hq.hq_moe_combine(c2, src, wts, t, k, hid, out, ws)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    # oracle layer
    ref, ids_ref, off_ref, src_ref = _layer_oracle(_bits(x), logits.numpy(), q1.numpy(), s1.numpy(), q2.numpy(),
                                                   s2.numpy(), k, e, inter, fused)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref) and np.array_equal(src.cpu().numpy(), src_ref)
    check_gemm(out, ref, inter, f"moe layer variant={variant} fused={fused}")
